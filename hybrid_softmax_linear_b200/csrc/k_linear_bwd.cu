// Backward of the elu+1 linear branch (model card "Video DeltaNet: ...", "Training": the
// linear branch is trained; article "VDN-MiniMax-H3 开源", 分阶段适配 A1/A2), on CUDA cores
// in fp32.  For a query row of group g with memories Num_g = S_txt + sum_{fk in mem(g)} S_fk
// and Den_g = z_txt + sum z_fk (the forward's Sf + Sb and zf + zb):
//   num = phi(q) Num_g, den = phi(q) . Den_g, o = num / den;
//   dnum = dO / den, dden = -(dO . o) / den, dphi(q) = Num_g dnum + Den_g dden,
//   dq = dphi(q) * phi'(q);
//   dNum_g = sum over the group's rows of phi(q)^T dnum, dDen_g = sum phi(q) dden;
// then back through the frame sums: dS_fk = sum of dNum_g over the groups whose memory holds
// fk, dS_txt = sum of all dNum_g (likewise dz), and per key row, with S_fk = sum phi(k)^T v:
//   dk = (dS_fk v + dz_fk) * phi'(k), dv = dS_fk^T phi(k).
// Every sum runs in a fixed order (no atomics), so a call repeats bit for bit.
#include "vdn_internal.cuh"

namespace vdn {
namespace {

constexpr int BT = 256;

__device__ __forceinline__ float phi1(float x) { return x > 0.f ? x + 1.f : expf(x); }
__device__ __forceinline__ float dphi1(float x) { return x > 0.f ? 1.f : expf(x); }

// Per (group, head): rows of the group's frames, BT / D at a time (thread t: row slot t / D,
// feature t % D).  Num_g and its transpose sit in shared memory.
template <int D>
__global__ void __launch_bounds__(BT) lin_bwd_rows_kernel(Dims d, const __nv_bfloat16 *__restrict__ q,
                                                          const float *__restrict__ dO,
                                                          const float *__restrict__ Sf, const float *__restrict__ Sb,
                                                          const float *__restrict__ zf, const float *__restrict__ zb,
                                                          const int32_t *__restrict__ gtab, float *__restrict__ dq,
                                                          float *__restrict__ dnum_out, float *__restrict__ dden_out) {
  constexpr int RS = BT / D;  // rows per pass
  extern __shared__ float sm[];
  float *Num = sm, *NumT = Num + D * D, *Den = NumT + D * D;
  float *ph = Den + D, *ov = ph + RS * D, *dn = ov + RS * D, *go = dn + RS * D;  // [RS][D] each
  const int g = blockIdx.x, h = blockIdx.y, t = threadIdx.x, rs = t / D, j = t % D;
  const int64_t DD = (int64_t)D * D, HD = (int64_t)d.H * D;
  const int64_t mo = ((int64_t)g * d.H + h) * DD;
  for (int e = t; e < D * D; e += BT) {
    const float v = Sf[mo + e] + Sb[mo + e];
    Num[e] = v;
    NumT[(e % D) * D + e / D] = v;
  }
  for (int e = t; e < D; e += BT) Den[e] = zf[((int64_t)g * d.H + h) * D + e] + zb[((int64_t)g * d.H + h) * D + e];
  __syncthreads();
  const int f0 = gtab[g * 16], f1 = gtab[g * 16 + 1];
  const int64_t r0 = (int64_t)f0 * d.T, r1 = (int64_t)f1 * d.T;
  for (int64_t rb = r0; rb < r1; rb += RS) {
    const int64_t row = rb + rs;
    const bool live = row < r1;
    const int64_t base = row * HD + (int64_t)h * D;
    float qj = 0.f, gj = 0.f;
    if (live) {
      qj = __bfloat162float(q[base + j]);
      gj = dO[base + j];
    }
    ph[rs * D + j] = live ? phi1(qj) : 0.f;
    go[rs * D + j] = gj;
    __syncthreads();
    // num_j and den (den by every thread of the slot, in the same order)
    const float *p = ph + rs * D;
    float num = 0.f, den = 0.f;
    for (int i = 0; i < D; ++i) {
      num = fmaf(p[i], Num[i * D + j], num);
      den = fmaf(p[i], Den[i], den);
    }
    const bool pos = den > 0.f;
    const float inv = pos ? 1.f / den : 0.f;
    ov[rs * D + j] = num * inv;
    const float dnj = gj * inv;
    dn[rs * D + j] = dnj;
    __syncthreads();
    float dot = 0.f;  // dO . o
    for (int i = 0; i < D; ++i) dot = fmaf(go[rs * D + i], ov[rs * D + i], dot);
    const float dden = pos ? -dot * inv : 0.f;
    // dphi_j = sum_e Num[j][e] dnum_e + Den_j dden (Num^T keeps the reads conflict-free)
    float dp = Den[j] * dden;
    for (int e = 0; e < D; ++e) dp = fmaf(NumT[e * D + j], dn[rs * D + e], dp);
    if (live) {
      dq[base + j] = dp * dphi1(qj);
      dnum_out[base + j] = dnj;
      if (j == 0) dden_out[row * d.H + h] = dden;
    }
    __syncthreads();  // the slot's rows are read before the next pass overwrites them
  }
}

// Per (group, head): dNum_g = sum over its rows of phi(q)^T dnum (each thread an R x R
// block of the D x D result in registers, rows streamed through shared memory 32 at a
// time) and dDen_g = sum phi(q) dden.
template <int D>
__global__ void __launch_bounds__(BT) lin_bwd_dnum_kernel(Dims d, const __nv_bfloat16 *__restrict__ q,
                                                          const float *__restrict__ dnum, const float *__restrict__ dden,
                                                          const int32_t *__restrict__ gtab, float *__restrict__ dN,
                                                          float *__restrict__ dZ) {
  constexpr int CH = 32, R = D / 16;  // 16 x 16 threads, R x R entries each
  __shared__ float ph[CH][D], dn[CH][D], dd[CH];
  const int g = blockIdx.x, h = blockIdx.y, t = threadIdx.x, ti = t / 16, tj = t % 16;
  const int64_t HD = (int64_t)d.H * D;
  const int f0 = gtab[g * 16], f1 = gtab[g * 16 + 1];
  const int64_t r0 = (int64_t)f0 * d.T, r1 = (int64_t)f1 * d.T;
  float acc[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.f;
  float zacc = 0.f;  // threads t < D: dDen_t
  for (int64_t rb = r0; rb < r1; rb += CH) {
    const int n = r1 - rb < CH ? (int)(r1 - rb) : CH;
    for (int e = t; e < CH * D; e += BT) {
      const int rr = e / D, c = e % D;
      const int64_t idx = (rb + rr) * HD + (int64_t)h * D + c;
      ph[rr][c] = rr < n ? phi1(__bfloat162float(q[idx])) : 0.f;
      dn[rr][c] = rr < n ? dnum[idx] : 0.f;
    }
    for (int e = t; e < CH; e += BT) dd[e] = e < n ? dden[(rb + e) * d.H + h] : 0.f;
    __syncthreads();
    for (int rr = 0; rr < CH; ++rr) {
      float a[R], b[R];
#pragma unroll
      for (int x = 0; x < R; ++x) a[x] = ph[rr][ti + 16 * x];
#pragma unroll
      for (int y = 0; y < R; ++y) b[y] = dn[rr][tj + 16 * y];
#pragma unroll
      for (int x = 0; x < R; ++x)
#pragma unroll
        for (int y = 0; y < R; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
      if (t < D) zacc = fmaf(ph[rr][t], dd[rr], zacc);
    }
    __syncthreads();
  }
  const int64_t mo = ((int64_t)g * d.H + h) * D * D;
#pragma unroll
  for (int x = 0; x < R; ++x)
#pragma unroll
    for (int y = 0; y < R; ++y) dN[mo + (int64_t)(ti + 16 * x) * D + tj + 16 * y] = acc[x][y];
  if (t < D) dZ[((int64_t)g * d.H + h) * D + t] = zacc;
}

// Per (key frame fk, head), fk == F for the text: dS = sum of dNum_g over the groups whose
// memory holds fk (every group for the text), in group order; then the frame's key rows.
template <int D>
__global__ void __launch_bounds__(BT) lin_bwd_keys_kernel(Dims d, const __nv_bfloat16 *__restrict__ k,
                                                          const __nv_bfloat16 *__restrict__ v,
                                                          const __nv_bfloat16 *__restrict__ kt,
                                                          const __nv_bfloat16 *__restrict__ vt,
                                                          const float *__restrict__ dN, const float *__restrict__ dZ,
                                                          const int32_t *__restrict__ gtab, int G,
                                                          float *__restrict__ dk, float *__restrict__ dv,
                                                          float *__restrict__ dkt, float *__restrict__ dvt) {
  constexpr int RS = BT / D;
  extern __shared__ float sm[];
  float *dS = sm, *dST = dS + D * D, *dz = dST + D * D;
  float *pk = dz + D, *vv = pk + RS * D;  // [RS][D] each
  const int fk = blockIdx.x, h = blockIdx.y, t = threadIdx.x, rs = t / D, j = t % D;
  const bool text = fk == d.F;
  const int64_t DD = (int64_t)D * D, HD = (int64_t)d.H * D;
  for (int e = t; e < D * D; e += BT) {
    float s = 0.f;
    for (int g = 0; g < G; ++g) {
      const int32_t *r = gtab + g * 16;
      const bool in = text || (fk >= r[12] && fk < r[13]) || (fk >= r[14] && fk < r[15]);
      if (in) s += dN[((int64_t)g * d.H + h) * DD + e];
    }
    dS[e] = s;
    dST[(e % D) * D + e / D] = s;
  }
  for (int e = t; e < D; e += BT) {
    float s = 0.f;
    for (int g = 0; g < G; ++g) {
      const int32_t *r = gtab + g * 16;
      const bool in = text || (fk >= r[12] && fk < r[13]) || (fk >= r[14] && fk < r[15]);
      if (in) s += dZ[((int64_t)g * d.H + h) * D + e];
    }
    dz[e] = s;
  }
  __syncthreads();
  const int ntok = text ? d.L : d.T;
  const __nv_bfloat16 *kb = text ? kt : k + (int64_t)fk * d.T * HD;
  const __nv_bfloat16 *vb = text ? vt : v + (int64_t)fk * d.T * HD;
  float *dkb = text ? dkt : dk + (int64_t)fk * d.T * HD;
  float *dvb = text ? dvt : dv + (int64_t)fk * d.T * HD;
  for (int rb = 0; rb < ntok; rb += RS) {
    const int row = rb + rs;
    const bool live = row < ntok;
    const int64_t base = (int64_t)row * HD + (int64_t)h * D;
    const float kj = live ? __bfloat162float(kb[base + j]) : 0.f;
    pk[rs * D + j] = live ? phi1(kj) : 0.f;
    vv[rs * D + j] = live ? __bfloat162float(vb[base + j]) : 0.f;
    __syncthreads();
    // dphi(k)_j = sum_e dS[j][e] v_e + dz_j; dv_j = sum_i dS[i][j] phi(k)_i
    float dpk = dz[j], dvj = 0.f;
    for (int e = 0; e < D; ++e) {
      dpk = fmaf(dST[e * D + j], vv[rs * D + e], dpk);
      dvj = fmaf(dS[e * D + j], pk[rs * D + e], dvj);
    }
    if (live) {
      dkb[base + j] = dpk * dphi1(kj);
      dvb[base + j] = dvj;
    }
    __syncthreads();
  }
}

template <int D>
cudaError_t lin_bwd_t(const Dims &d, int stage, const void *q, const void *k, const void *v, const void *kt,
                      const void *vt, const float *dO, const float *Sf, const float *Sb, const float *zf,
                      const float *zb, const int32_t *gtab, int G, float *dnum, float *dden, float *dN, float *dZ,
                      float *dq, float *dk, float *dv, float *dkt, float *dvt, cudaStream_t st) {
  constexpr int RS = BT / D;
  cudaError_t e = cudaSuccess;
  if (stage == 0) {
    const size_t smem_rows = (size_t)(2 * D * D + D + 4 * RS * D) * sizeof(float);
    e = cudaFuncSetAttribute(lin_bwd_rows_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_rows);
    if (e != cudaSuccess) return e;
    lin_bwd_rows_kernel<D><<<dim3(G, d.H), BT, smem_rows, st>>>(d, (const __nv_bfloat16 *)q, dO, Sf, Sb, zf, zb,
                                                                 gtab, dq, dnum, dden);
  } else if (stage == 1) {
    lin_bwd_dnum_kernel<D><<<dim3(G, d.H), BT, 0, st>>>(d, (const __nv_bfloat16 *)q, dnum, dden, gtab, dN, dZ);
  } else if (stage == 2) {
    const size_t smem_keys = (size_t)(2 * D * D + D + 2 * RS * D) * sizeof(float);
    e = cudaFuncSetAttribute(lin_bwd_keys_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_keys);
    if (e != cudaSuccess) return e;
    lin_bwd_keys_kernel<D><<<dim3(d.F + 1, d.H), BT, smem_keys, st>>>(
        d, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, (const __nv_bfloat16 *)kt, (const __nv_bfloat16 *)vt,
        dN, dZ, gtab, G, dk, dv, dkt, dvt);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_linear_bwd(const Dims &d, int stage, const void *q, const void *k, const void *v, const void *kt,
                              const void *vt, const float *dO, const float *Sf, const float *Sb, const float *zf,
                              const float *zb, const int32_t *gtab, int G, float *dnum, float *dden, float *dN,
                              float *dZ, float *dq, float *dk, float *dv, float *dkt, float *dvt, cudaStream_t st) {
#define VDN_LB(DD) \
  return lin_bwd_t<DD>(d, stage, q, k, v, kt, vt, dO, Sf, Sb, zf, zb, gtab, G, dnum, dden, dN, dZ, dq, dk, dv, dkt, dvt, st)
  if (d.D == 32) VDN_LB(32);
  if (d.D == 64) VDN_LB(64);
  if (d.D == 128) VDN_LB(128);
#undef VDN_LB
  return cudaErrorInvalidValue;
}

}  // namespace vdn
