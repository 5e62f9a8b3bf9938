// CUDA-core kernels: the float32 path of every step, and the bf16 path of the steps
// that are bound by HBM traffic.  All accumulate in float32.
#include "vdn_internal.cuh"

namespace vdn {

constexpr unsigned FULL = 0xffffffffu;
constexpr float LN2 = 0.69314718055994530942f;

__device__ __forceinline__ float warp_max(float x) {
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
  return x;
}

// 8 consecutive elements (16 B for bf16, 2 x 16 B for float) as float.
__device__ __forceinline__ void load8(const float *p, float *o) {
  float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *o) {
  uint4 u = *reinterpret_cast<const uint4 *>(p);
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    o[2 * i] = f.x; o[2 * i + 1] = f.y;
  }
}

// ------------------------------------------------------------------ softmax (SIMT)
// One warp per (video query row, head).  Keys are walked in batches of 32, one key per
// lane for the score, then the batch's probabilities are broadcast lane by lane for
// the P.V update where each lane owns D/32 output columns.
template <typename T, int D>
__global__ void __launch_bounds__(256) softmax_simt_kernel(Dims d, const T *__restrict__ q, const T *__restrict__ k,
                                                           const T *__restrict__ v, const T *__restrict__ kt,
                                                           const T *__restrict__ vt, float scale_log2,
                                                           T *__restrict__ o, float *__restrict__ lse,
                                                           const int32_t *__restrict__ ftab,
                                                           const int32_t *__restrict__ gtab) {
  constexpr int WARPS = 8, NC = D / 32;
  __shared__ float qs[WARPS][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * WARPS + warp;
  const int h = blockIdx.y;
  if (row >= d.Nv()) return;
  const int64_t HD = (int64_t)d.H * D;
  for (int i = lane; i < D; i += 32) qs[warp][i] = to_f(q[row * HD + h * D + i]);
  __syncwarp();
  const int f = (int)(row / d.T);
  const int32_t *gr = gtab + ftab[f * 8] * 16;
  float m = -INFINITY, l = 0.f, acc[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) acc[c] = 0.f;
  for (int s = 0; s < gr[2]; ++s) {
    const int lo = gr[4 + 2 * s], hi = gr[5 + 2 * s];
    for (int base = lo; base < hi; base += 32) {
      const int j = base + lane;
      float sc = -INFINITY;
      if (j < hi) {
        const T *kr = j < d.L ? kt + (int64_t)j * HD + h * D : k + (int64_t)(j - d.L) * HD + h * D;
        float dot = 0.f;
#pragma unroll 4
        for (int i = 0; i < D; i += 8) {
          float x[8];
          load8(kr + i, x);
#pragma unroll
          for (int e = 0; e < 8; ++e) dot = fmaf(qs[warp][i + e], x[e], dot);
        }
        sc = dot * scale_log2;
      }
      const float mn = fmaxf(m, warp_max(sc));
      const float alpha = exp2f(m - mn);
      const float p = j < hi ? exp2f(sc - mn) : 0.f;
      l = l * alpha + p;
#pragma unroll
      for (int c = 0; c < NC; ++c) acc[c] *= alpha;
      const int nvalid = min(32, hi - base);
      for (int t = 0; t < nvalid; ++t) {
        const float pt = __shfl_sync(FULL, p, t);
        const int jt = base + t;
        const T *vr = jt < d.L ? vt + (int64_t)jt * HD + h * D : v + (int64_t)(jt - d.L) * HD + h * D;
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[c] = fmaf(pt, to_f(vr[lane + 32 * c]), acc[c]);
      }
      m = mn;
    }
  }
  l = warp_sum(l);
  const float inv = 1.f / l;
#pragma unroll
  for (int c = 0; c < NC; ++c) o[row * HD + h * D + lane + 32 * c] = from_f<T>(acc[c] * inv);
  if (lse != nullptr && lane == 0) lse[row * d.H + h] = (m + log2f(l)) * LN2;
}

template <typename T, int D>
static cudaError_t softmax_simt_t(const Dims &d, const void *q, const void *k, const void *v, const void *kt,
                                  const void *vt, float sl2, void *o, float *lse, const int32_t *ftab,
                                  const int32_t *gtab, cudaStream_t st) {
  dim3 grid((unsigned)((d.Nv() + 7) / 8), d.H);
  softmax_simt_kernel<T, D><<<grid, 256, 0, st>>>(d, (const T *)q, (const T *)k, (const T *)v, (const T *)kt,
                                                  (const T *)vt, sl2, (T *)o, lse, ftab, gtab);
  return cudaGetLastError();
}

cudaError_t launch_softmax_simt(const Dims &d, vdn_dtype dt, const void *q, const void *k, const void *v,
                                const void *kt, const void *vt, float sl2, void *o, float *lse, char *ws,
                                const WsPlan &p, cudaStream_t st) {
  const int32_t *ftab = (const int32_t *)(ws + p.ftab), *gtab = (const int32_t *)(ws + p.gtab);
#define VDN_SM(T, DD) return softmax_simt_t<T, DD>(d, q, k, v, kt, vt, sl2, o, lse, ftab, gtab, st)
  if (dt == VDN_F32) {
    if (d.D == 32) VDN_SM(float, 32);
    if (d.D == 64) VDN_SM(float, 64);
    if (d.D == 128) VDN_SM(float, 128);
  } else if (dt == VDN_BF16) {
    if (d.D == 32) VDN_SM(__nv_bfloat16, 32);
    if (d.D == 64) VDN_SM(__nv_bfloat16, 64);
    if (d.D == 128) VDN_SM(__nv_bfloat16, 128);
  }
#undef VDN_SM
  return cudaErrorInvalidValue;
}

// Block-wide maximum of a non-negative float (every thread passes its own), then one
// atomicMax on the float's bit pattern (which orders like the value for non-negative
// floats) by thread 0.  red: shared scratch of blockDim.x / 32 floats.  Every thread of the
// block must call it.
__device__ __forceinline__ void block_amax_to(float m, float *red, uint32_t *dst) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t = fmaxf(t, red[w]);
    atomicMax(dst, __float_as_uint(t));
  }
}

// ------------------------------------------------------------------ per-frame states
// Block per (frame or text, head).  Tokens are staged 32 at a time in shared memory as
// float (phi(k) or the L2-normalised key for the delta text init, and v); thread t owns
// the D/16 x D/16 entries (i, j) = (t/16 + 16 r, t%16 + 16 c) of the D x D sum.
template <typename T, int D>
__global__ void __launch_bounds__(256) state_build_kernel(Dims d, const T *__restrict__ k, const T *__restrict__ v,
                                                          const T *__restrict__ kt, const T *__restrict__ vt,
                                                          float *__restrict__ S, float *__restrict__ z,
                                                          float *__restrict__ St, float *__restrict__ zt,
                                                          int nframes, int normalise_rows, uint32_t *__restrict__ amax) {
  constexpr int R = D / 16, TK = 32;
  __shared__ float ks[TK][D], vs[TK][D];
  const int h = blockIdx.y, tid = threadIdx.x;
  const bool text = (int)blockIdx.x == nframes;  // the block after the frames is the text
  const int ntok = text ? d.L : d.T;
  const int64_t HD = (int64_t)d.H * D;
  const T *kb = text ? kt : k + (int64_t)blockIdx.x * d.T * HD;
  const T *vb = text ? vt : v + (int64_t)blockIdx.x * d.T * HD;
  float acc[R][R];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int c = 0; c < R; ++c) acc[r][c] = 0.f;
  float zacc = 0.f, ak = 0.f, av = 0.f;  // ak, av: max |k|, |v| of the rows read (amax)
  const int i0 = tid >> 4, j0 = tid & 15;
  for (int t0 = 0; t0 < ntok; t0 += TK) {
    const int nt = min(TK, ntok - t0);
    for (int e = tid; e < TK * D; e += 256) {
      const int t = e / D, i = e % D;
      float kx = 0.f, vx = 0.f;
      if (t < nt) {
        kx = to_f(kb[(int64_t)(t0 + t) * HD + h * D + i]);
        vx = to_f(vb[(int64_t)(t0 + t) * HD + h * D + i]);
        ak = fmaxf(ak, fabsf(kx));
        av = fmaxf(av, fabsf(vx));
        if (!normalise_rows) kx = phi_elu1(kx);
      }
      ks[t][i] = kx; vs[t][i] = vx;
    }
    __syncthreads();
    if (normalise_rows) {  // delta text init: k_hat = k / ||k||, a zero row stays zero
      const int warp = tid >> 5, lane = tid & 31;
      for (int t = warp; t < nt; t += 8) {
        float ss = 0.f;
        for (int i = lane; i < D; i += 32) ss += ks[t][i] * ks[t][i];
        ss = warp_sum(ss);
        const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
        for (int i = lane; i < D; i += 32) ks[t][i] *= inv;
      }
      __syncthreads();
    }
    for (int t = 0; t < nt; ++t) {
      float a[R], b[R];
#pragma unroll
      for (int r = 0; r < R; ++r) a[r] = ks[t][i0 + 16 * r];
#pragma unroll
      for (int c = 0; c < R; ++c) b[c] = vs[t][j0 + 16 * c];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int c = 0; c < R; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
      if (tid < D) zacc += ks[t][tid];
    }
    __syncthreads();
  }
  float *So = text ? St + (int64_t)h * D * D : S + ((int64_t)blockIdx.x * d.H + h) * D * D;
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int c = 0; c < R; ++c) So[(i0 + 16 * r) * D + j0 + 16 * c] = acc[r][c];
  float *zo = text ? zt : z;
  if (zo != nullptr && tid < D) zo[(text ? (int64_t)h * D : ((int64_t)blockIdx.x * d.H + h) * D) + tid] = zacc;
  if (amax != nullptr && text) {  // block-uniform: the delta text init's max |k|, |v| per head
    __shared__ float red[256 / 32];
    block_amax_to(ak, red, amax + d.H + h);
    block_amax_to(av, red, amax + 2 * d.H + h);
  }
}

// Delta-rule frame statistics: kbar = mean key (L2-normalised), vbar = mean value.
template <typename T, int D>
__global__ void __launch_bounds__(D) delta_stats_kernel(Dims d, const T *__restrict__ k, const T *__restrict__ v,
                                                        float *__restrict__ kbar, float *__restrict__ vbar) {
  __shared__ float red[D / 32];
  const int f = blockIdx.x, h = blockIdx.y, i = threadIdx.x;
  const int64_t HD = (int64_t)d.H * D;
  const T *kb = k + (int64_t)f * d.T * HD + h * D + i;
  const T *vb = v + (int64_t)f * d.T * HD + h * D + i;
  float sk = 0.f, sv = 0.f;
  for (int t = 0; t < d.T; ++t) { sk += to_f(kb[t * HD]); sv += to_f(vb[t * HD]); }
  sk /= (float)d.T; sv /= (float)d.T;
  float ss = warp_sum(sk * sk);
  if ((i & 31) == 0) red[i >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < D / 32; ++w) tot += red[w];
  const float inv = tot > 0.f ? rsqrtf(tot) : 0.f;
  kbar[((int64_t)f * d.H + h) * D + i] = sk * inv;
  vbar[((int64_t)f * d.H + h) * D + i] = sv;
}

// Frame means for the delta rule, bf16 and D = 128: 16 threads cover a token row of one
// head with 16-byte loads (8 values each) and the block's 16 token slices are summed
// through shared memory; then kbar is L2-normalised.
constexpr int DS_THREADS = 256, DS_SLICES = DS_THREADS / 16;
// amax (optional): the per-head max |k| and |v| of these rows go into amax[H + h] and
// amax[2H + h] (float bits), as a by-product of reading them
__global__ void __launch_bounds__(DS_THREADS) delta_stats_bf16_kernel(Dims d, const __nv_bfloat16 *__restrict__ k,
                                                                      const __nv_bfloat16 *__restrict__ v,
                                                                      float *__restrict__ kbar,
                                                                      float *__restrict__ vbar,
                                                                      uint32_t *__restrict__ amax) {
  constexpr int D = 128;
  __shared__ float acc[2][DS_SLICES][D];
  __shared__ float nrm;
  const int f = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int c8 = (tid & 15) * 8, sl = tid >> 4;
  const int64_t HD = (int64_t)d.H * D;
  const __nv_bfloat16 *kb = k + (int64_t)f * d.T * HD + h * D + c8;
  const __nv_bfloat16 *vb = v + (int64_t)f * d.T * HD + h * D + c8;
  float sk[8], sv[8], ak = 0.f, av = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) sk[e] = sv[e] = 0.f;
#pragma unroll 4
  for (int t = sl; t < d.T; t += DS_SLICES) {
    float a[8], b[8];
    load8(kb + (int64_t)t * HD, a);
    load8(vb + (int64_t)t * HD, b);
#pragma unroll
    for (int e = 0; e < 8; ++e) { sk[e] += a[e]; sv[e] += b[e]; }
    if (amax != nullptr) {
#pragma unroll
      for (int e = 0; e < 8; ++e) { ak = fmaxf(ak, fabsf(a[e])); av = fmaxf(av, fabsf(b[e])); }
    }
  }
  if (amax != nullptr) {  // block-uniform
    __shared__ float red[DS_THREADS / 32];
    block_amax_to(ak, red, amax + d.H + h);
    block_amax_to(av, red, amax + 2 * d.H + h);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) { acc[0][sl][c8 + e] = sk[e]; acc[1][sl][c8 + e] = sv[e]; }
  __syncthreads();
  float mk = 0.f, mv = 0.f;
  if (tid < D) {
#pragma unroll
    for (int q = 0; q < DS_SLICES; ++q) { mk += acc[0][q][tid]; mv += acc[1][q][tid]; }
    mk /= (float)d.T;
    mv /= (float)d.T;
  }
  const float ss = warp_sum(tid < D ? mk * mk : 0.f);
  __syncthreads();  // acc is reused for the per-warp sums of squares
  if ((tid & 31) == 0) acc[0][0][tid >> 5] = ss;
  __syncthreads();
  if (tid == 0) {
    float tot = 0.f;
    for (int w = 0; w < DS_THREADS / 32; ++w) tot += acc[0][0][w];
    nrm = tot > 0.f ? rsqrtf(tot) : 0.f;
  }
  __syncthreads();
  if (tid < D) {
    kbar[((int64_t)f * d.H + h) * D + tid] = mk * nrm;
    vbar[((int64_t)f * d.H + h) * D + tid] = mv;
  }
}

template <typename T, int D>
static cudaError_t state_build_t(const Dims &d, vdn_lin_kind kind, const void *k, const void *v, const void *kt,
                                 const void *vt, float *S, float *z, float *St, float *zt, cudaStream_t st,
                                 uint32_t *amax) {
  if (kind == VDN_LIN_ELU1) {
    state_build_kernel<T, D><<<dim3(d.F + 1, d.H), 256, 0, st>>>(d, (const T *)k, (const T *)v, (const T *)kt,
                                                                 (const T *)vt, S, z, St, zt, d.F, 0, nullptr);
    return cudaGetLastError();
  }
  if constexpr (D == 128 && sizeof(T) == 2)
    delta_stats_bf16_kernel<<<dim3(d.F, d.H), DS_THREADS, 0, st>>>(d, (const T *)k, (const T *)v, S, z, amax);
  else
    delta_stats_kernel<T, D><<<dim3(d.F, d.H), D, 0, st>>>(d, (const T *)k, (const T *)v, S, z);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // text init only: one block per head, with L2-normalised text keys
  state_build_kernel<T, D><<<dim3(1, d.H), 256, 0, st>>>(d, (const T *)k, (const T *)v, (const T *)kt,
                                                         (const T *)vt, nullptr, nullptr, St, nullptr, 0, 1, amax);
  return cudaGetLastError();
}

cudaError_t launch_state_build(const Dims &d, vdn_lin_kind kind, vdn_dtype dt, const void *k, const void *v,
                               const void *kt, const void *vt, float *S, float *z, float *St, float *zt,
                               cudaStream_t st, uint32_t *amax) {
  // the amax by-product exists on the delta rule's bf16, D = 128 path only
  if (amax != nullptr && !(kind == VDN_LIN_DELTA && dt == VDN_BF16 && d.D == 128)) return cudaErrorInvalidValue;
#define VDN_SB(T, DD) return state_build_t<T, DD>(d, kind, k, v, kt, vt, S, z, St, zt, st, amax)
  if (dt == VDN_F32) {
    if (d.D == 32) VDN_SB(float, 32);
    if (d.D == 64) VDN_SB(float, 64);
    if (d.D == 128) VDN_SB(float, 128);
  } else if (dt == VDN_BF16) {
    if (d.D == 32) VDN_SB(__nv_bfloat16, 32);
    if (d.D == 64) VDN_SB(__nv_bfloat16, 64);
    if (d.D == 128) VDN_SB(__nv_bfloat16, 128);
  }
#undef VDN_SB
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ window-offset scan
// Group g's forward memory is the sum over frames [1, e_g) (e_g = fwd_hi, or 1 when
// empty), its backward memory the sum over [b_g, F-1) (b_g = bwd_lo, or F-1 when empty);
// both start from half the text state.  One thread owns 4 consecutive entries of the
// flattened [D*D | D] state of one head and walks the frames once per direction,
// writing each group's memory when the walk reaches its boundary.
__global__ void __launch_bounds__(256) scan_elu1_kernel(Dims d, const float *__restrict__ S,
                                                        const float *__restrict__ z, const float *__restrict__ St,
                                                        const float *__restrict__ zt, float *__restrict__ Sf,
                                                        float *__restrict__ Sb, float *__restrict__ zf,
                                                        float *__restrict__ zb, const int32_t *__restrict__ gtab,
                                                        int G) {
  const int D = d.D, h = blockIdx.y, dir = blockIdx.z;
  const int64_t DD = (int64_t)D * D;
  const int64_t e = ((int64_t)blockIdx.x * 256 + threadIdx.x) * 4;
  if (e >= DD + D) return;
  const bool isz = e >= DD;
  const int64_t off = isz ? e - DD : e;
  const int64_t per = isz ? D : DD;         // entries per (frame, head)
  const float *src = isz ? z : S;
  const float *txt = (isz ? zt : St) + h * per + off;
  float *dst = dir == 0 ? (isz ? zf : Sf) : (isz ? zb : Sb);
  float4 t4 = *reinterpret_cast<const float4 *>(txt);
  float4 acc = make_float4(0.5f * t4.x, 0.5f * t4.y, 0.5f * t4.z, 0.5f * t4.w);
  auto add = [&](int f) {
    float4 s4 = *reinterpret_cast<const float4 *>(src + ((int64_t)f * d.H + h) * per + off);
    acc.x += s4.x; acc.y += s4.y; acc.z += s4.z; acc.w += s4.w;
  };
  auto emit = [&](int f) {
    for (int g = 0; g < G; ++g) {
      const int32_t *r = gtab + g * 16;
      const int bound = dir == 0 ? (r[13] > r[12] ? r[13] : 1) : (r[15] > r[14] ? r[14] : d.F - 1);
      if (bound == f) *reinterpret_cast<float4 *>(dst + ((int64_t)g * d.H + h) * per + off) = acc;
    }
  };
  if (dir == 0) {
    for (int f = 1;; ++f) {
      emit(f);
      if (f > d.F - 2) break;
      add(f);
    }
  } else {
    for (int f = d.F - 1;; --f) {
      emit(f);
      if (f - 1 < 1) break;
      add(f - 1);
    }
  }
}

// Delta-rule scan.  The update S <- (I - beta kbar kbar^T) S + beta kbar vbar^T acts on each
// column of S separately (u_j = kbar . S[:, j]; S[:, j] += beta kbar (vbar_j - u_j)), so a
// block owns DCB columns of one head's state in one direction, walks the frames in order and
// emits its slice of every group's memory when the walk reaches the group's boundary.  The
// frame means of the head and the block's value columns are staged in shared memory first;
// each thread keeps 8 state entries (one column, 8 rows) in registers, and a step needs one
// block barrier (the column sums u are reduced through a parity-double-buffered array).
constexpr int DCB = 16;            // state columns per block
constexpr int DELTA_THREADS = 256;

template <int D>
__global__ void __launch_bounds__(DELTA_THREADS) scan_delta_kernel(Dims d, const float *__restrict__ kbar,
                                                                   const float *__restrict__ vbar,
                                                                   const float *__restrict__ St,
                                                                   const float *__restrict__ beta,
                                                                   float *__restrict__ Sf, float *__restrict__ Sb,
                                                                   const int32_t *__restrict__ gtab, int G) {
  constexpr int RPT = D / (2 * DELTA_THREADS / 32);  // rows per thread: 16 row groups of 8 (D = 128)
  static_assert(RPT * 2 * (DELTA_THREADS / 32) == D, "row split");
  extern __shared__ float sm[];
  const int h = blockIdx.x, dir = blockIdx.y, j0 = blockIdx.z * DCB;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int col = lane & 15;                       // column j0 + col
  const int rg = (lane >> 4) + 2 * warp;           // row group: rows rg * RPT .. + RPT - 1
  const int F = d.F;
  float *kb = sm;                                  // [F][D]
  float *vb = kb + (size_t)F * D;                  // [F][DCB]
  float *bt = vb + (size_t)F * DCB;                // [F]
  float *part = bt + F;                            // [2][8 warps][DCB]
  int *bound = reinterpret_cast<int *>(part + 2 * (DELTA_THREADS / 32) * DCB);  // [G]
  int *any = bound + G;                            // [F]: some group's memory ends at this frame
  for (int e = tid; e < F * D; e += DELTA_THREADS) kb[e] = kbar[((int64_t)(e / D) * d.H + h) * D + e % D];
  for (int e = tid; e < F * DCB; e += DELTA_THREADS)
    vb[e] = vbar[((int64_t)(e / DCB) * d.H + h) * D + j0 + e % DCB];
  for (int e = tid; e < F; e += DELTA_THREADS) bt[e] = beta[(int64_t)e * d.H + h];
  for (int e = tid; e < F; e += DELTA_THREADS) any[e] = 0;
  __syncthreads();
  for (int g = tid; g < G; g += DELTA_THREADS) {
    const int32_t *r = gtab + g * 16;
    const int b = dir == 0 ? (r[13] > r[12] ? r[13] : 1) : (r[15] > r[14] ? r[14] : F - 1);
    bound[g] = b;
    any[b] = 1;
  }
  float sreg[RPT];
#pragma unroll
  for (int m = 0; m < RPT; ++m) sreg[m] = 0.5f * St[((int64_t)h * D + rg * RPT + m) * D + j0 + col];
  __syncthreads();
  float *dst = dir == 0 ? Sf : Sb;
  auto emit = [&](int f) {
    if (f < F && !any[f]) return;  // the forward walk ends at frame F-1 (frame 1 when F = 1)
    for (int g = 0; g < G; ++g)
      if (bound[g] == f) {
#pragma unroll
        for (int m = 0; m < RPT; ++m) dst[(((int64_t)g * d.H + h) * D + rg * RPT + m) * D + j0 + col] = sreg[m];
      }
  };
  int par = 0;
  auto step = [&](int f) {
    const float *k = kb + (size_t)f * D + rg * RPT;
    float u = 0.f;
#pragma unroll
    for (int m = 0; m < RPT; ++m) u = fmaf(k[m], sreg[m], u);
    u += __shfl_xor_sync(0xffffffffu, u, 16);      // the two row groups of this warp
    float *pp = part + par * (DELTA_THREADS / 32) * DCB;
    if (lane < 16) pp[warp * DCB + col] = u;
    __syncthreads();
    float uj = 0.f;
#pragma unroll
    for (int w = 0; w < DELTA_THREADS / 32; ++w) uj += pp[w * DCB + col];
    const float c = bt[f] * (vb[(size_t)f * DCB + col] - uj);
#pragma unroll
    for (int m = 0; m < RPT; ++m) sreg[m] = fmaf(k[m], c, sreg[m]);
    par ^= 1;
  };
  if (dir == 0) {
    for (int f = 1;; ++f) {
      emit(f);
      if (f > F - 2) break;
      step(f);
    }
  } else {
    for (int f = F - 1;; --f) {
      emit(f);
      if (f - 1 < 1) break;
      step(f - 1);
    }
  }
}

// Fallback for head dims without the column split: one block per (head, direction), the
// whole D x D state in shared memory.
__global__ void __launch_bounds__(256) scan_delta_small_kernel(Dims d, const float *__restrict__ kbar,
                                                               const float *__restrict__ vbar,
                                                               const float *__restrict__ St,
                                                               const float *__restrict__ beta, float *__restrict__ Sf,
                                                               float *__restrict__ Sb,
                                                               const int32_t *__restrict__ gtab, int G) {
  extern __shared__ float sm[];
  const int D = d.D, h = blockIdx.x, dir = blockIdx.y, tid = threadIdx.x;
  const int DD = D * D;
  float *Ss = sm, *kb = sm + DD, *vb = kb + D, *u = vb + D;
  for (int e = tid; e < DD; e += 256) Ss[e] = 0.5f * St[(int64_t)h * DD + e];
  __syncthreads();
  float *dst = dir == 0 ? Sf : Sb;
  auto emit = [&](int f) {
    for (int g = 0; g < G; ++g) {
      const int32_t *r = gtab + g * 16;
      const int bound = dir == 0 ? (r[13] > r[12] ? r[13] : 1) : (r[15] > r[14] ? r[14] : d.F - 1);
      if (bound == f)
        for (int e = tid; e < DD; e += 256) dst[((int64_t)g * d.H + h) * DD + e] = Ss[e];
    }
  };
  auto step = [&](int f) {
    for (int i = tid; i < D; i += 256) {
      kb[i] = kbar[((int64_t)f * d.H + h) * D + i];
      vb[i] = vbar[((int64_t)f * d.H + h) * D + i];
    }
    __syncthreads();
    for (int j = tid; j < D; j += 256) {
      float s = 0.f;
      for (int i = 0; i < D; ++i) s = fmaf(kb[i], Ss[i * D + j], s);
      u[j] = s;
    }
    __syncthreads();
    const float b = beta[(int64_t)f * d.H + h];
    for (int e = tid; e < DD; e += 256) {
      const int i = e / D, j = e % D;
      Ss[e] = fmaf(b * kb[i], vb[j] - u[j], Ss[e]);
    }
    __syncthreads();
  };
  if (dir == 0) {
    for (int f = 1;; ++f) {
      emit(f);
      if (f > d.F - 2) break;
      step(f);
    }
  } else {
    for (int f = d.F - 1;; --f) {
      emit(f);
      if (f - 1 < 1) break;
      step(f - 1);
    }
  }
}

// Segmented scan of the ELU1 memories.  A block owns 128 consecutive entries (32 lanes x
// float4) of the flattened [D*D | D] state of one head.  Its warps first sum the frames
// of each segment (the frames between two consecutive memory boundaries; eight loads in
// flight per lane), then warp 0 forms the exclusive prefix sums and warp 1 the suffix
// sums over the segments, and every group's memories are read off those:
// S_fwd = S_txt/2 + prefix[ie_g], S_bwd = S_txt/2 + suffix[ib_g].  With SUM the block
// stores S_fwd + S_bwd in bf16 and z_fwd + z_bwd in float, the operands of the
// tensor-core read, instead of the four float memories.
constexpr int SCAN_THREADS = 256;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

template <bool SUM>
__global__ void __launch_bounds__(SCAN_THREADS) scan_seg_kernel(Dims d, const float *__restrict__ S,
                                                                const float *__restrict__ z,
                                                                const float *__restrict__ St,
                                                                const float *__restrict__ zt, float *__restrict__ Sf,
                                                                float *__restrict__ Sb, float *__restrict__ zf,
                                                                float *__restrict__ zb,
                                                                __nv_bfloat16 *__restrict__ ssum,
                                                                float *__restrict__ zsum,
                                                                const int32_t *__restrict__ splan, int gcap,
                                                                DevStatus *stat) {
  extern __shared__ float4 sm4[];
  const int nseg = splan[0], G = splan[1];
  float4 *seg = sm4, *pre = sm4 + nseg * 32, *suf = pre + (nseg + 1) * 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int D = d.D, h = blockIdx.y;
  const int64_t DD = (int64_t)D * D;
  const int64_t c0 = (int64_t)blockIdx.x * 128;
  const bool isz = c0 >= DD;  // D*D is a multiple of 128: a block never straddles S and z
  const int64_t per = isz ? D : DD;
  const int64_t off = (isz ? c0 - DD : c0) + lane * 4;
  const bool valid = off < per;
  const float *src = (isz ? z : S) + h * per + off;
  const int64_t fstride = (int64_t)d.H * per;
  const int32_t *bnd = splan + 4;
  for (int j = warp; j < nseg; j += SCAN_THREADS / 32) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    // range-check build: segment bounds inside the frames the memories may hold
    if (valid && in_range(stat, bnd[j] - 1, d.F - 2, K_SCAN, 1) && in_range(stat, bnd[j + 1] - 2, d.F - 2, K_SCAN, 2)) {
      const int hi = bnd[j + 1];
      // eight frames per round trip: a segment of up to eight frames costs one memory latency
      for (int f = bnd[j]; f < hi; f += 8) {
        float4 x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          x[k] = f + k < hi ? __ldg(reinterpret_cast<const float4 *>(src + (int64_t)(f + k) * fstride))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        a = f4add(a, f4add(f4add(x[0], x[1]), f4add(x[2], x[3])));
        b = f4add(b, f4add(f4add(x[4], x[5]), f4add(x[6], x[7])));
      }
    }
    seg[j * 32 + lane] = f4add(a, b);
  }
  // the text state's entries, loaded while the segments are summed
  const float4 t = valid ? *reinterpret_cast<const float4 *>((isz ? zt : St) + h * per + off)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  // prefix (warp 0) and suffix (warp 1) sums over the segments, in segment order; eight
  // segments' loads are issued ahead of their chain of adds
  if (warp == 0) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int j = 0;
    for (; j + 8 <= nseg; j += 8) {
      float4 x[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = seg[(j + k) * 32 + lane];
#pragma unroll
      for (int k = 0; k < 8; ++k) { pre[(j + k) * 32 + lane] = acc; acc = f4add(acc, x[k]); }
    }
    for (; j < nseg; ++j) { pre[j * 32 + lane] = acc; acc = f4add(acc, seg[j * 32 + lane]); }
    pre[nseg * 32 + lane] = acc;
  } else if (warp == 1) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    suf[nseg * 32 + lane] = acc;
    int j = nseg - 1;
    for (; j - 8 >= -1; j -= 8) {
      float4 x[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = seg[(j - k) * 32 + lane];
#pragma unroll
      for (int k = 0; k < 8; ++k) { acc = f4add(acc, x[k]); suf[(j - k) * 32 + lane] = acc; }
    }
    for (; j >= 0; --j) { acc = f4add(acc, seg[j * 32 + lane]); suf[j * 32 + lane] = acc; }
  }
  __syncthreads();
  if (!valid) return;
  const int32_t *ie = splan + splan_ie(d.F), *ib = splan + splan_ib(d.F, gcap);
  for (int g = warp; g < G; g += SCAN_THREADS / 32) {
    if (!(in_range(stat, g, gcap, K_SCAN, 3) && in_range(stat, ie[g], nseg + 1, K_SCAN, 4) &&
          in_range(stat, ib[g], nseg + 1, K_SCAN, 5)))
      continue;
    const float4 pf = pre[ie[g] * 32 + lane], sb = suf[ib[g] * 32 + lane];
    const int64_t o = ((int64_t)g * d.H + h) * per + off;
    if (SUM) {
      const float4 v = f4add(t, f4add(pf, sb));
      if (isz) {
        *reinterpret_cast<float4 *>(zsum + o) = v;
      } else {
        uint2 u;
        u.x = pack_bf16x2(v.x, v.y);
        u.y = pack_bf16x2(v.z, v.w);
        *reinterpret_cast<uint2 *>(ssum + o) = u;
      }
    } else {
      const float4 ht = make_float4(0.5f * t.x, 0.5f * t.y, 0.5f * t.z, 0.5f * t.w);
      *reinterpret_cast<float4 *>((isz ? zf : Sf) + o) = f4add(ht, pf);
      *reinterpret_cast<float4 *>((isz ? zb : Sb) + o) = f4add(ht, sb);
    }
  }
}

template <bool SUM>
cudaError_t launch_scan_seg(const Dims &d, const float *S, const float *z, const float *St, const float *zt,
                            float *Sf, float *Sb, float *zf, float *zb, __nv_bfloat16 *ssum, float *zsum,
                            char *ws, const WsPlan &p, int nseg, cudaStream_t st) {
  const size_t smem = (size_t)(3 * nseg + 2) * 32 * sizeof(float4);
  cudaError_t e = cudaFuncSetAttribute(scan_seg_kernel<SUM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t DD = (int64_t)d.D * d.D;
  dim3 grid((unsigned)(DD / 128 + (d.D + 127) / 128), d.H);
  scan_seg_kernel<SUM><<<grid, SCAN_THREADS, smem, st>>>(d, S, z, St, zt, Sf, Sb, zf, zb, ssum, zsum,
                                                          (const int32_t *)(ws + p.splan), max_groups(d.F, d.C),
                                                          (DevStatus *)(ws + p.status));
  return cudaGetLastError();
}

cudaError_t launch_state_scan_sum(const Dims &d, const float *S, const float *z, const float *St, const float *zt,
                                  char *ws, const WsPlan &p, cudaStream_t st) {
  const int nseg = host_scan_segments(d.F, d.T, d.C, d.L);
  if (nseg > SCAN_SEG_MAX) return cudaErrorInvalidValue;
  return launch_scan_seg<true>(d, S, z, St, zt, nullptr, nullptr, nullptr, nullptr,
                               (__nv_bfloat16 *)(ws + p.ssum), (float *)(ws + p.zsum), ws, p, nseg, st);
}

cudaError_t launch_state_scan(const Dims &d, vdn_lin_kind kind, const float *S, const float *z, const float *St,
                              const float *zt, const float *beta, float *Sf, float *Sb, float *zf, float *zb,
                              char *ws, const WsPlan &p, cudaStream_t st) {
  const int32_t *gtab = (const int32_t *)(ws + p.gtab);
  const int G = host_group_count(d);
  if (kind == VDN_LIN_ELU1) {
    const int nseg = host_scan_segments(d.F, d.T, d.C, d.L);
    if (nseg <= SCAN_SEG_MAX)
      return launch_scan_seg<false>(d, S, z, St, zt, Sf, Sb, zf, zb, nullptr, nullptr, ws, p, nseg, st);
    const int64_t n4 = ((int64_t)d.D * d.D + d.D) / 4;
    dim3 grid((unsigned)((n4 + 255) / 256), d.H, 2);
    scan_elu1_kernel<<<grid, 256, 0, st>>>(d, S, z, St, zt, Sf, Sb, zf, zb, gtab, G);
    return cudaGetLastError();
  }
  // column-split recurrence for D = 128 while the frame means fit in shared memory
  const size_t smem_cols = ((size_t)d.F * (d.D + DCB + 1) + 2 * (DELTA_THREADS / 32) * DCB) * sizeof(float) +
                           ((size_t)max_groups(d.F, d.C) + d.F) * sizeof(int);
  if (d.D == 128 && smem_cols <= 200 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(scan_delta_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_cols);
    if (e != cudaSuccess) return e;
    scan_delta_kernel<128><<<dim3(d.H, 2, 128 / DCB), DELTA_THREADS, smem_cols, st>>>(d, S, z, St, beta, Sf, Sb, gtab,
                                                                                      G);
    return cudaGetLastError();
  }
  size_t smem = ((size_t)d.D * d.D + 3 * d.D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(scan_delta_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  scan_delta_small_kernel<<<dim3(d.H, 2), 256, smem, st>>>(d, S, z, St, beta, Sf, Sb, gtab, G);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ linear read
// Block per (query tile, head) from the tile list (a tile never straddles a group).
// The group's summed memory sits in shared memory; each warp takes rows, each lane D/32
// output columns.
template <typename T, int D>
__global__ void __launch_bounds__(256) linear_read_kernel(Dims d, int delta, const T *__restrict__ q,
                                                          const float *__restrict__ Sf, const float *__restrict__ Sb,
                                                          const float *__restrict__ zf, const float *__restrict__ zb,
                                                          T *__restrict__ o, const int32_t *__restrict__ tiles) {
  extern __shared__ float sm[];
  constexpr int NC = D / 32;
  float *Ss = sm, *zs = sm + D * D, *qs = zs + D;  // qs [8][D]
  const int h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t *tr = tiles + (int64_t)blockIdx.x * TILE_REC;
  const int g = tr[0];
  const int64_t r0 = tr[1], r1 = tr[2];
  const float *sf = Sf + ((int64_t)g * d.H + h) * D * D, *sb = Sb + ((int64_t)g * d.H + h) * D * D;
  for (int e = tid * 4; e < D * D; e += 256 * 4) {
    float4 a = *reinterpret_cast<const float4 *>(sf + e), b = *reinterpret_cast<const float4 *>(sb + e);
    *reinterpret_cast<float4 *>(Ss + e) = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
  }
  if (!delta && tid < D) zs[tid] = zf[((int64_t)g * d.H + h) * D + tid] + zb[((int64_t)g * d.H + h) * D + tid];
  __syncthreads();
  const int64_t HD = (int64_t)d.H * D;
  float *qw = qs + warp * D;
  for (int64_t r = r0 + warp; r < r1; r += 8) {
    float ss = 0.f;
    for (int i = lane; i < D; i += 32) {
      float x = to_f(q[r * HD + h * D + i]);
      if (!delta) x = phi_elu1(x);
      ss += x * x;
      qw[i] = x;
    }
    __syncwarp();
    float scale = 1.f;
    if (delta) {
      ss = warp_sum(ss);
      scale = ss > 0.f ? rsqrtf(ss) : 0.f;
    }
    float acc[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[c] = 0.f;
    float den = 0.f;
    for (int i = 0; i < D; ++i) {
      const float x = qw[i];
#pragma unroll
      for (int c = 0; c < NC; ++c) acc[c] = fmaf(x, Ss[i * D + lane + 32 * c], acc[c]);
      if (!delta) den = fmaf(x, zs[i], den);
    }
    float mul = delta ? scale : (den > 0.f ? 1.f / den : 0.f);
#pragma unroll
    for (int c = 0; c < NC; ++c) o[r * HD + h * D + lane + 32 * c] = from_f<T>(acc[c] * mul);
    __syncwarp();
  }
}

template <typename T, int D>
static cudaError_t linear_read_t(const Dims &d, int delta, const void *q, const float *Sf, const float *Sb,
                                 const float *zf, const float *zb, void *o, const int32_t *tiles, int ntiles,
                                 cudaStream_t st) {
  size_t smem = ((size_t)D * D + D + 8 * D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(linear_read_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  linear_read_kernel<T, D><<<dim3(ntiles, d.H), 256, smem, st>>>(d, delta, (const T *)q, Sf, Sb, zf, zb, (T *)o,
                                                                 tiles);
  return cudaGetLastError();
}

cudaError_t launch_linear_read(const Dims &d, vdn_lin_kind kind, vdn_dtype dt, const void *q, const float *Sf,
                               const float *Sb, const float *zf, const float *zb, void *o, char *ws,
                               const WsPlan &p, cudaStream_t st) {
  const int32_t *tiles = (const int32_t *)(ws + p.tiles);
  const int nt = host_tile_count(d);
  const int delta = kind == VDN_LIN_DELTA;
#define VDN_LR(T, DD) return linear_read_t<T, DD>(d, delta, q, Sf, Sb, zf, zb, o, tiles, nt, st)
  if (dt == VDN_F32) {
    if (d.D == 32) VDN_LR(float, 32);
    if (d.D == 64) VDN_LR(float, 64);
    if (d.D == 128) VDN_LR(float, 128);
  } else if (dt == VDN_BF16) {
    if (d.D == 32) VDN_LR(__nv_bfloat16, 32);
    if (d.D == 64) VDN_LR(__nv_bfloat16, 64);
    if (d.D == 128) VDN_LR(__nv_bfloat16, 128);
  }
#undef VDN_LR
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ fuse
// Block per (128 video rows, head); W_l[h] in shared memory; warp per row.
template <typename T, int D>
__global__ void __launch_bounds__(256) fuse_kernel(Dims d, const T *__restrict__ q, const T *__restrict__ os,
                                                   const T *__restrict__ ol, const float *__restrict__ wgs,
                                                   const float *__restrict__ wgl, int G_l,
                                                   const float *__restrict__ gamma, float eps, T *__restrict__ a) {
  extern __shared__ float sm[];
  constexpr int NC = D / 32;
  float *wl = sm, *qs = sm + D * G_l;  // qs [8][D]
  const int h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < D * G_l; e += 256) wl[e] = wgl[(int64_t)h * D * G_l + e];
  __syncthreads();
  const int64_t HD = (int64_t)d.H * D;
  float ws_l[NC], gm[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) { ws_l[c] = wgs[h * D + lane + 32 * c]; gm[c] = gamma[h * D + lane + 32 * c]; }
  float *qw = qs + warp * D;
  const int64_t r0 = (int64_t)blockIdx.x * 128, r1 = min(r0 + 128, d.Nv());
  for (int64_t r = r0 + warp; r < r1; r += 8) {
    float qv[NC], sv[NC], lv[NC];
    float dot_s = 0.f, ss = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int64_t idx = r * HD + h * D + lane + 32 * c;
      qv[c] = to_f(q[idx]); sv[c] = to_f(os[idx]); lv[c] = to_f(ol[idx]);
      qw[lane + 32 * c] = qv[c];
      dot_s = fmaf(qv[c], ws_l[c], dot_s);
      ss = fmaf(lv[c], lv[c], ss);
    }
    __syncwarp();
    dot_s = warp_sum(dot_s);
    ss = warp_sum(ss);
    const float g_s = 1.f / (1.f + expf(-dot_s));
    const float rinv = rsqrtf(ss / (float)D + eps);
    float gl[NC];
    if (G_l == D) {
#pragma unroll
      for (int c = 0; c < NC; ++c) gl[c] = 0.f;
      for (int i = 0; i < D; ++i) {
        const float x = qw[i];
#pragma unroll
        for (int c = 0; c < NC; ++c) gl[c] = fmaf(x, wl[i * D + lane + 32 * c], gl[c]);
      }
#pragma unroll
      for (int c = 0; c < NC; ++c) gl[c] = 1.f / (1.f + expf(-gl[c]));
    } else {
      float t = 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) t = fmaf(qv[c], wl[lane + 32 * c], t);
      t = warp_sum(t);
      const float g = 1.f / (1.f + expf(-t));
#pragma unroll
      for (int c = 0; c < NC; ++c) gl[c] = g;
    }
    T *arow = a + r * 2 * HD;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      arow[h * D + lane + 32 * c] = from_f<T>(g_s * sv[c]);
      arow[HD + h * D + lane + 32 * c] = from_f<T>(gl[c] * gm[c] * lv[c] * rinv);
    }
    __syncwarp();
  }
}

template <typename T, int D>
static cudaError_t fuse_t(const Dims &d, const void *q, const void *os, const void *ol, const float *wgs,
                          const float *wgl, int G_l, const float *gamma, float eps, void *a, cudaStream_t st) {
  size_t smem = ((size_t)D * G_l + 8 * D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(fuse_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((d.Nv() + 127) / 128), d.H);
  fuse_kernel<T, D><<<grid, 256, smem, st>>>(d, (const T *)q, (const T *)os, (const T *)ol, wgs, wgl, G_l, gamma,
                                             eps, (T *)a);
  return cudaGetLastError();
}

cudaError_t launch_fuse(const Dims &d, vdn_dtype dt, const void *q, const void *os, const void *ol,
                        const float *wgs, const float *wgl, int G_l, const float *gamma, float eps, void *a,
                        cudaStream_t st) {
#define VDN_FU(T, DD) return fuse_t<T, DD>(d, q, os, ol, wgs, wgl, G_l, gamma, eps, a, st)
  if (dt == VDN_F32) {
    if (d.D == 32) VDN_FU(float, 32);
    if (d.D == 64) VDN_FU(float, 64);
    if (d.D == 128) VDN_FU(float, 128);
  } else if (dt == VDN_BF16) {
    if (d.D == 32) VDN_FU(__nv_bfloat16, 32);
    if (d.D == 64) VDN_FU(__nv_bfloat16, 64);
    if (d.D == 128) VDN_FU(__nv_bfloat16, 128);
  }
#undef VDN_FU
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ output projection (SIMT)
// y[M][N] = A[M][2N'] Wcat^T with Wcat = [W_os | W_ol] (N' = N = HD).  64 x 64 tiles,
// 16 x 16 threads, 4 x 4 outputs per thread, K staged 16 at a time.
template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(int64_t M, int N, const T *__restrict__ A,
                                                        const T *__restrict__ W1, const T *__restrict__ W2,
                                                        T *__restrict__ Y) {
  __shared__ float As[16][64 + 4], Bs[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = (int64_t)blockIdx.y * 64;
  const int n0 = blockIdx.x * 64;
  const int K = 2 * N;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {
      const int r = e / 16, kk = e % 16;
      const int64_t m = m0 + r;
      const int k = k0 + kk;
      As[kk][r] = (m < M && k < K) ? to_f(A[m * K + k]) : 0.f;
      const int n = n0 + r;
      float b = 0.f;
      if (n < N && k < K) b = k < N ? to_f(W1[(int64_t)n * N + k]) : to_f(W2[(int64_t)n * N + (k - N)]);
      Bs[kk][r] = b;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty + 16 * i]; b[i] = Bs[kk][tx + 16 * i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n < N) Y[m * N + n] = from_f<T>(acc[i][j]);
    }
  }
}

cudaError_t launch_out_proj_simt(const Dims &d, vdn_dtype dt, const void *a, const void *wos, const void *wol,
                                 void *y, cudaStream_t st) {
  const int N = d.H * d.D;
  const int64_t M = d.Nv();
  dim3 grid((N + 63) / 64, (unsigned)((M + 63) / 64));
  if (dt == VDN_F32)
    gemm_simt_kernel<float><<<grid, 256, 0, st>>>(M, N, (const float *)a, (const float *)wos, (const float *)wol,
                                                  (float *)y);
  else
    gemm_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(M, N, (const __nv_bfloat16 *)a,
                                                          (const __nv_bfloat16 *)wos, (const __nv_bfloat16 *)wol,
                                                          (__nv_bfloat16 *)y);
  return cudaGetLastError();
}

}  // namespace vdn
