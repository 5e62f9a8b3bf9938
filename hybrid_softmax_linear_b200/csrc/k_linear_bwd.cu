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
//
// Every product is a matrix product with a D x D memory, so the kernels share one
// register-tiled scheme: 256 threads as 16 x 16, each owning 4 rows x D/16 columns of a
// 64-row tile (or D/16 x D/16 entries of a D x D sum), operands in shared memory with rows
// padded by 4 floats, packed fp32 FMAs.  Every sum runs in a fixed order (no atomics), so a
// call repeats bit for bit.
#include "vdn_internal.cuh"

namespace vdn {
namespace {

constexpr int BT = 256;  // threads per block, 16 x 16
constexpr int BM = 64;   // rows per tile of the row-wise products
constexpr int KC = 32;   // rows per chunk of the per-frame sums

__device__ __forceinline__ float phi1(float x) { return x > 0.f ? x + 1.f : expf(x); }
// phi'(x) is 1 for x > 0 and e^x otherwise, which is min(phi(x), 1): phi(x) >= 1 exactly when
// x >= 0, and phi(0) = 1.
__device__ __forceinline__ float dphi_of_phi(float p) { return fminf(p, 1.f); }

template <int D>
struct Lay {
  static constexpr int LD = D + 4;               // shared-memory row stride in floats (16-byte rows)
  static constexpr int CPT = D / 16;             // columns (rows of a D x D sum) per thread
  static constexpr int VW = CPT >= 4 ? 4 : CPT;  // vector width of a thread's column run
  static constexpr int NV = CPT / VW;            // runs per thread
  static constexpr int NP = CPT / 2;             // packed pairs per row
  __device__ static __forceinline__ int col(int x, int v) { return v * 16 * VW + x * VW; }
};

template <int VW>
__device__ __forceinline__ void ld_vec(const float *p, float *o) {
  if constexpr (VW == 4) {
    const float4 x = *reinterpret_cast<const float4 *>(p);
    o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
  } else {
    const float2 x = *reinterpret_cast<const float2 *>(p);
    o[0] = x.x; o[1] = x.y;
  }
}

template <int VW>
__device__ __forceinline__ void st_vec(float *p, const float *o) {
  if constexpr (VW == 4) {
    *reinterpret_cast<float4 *>(p) = make_float4(o[0], o[1], o[2], o[3]);
  } else {
    *reinterpret_cast<float2 *>(p) = make_float2(o[0], o[1]);
  }
}

__device__ __forceinline__ float pick(const float2 &p, int c) { return (c & 1) ? p.y : p.x; }

// acc[r] += A[ty*4 + r][:] B over k < D: A a [64][LD] tile, B a [D][LD] matrix, both in
// shared memory; thread columns Lay::col(tx, v) + 0..VW-1, held as packed pairs.
template <int D>
__device__ __forceinline__ void tile_mma(const float *A, const float *B, int ty, int tx,
                                         float2 (&acc)[4][Lay<D>::NP]) {
  using L = Lay<D>;
#pragma unroll 2
  for (int k0 = 0; k0 < D; k0 += 4) {
    float a[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r) ld_vec<4>(A + (ty * 4 + r) * L::LD + k0, a[r]);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      float b[L::CPT];
#pragma unroll
      for (int v = 0; v < L::NV; ++v) ld_vec<L::VW>(B + (k0 + kk) * L::LD + L::col(tx, v), b + v * L::VW);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float2 ar = make_float2(a[r][kk], a[r][kk]);
#pragma unroll
        for (int p = 0; p < L::NP; ++p) acc[r][p] = __ffma2_rn(ar, make_float2(b[2 * p], b[2 * p + 1]), acc[r][p]);
      }
    }
  }
}

// Two independent products over the same k: acc1 += A1 B1, acc2 += A2 B2.
template <int D>
__device__ __forceinline__ void tile_mma2(const float *A1, const float *B1, const float *A2, const float *B2, int ty,
                                          int tx, float2 (&acc1)[4][Lay<D>::NP], float2 (&acc2)[4][Lay<D>::NP]) {
  using L = Lay<D>;
#pragma unroll 2
  for (int k0 = 0; k0 < D; k0 += 4) {
    float a1[4][4], a2[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      ld_vec<4>(A1 + (ty * 4 + r) * L::LD + k0, a1[r]);
      ld_vec<4>(A2 + (ty * 4 + r) * L::LD + k0, a2[r]);
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      float b1[L::CPT], b2[L::CPT];
#pragma unroll
      for (int v = 0; v < L::NV; ++v) {
        ld_vec<L::VW>(B1 + (k0 + kk) * L::LD + L::col(tx, v), b1 + v * L::VW);
        ld_vec<L::VW>(B2 + (k0 + kk) * L::LD + L::col(tx, v), b2 + v * L::VW);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float2 x1 = make_float2(a1[r][kk], a1[r][kk]), x2 = make_float2(a2[r][kk], a2[r][kk]);
#pragma unroll
        for (int p = 0; p < L::NP; ++p) {
          acc1[r][p] = __ffma2_rn(x1, make_float2(b1[2 * p], b1[2 * p + 1]), acc1[r][p]);
          acc2[r][p] = __ffma2_rn(x2, make_float2(b2[2 * p], b2[2 * p + 1]), acc2[r][p]);
        }
      }
    }
  }
}

// A 64-row tile of bf16 rows of D features moves in two steps, so that its global loads can
// be in flight while the previous tile is being multiplied: fetch_tile reads n (<= 64) rows
// (row stride `stride` elements) into registers, 16 bytes per piece; put_tile converts them
// to float (phi applied when PHI) into a [64][LD] tile in shared memory, rows n..63 zero.
template <int D>
struct TileRegs {
  static constexpr int PER_ROW = D / 8;               // 16-byte pieces per row
  static constexpr int N = BM * PER_ROW / BT;         // pieces per thread (exact for D >= 32)
  uint4 r[N];
};

template <int D>
__device__ __forceinline__ void fetch_tile(const __nv_bfloat16 *__restrict__ src, int64_t stride, int n,
                                           TileRegs<D> &x, int t) {
  constexpr int PR = TileRegs<D>::PER_ROW;
#pragma unroll
  for (int u = 0; u < TileRegs<D>::N; ++u) {
    const int e = t + u * BT, row = e / PR;
    x.r[u] = row < n ? *reinterpret_cast<const uint4 *>(src + row * stride + (e % PR) * 8) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <int D, bool PHI>
__device__ __forceinline__ void put_tile(const TileRegs<D> &x, int n, float *dst, int t) {
  using L = Lay<D>;
  constexpr int PR = TileRegs<D>::PER_ROW;
#pragma unroll
  for (int u = 0; u < TileRegs<D>::N; ++u) {
    const int e = t + u * BT, row = e / PR, c8 = (e % PR) * 8;
    float y[8];
    const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&x.r[u]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p2[i]);
      y[2 * i] = PHI && row < n ? phi1(f.x) : f.x;  // a dead row was fetched as zeros and stays zero
      y[2 * i + 1] = PHI && row < n ? phi1(f.y) : f.y;
    }
    st_vec<4>(dst + row * L::LD + c8, y);
    st_vec<4>(dst + row * L::LD + c8 + 4, y + 4);
  }
}

// ---------------------------------------------------------------- per-frame sums
// C[i][j] = sum over the rows r of one frame (or of the text) of phi(a_r)[i] b_r[j] and
// c[i] = sum_r w_r phi(a_r)[i], the rows in ascending order.  States (GRAD false): a = k,
// b = v (bf16), w = 1, the text block (blockIdx.x == nframes) writing Ct, ct.  Gradient sums
// (GRAD true): a = q, b = dnum (f32), w = dden.  Chunks of 32 rows are double-buffered in
// shared memory, the next chunk's global loads in flight while the current one is summed;
// thread (ty, tx) owns rows Lay::col(ty, .) and columns Lay::col(tx, .) of C.
template <int D, bool GRAD>
__global__ void __launch_bounds__(BT, 2) lin_outer_kernel(Dims d, const __nv_bfloat16 *__restrict__ a,
                                                          const void *__restrict__ b, const __nv_bfloat16 *__restrict__ at,
                                                          const __nv_bfloat16 *__restrict__ bt,
                                                          const float *__restrict__ w, float *__restrict__ C,
                                                          float *__restrict__ c, float *__restrict__ Ct,
                                                          float *__restrict__ ct, int nframes) {
  using L = Lay<D>;
  constexpr int AP = KC * D / 8;                  // 16-byte pieces of a chunk of a (bf16)
  constexpr int BP = GRAD ? KC * D / 4 : AP;      // of b (f32 or bf16)
  constexpr int NA = (AP + BT - 1) / BT, NB = (BP + BT - 1) / BT;
  constexpr int A_ROW = D / 8, B_ROW = GRAD ? D / 4 : D / 8;
  extern __shared__ __align__(16) float sm[];
  float *As = sm, *Bs = As + 2 * KC * L::LD, *Ws = Bs + 2 * KC * L::LD;  // [2][KC][LD], [2][KC][LD], [2][KC]
  const int h = blockIdx.y, t = threadIdx.x, ty = t >> 4, tx = t & 15;
  const bool text = !GRAD && (int)blockIdx.x == nframes;
  const int ntok = text ? d.L : d.T;
  const int64_t HD = (int64_t)d.H * D;
  const int64_t r0 = text ? 0 : (int64_t)blockIdx.x * d.T;  // first row
  const __nv_bfloat16 *ab = (text ? at : a) + r0 * HD + (int64_t)h * D;
  const char *bb = text ? (const char *)bt : (const char *)b;
  const int64_t belem = r0 * HD + (int64_t)h * D;  // element offset of b's first row
  const int nch = (ntok + KC - 1) / KC;

  uint4 ra[NA], rb[NB];
  float rw = 0.f;
  auto fetch = [&](int ch) {
    const int m0 = ch * KC, n = min(KC, ntok - m0);
#pragma unroll
    for (int u = 0; u < NA; ++u) {
      const int e = t + u * BT, row = e / A_ROW;
      ra[u] = make_uint4(0u, 0u, 0u, 0u);
      if (e < AP && row < n) ra[u] = *reinterpret_cast<const uint4 *>(ab + (int64_t)(m0 + row) * HD + (e % A_ROW) * 8);
    }
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const int e = t + u * BT, row = e / B_ROW;
      rb[u] = make_uint4(0u, 0u, 0u, 0u);
      if (e < BP && row < n) {
        if (GRAD) {
          rb[u] = *reinterpret_cast<const uint4 *>((const float *)bb + belem + (int64_t)(m0 + row) * HD + (e % B_ROW) * 4);
        } else {
          rb[u] = *reinterpret_cast<const uint4 *>((const __nv_bfloat16 *)bb + belem + (int64_t)(m0 + row) * HD +
                                                   (e % B_ROW) * 8);
        }
      }
    }
    if (t < KC) rw = (t < n) ? (GRAD ? w[(r0 + m0 + t) * d.H + h] : 1.f) : 0.f;
  };
  auto stash = [&](int buf) {
    float *as = As + buf * KC * L::LD, *bs = Bs + buf * KC * L::LD;
#pragma unroll
    for (int u = 0; u < NA; ++u) {
      const int e = t + u * BT;
      if (e < AP) {
        const int row = e / A_ROW;  // a dead row becomes phi(0) = 1 here; the sums stop before it
        const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&ra[u]);
        float x[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(p2[i]);
          x[2 * i] = phi1(f.x);
          x[2 * i + 1] = phi1(f.y);
        }
        st_vec<4>(as + row * L::LD + (e % A_ROW) * 8, x);
        st_vec<4>(as + row * L::LD + (e % A_ROW) * 8 + 4, x + 4);
      }
    }
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const int e = t + u * BT;
      if (e < BP) {
        const int row = e / B_ROW;
        if (GRAD) {
          const float4 x = *reinterpret_cast<const float4 *>(&rb[u]);
          *reinterpret_cast<float4 *>(bs + row * L::LD + (e % B_ROW) * 4) = x;
        } else {
          const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&rb[u]);
          float x[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(p2[i]);
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
          }
          st_vec<4>(bs + row * L::LD + (e % B_ROW) * 8, x);
          st_vec<4>(bs + row * L::LD + (e % B_ROW) * 8 + 4, x + 4);
        }
      }
    }
    if (t < KC) Ws[buf * KC + t] = rw;
  };

  float2 acc[L::CPT][L::NP];
#pragma unroll
  for (int i = 0; i < L::CPT; ++i)
#pragma unroll
    for (int p = 0; p < L::NP; ++p) acc[i][p] = make_float2(0.f, 0.f);
  float zacc = 0.f;  // threads t < D: c[t]
  if (nch > 0) {
    fetch(0);
    stash(0);
  }
  __syncthreads();
  for (int ch = 0; ch < nch; ++ch) {
    const int buf = ch & 1, n = min(KC, ntok - ch * KC);
    if (ch + 1 < nch) fetch(ch + 1);
    const float *as = As + buf * KC * L::LD, *bs = Bs + buf * KC * L::LD, *ws = Ws + buf * KC;
    for (int kr = 0; kr < n; ++kr) {
      float av[L::CPT], bv[L::CPT];
#pragma unroll
      for (int v = 0; v < L::NV; ++v) {
        ld_vec<L::VW>(as + kr * L::LD + L::col(ty, v), av + v * L::VW);
        ld_vec<L::VW>(bs + kr * L::LD + L::col(tx, v), bv + v * L::VW);
      }
#pragma unroll
      for (int i = 0; i < L::CPT; ++i) {
        const float2 x = make_float2(av[i], av[i]);
#pragma unroll
        for (int p = 0; p < L::NP; ++p) acc[i][p] = __ffma2_rn(x, make_float2(bv[2 * p], bv[2 * p + 1]), acc[i][p]);
      }
      if (t < D) zacc = GRAD ? fmaf(as[kr * L::LD + t], ws[kr], zacc) : zacc + as[kr * L::LD + t];
    }
    if (ch + 1 < nch) stash(buf ^ 1);
    __syncthreads();
  }
  float *Co = text ? Ct + (int64_t)h * D * D : C + ((int64_t)blockIdx.x * d.H + h) * D * D;
#pragma unroll
  for (int v = 0; v < L::NV; ++v)
#pragma unroll
    for (int i = 0; i < L::VW; ++i) {
      const int row = L::col(ty, v) + i, ci = v * L::VW + i;
#pragma unroll
      for (int u = 0; u < L::NV; ++u) {
        float o[L::VW];
#pragma unroll
        for (int q2 = 0; q2 < L::VW; ++q2) o[q2] = pick(acc[ci][(u * L::VW + q2) >> 1], u * L::VW + q2);
        st_vec<L::VW>(Co + (int64_t)row * D + L::col(tx, u), o);
      }
    }
  float *co = text ? ct + (int64_t)h * D : c + ((int64_t)blockIdx.x * d.H + h) * D;
  if (t < D) co[t] = zacc;
}

// ---------------------------------------------------------------- per query row
// Block per (query frame f, head): the frame's group memory Num_g (and its transpose) and
// Den_g in shared memory; per 64-row tile: phi(q), den, num = phi(q) Num_g, the per-row
// dnum and dden, then dphi(q) = dnum Num_g^T + Den_g dden and dq.
template <int D>
__global__ void __launch_bounds__(BT, 1) lin_bwd_rows_kernel(Dims d, const __nv_bfloat16 *__restrict__ q,
                                                             const float *__restrict__ dO, const float *__restrict__ Sf,
                                                             const float *__restrict__ Sb, const float *__restrict__ zf,
                                                             const float *__restrict__ zb, const int32_t *__restrict__ ftab,
                                                             float *__restrict__ dq, float *__restrict__ dnum_out,
                                                             float *__restrict__ dden_out) {
  using L = Lay<D>;
  extern __shared__ __align__(16) float sm[];
  float *Num = sm, *NumT = Num + D * L::LD, *P = NumT + D * L::LD, *DN = P + BM * L::LD;
  float *Den = DN + BM * L::LD, *dpart = Den + D, *rinv = dpart + 4 * BM, *rdd = rinv + BM;
  const int f = blockIdx.x, h = blockIdx.y, t = threadIdx.x, ty = t >> 4, tx = t & 15;
  const int g = ftab[f * 8];
  const int64_t HD = (int64_t)d.H * D, mo = ((int64_t)g * d.H + h) * D * D;
  // Num = Sf + Sb row-major and transposed: thread e takes row i = e % D, columns j0..j0+3,
  // so both shared-memory stores are conflict-free
  for (int e = t; e < D * D / 4; e += BT) {
    const int i = e % D, j0 = 4 * (e / D);
    const float4 x = *reinterpret_cast<const float4 *>(Sf + mo + i * D + j0);
    const float4 y = *reinterpret_cast<const float4 *>(Sb + mo + i * D + j0);
    const float s[4] = {x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w};
    st_vec<4>(Num + i * L::LD + j0, s);
#pragma unroll
    for (int u = 0; u < 4; ++u) NumT[(j0 + u) * L::LD + i] = s[u];
  }
  for (int e = t; e < D; e += BT) Den[e] = zf[((int64_t)g * d.H + h) * D + e] + zb[((int64_t)g * d.H + h) * D + e];
  __syncthreads();
  const int64_t fr0 = (int64_t)f * d.T;
  const __nv_bfloat16 *qb = q + fr0 * HD + (int64_t)h * D;
  TileRegs<D> rq;
  fetch_tile<D>(qb, HD, min(BM, d.T), rq, t);
  for (int m0 = 0; m0 < d.T; m0 += BM) {
    const int n = min(BM, d.T - m0);
    put_tile<D, true>(rq, n, P, t);
    __syncthreads();
    // this tile's dO and the next tile's q are in flight while den and num are computed
    float go[4][L::CPT];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = ty * 4 + r;
#pragma unroll
      for (int c = 0; c < L::CPT; ++c) go[r][c] = 0.f;
      if (row < n) {
#pragma unroll
        for (int v = 0; v < L::NV; ++v)
          ld_vec<L::VW>(dO + (fr0 + m0 + row) * HD + (int64_t)h * D + L::col(tx, v), go[r] + v * L::VW);
      }
    }
    if (m0 + BM < d.T) fetch_tile<D>(qb + (int64_t)(m0 + BM) * HD, HD, min(BM, d.T - m0 - BM), rq, t);
    {  // den partials over quarters of the features: row t / 4, quarter t % 4
      const int row = t >> 2, qq = t & 3;
      const float *pr = P + row * L::LD + qq * (D / 4), *dr = Den + qq * (D / 4);
      float s = 0.f;
#pragma unroll 8
      for (int i = 0; i < D / 4; ++i) s = fmaf(pr[i], dr[i], s);
      dpart[qq * BM + row] = s;
    }
    __syncthreads();
    if (t < BM) {
      const float den = ((dpart[t] + dpart[BM + t]) + dpart[2 * BM + t]) + dpart[3 * BM + t];
      rinv[t] = den > 0.f ? 1.f / den : 0.f;
    }
    float2 acc[4][L::NP];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int p = 0; p < L::NP; ++p) acc[r][p] = make_float2(0.f, 0.f);
    tile_mma<D>(P, Num, ty, tx, acc);
    __syncthreads();  // rinv
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = ty * 4 + r;
      const bool live = row < n;
      const float inv = rinv[row];
      const int64_t gb = (fr0 + m0 + row) * HD + (int64_t)h * D;
      float dot = 0.f;
#pragma unroll
      for (int v = 0; v < L::NV; ++v) {
        float dn[L::VW];
#pragma unroll
        for (int c = 0; c < L::VW; ++c) {
          const int ci = v * L::VW + c;
          const float o = pick(acc[r][ci >> 1], ci) * inv;
          dot = fmaf(go[r][ci], o, dot);
          dn[c] = go[r][ci] * inv;
        }
        st_vec<L::VW>(DN + row * L::LD + L::col(tx, v), dn);
        if (live) st_vec<L::VW>(dnum_out + gb + L::col(tx, v), dn);
      }
      // dO . o over the row's 16 threads (lanes tx = 0..15 of a half warp), a fixed tree
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const float dden = inv > 0.f ? -dot * inv : 0.f;
      if (tx == 0) {
        rdd[row] = dden;
        if (live) dden_out[(fr0 + m0 + row) * d.H + h] = dden;
      }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int p = 0; p < L::NP; ++p) acc[r][p] = make_float2(0.f, 0.f);
    tile_mma<D>(DN, NumT, ty, tx, acc);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = ty * 4 + r;
      if (row >= n) continue;
      const float dd = rdd[row];
      const int64_t gb = (fr0 + m0 + row) * HD + (int64_t)h * D;
#pragma unroll
      for (int v = 0; v < L::NV; ++v) {
        float pv[L::VW], out[L::VW];
        ld_vec<L::VW>(P + row * L::LD + L::col(tx, v), pv);
#pragma unroll
        for (int c = 0; c < L::VW; ++c) {
          const int ci = v * L::VW + c;
          out[c] = fmaf(Den[L::col(tx, v) + c], dd, pick(acc[r][ci >> 1], ci)) * dphi_of_phi(pv[c]);
        }
        st_vec<L::VW>(dq + gb + L::col(tx, v), out);
      }
    }
    __syncthreads();  // P, DN, rinv and rdd are rewritten by the next tile
  }
}

// dNum_g = sum over the group's frames (ascending) of the per-frame gradient sums; likewise dDen_g.
template <int D>
__global__ void __launch_bounds__(BT) lin_bwd_group_sum_kernel(Dims d, const float *__restrict__ part,
                                                               const float *__restrict__ zpart,
                                                               const int32_t *__restrict__ gtab, float *__restrict__ dN,
                                                               float *__restrict__ dZ) {
  const int g = blockIdx.x, h = blockIdx.y, t = threadIdx.x;
  const int f0 = gtab[g * 16], f1 = gtab[g * 16 + 1];
  const int64_t DD = (int64_t)D * D;
  for (int e = t; e < D * D / 4; e += BT) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int f = f0; f < f1; ++f) {
      const float4 x = *reinterpret_cast<const float4 *>(part + ((int64_t)f * d.H + h) * DD + 4 * e);
      s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
    }
    *reinterpret_cast<float4 *>(dN + ((int64_t)g * d.H + h) * DD + 4 * e) = s;
  }
  for (int e = t; e < D; e += BT) {
    float s = 0.f;
    for (int f = f0; f < f1; ++f) s += zpart[((int64_t)f * d.H + h) * D + e];
    dZ[((int64_t)g * d.H + h) * D + e] = s;
  }
}

// ---------------------------------------------------------------- per key row
// Block per (key frame fk, head), fk == F for the text: dS = sum of dNum_g over the groups
// whose memory holds fk (every group for the text), in group order, and its transpose; then
// per 64-row tile of the frame's keys: dphi(k) = v dS^T + dz and dv = phi(k) dS.
template <int D>
__global__ void __launch_bounds__(BT, 1) lin_bwd_keys_kernel(Dims d, const __nv_bfloat16 *__restrict__ k,
                                                             const __nv_bfloat16 *__restrict__ v,
                                                             const __nv_bfloat16 *__restrict__ kt,
                                                             const __nv_bfloat16 *__restrict__ vt,
                                                             const float *__restrict__ dN, const float *__restrict__ dZ,
                                                             const int32_t *__restrict__ gtab, int G,
                                                             float *__restrict__ dk, float *__restrict__ dv,
                                                             float *__restrict__ dkt, float *__restrict__ dvt) {
  using L = Lay<D>;
  extern __shared__ __align__(16) float sm[];
  float *dS = sm, *dST = dS + D * L::LD, *Vs = dST + D * L::LD, *PK = Vs + BM * L::LD, *dz = PK + BM * L::LD;
  unsigned char *held = reinterpret_cast<unsigned char *>(dz + D);  // [G]: group g's memory holds fk
  const int fk = blockIdx.x, h = blockIdx.y, t = threadIdx.x, ty = t >> 4, tx = t & 15;
  const bool text = fk == d.F;
  const int64_t DD = (int64_t)D * D, HD = (int64_t)d.H * D;
  const int ntok = text ? d.L : d.T;
  const __nv_bfloat16 *kb = (text ? kt : k + (int64_t)fk * d.T * HD) + (int64_t)h * D;
  const __nv_bfloat16 *vb = (text ? vt : v + (int64_t)fk * d.T * HD) + (int64_t)h * D;
  float *dkb = (text ? dkt : dk + (int64_t)fk * d.T * HD) + (int64_t)h * D;
  float *dvb = (text ? dvt : dv + (int64_t)fk * d.T * HD) + (int64_t)h * D;
  TileRegs<D> rk, rv;  // the first tile's loads are in flight during the gather
  fetch_tile<D>(kb, HD, min(BM, ntok), rk, t);
  fetch_tile<D>(vb, HD, min(BM, ntok), rv, t);
  for (int g = t; g < G; g += BT) {
    const int32_t *r = gtab + g * 16;
    held[g] = (text || (fk >= r[12] && fk < r[13]) || (fk >= r[14] && fk < r[15])) ? 1 : 0;
  }
  __syncthreads();
  // loads of 8 groups at a time, added in group order
  constexpr int GB = 8;
  for (int e = t; e < D * D / 4; e += BT) {
    const int i = e % D, j0 = 4 * (e / D);
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    for (int g0 = 0; g0 < G; g0 += GB) {
      float4 x[GB];
#pragma unroll
      for (int u = 0; u < GB; ++u) {
        const int g = g0 + u;
        x[u] = (g < G && held[g]) ? *reinterpret_cast<const float4 *>(dN + ((int64_t)g * d.H + h) * DD + i * D + j0)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < GB; ++u) {
        if (g0 + u < G && held[g0 + u]) {
          s[0] += x[u].x; s[1] += x[u].y; s[2] += x[u].z; s[3] += x[u].w;
        }
      }
    }
    st_vec<4>(dS + i * L::LD + j0, s);
#pragma unroll
    for (int u = 0; u < 4; ++u) dST[(j0 + u) * L::LD + i] = s[u];
  }
  for (int e = t; e < D; e += BT) {
    float s = 0.f;
    for (int g = 0; g < G; ++g)
      if (held[g]) s += dZ[((int64_t)g * d.H + h) * D + e];
    dz[e] = s;
  }
  for (int m0 = 0; m0 < ntok; m0 += BM) {
    const int n = min(BM, ntok - m0);
    put_tile<D, true>(rk, n, PK, t);
    put_tile<D, false>(rv, n, Vs, t);
    __syncthreads();
    if (m0 + BM < ntok) {
      fetch_tile<D>(kb + (int64_t)(m0 + BM) * HD, HD, min(BM, ntok - m0 - BM), rk, t);
      fetch_tile<D>(vb + (int64_t)(m0 + BM) * HD, HD, min(BM, ntok - m0 - BM), rv, t);
    }
    float2 a1[4][L::NP], a2[4][L::NP];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int p = 0; p < L::NP; ++p) a1[r][p] = a2[r][p] = make_float2(0.f, 0.f);
    tile_mma2<D>(Vs, dST, PK, dS, ty, tx, a1, a2);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = ty * 4 + r;
      if (row >= n) continue;
      const int64_t gb = (int64_t)(m0 + row) * HD;
#pragma unroll
      for (int u = 0; u < L::NV; ++u) {
        float pv[L::VW], ok[L::VW], ov[L::VW];
        ld_vec<L::VW>(PK + row * L::LD + L::col(tx, u), pv);
#pragma unroll
        for (int c = 0; c < L::VW; ++c) {
          const int ci = u * L::VW + c;
          ok[c] = (pick(a1[r][ci >> 1], ci) + dz[L::col(tx, u) + c]) * dphi_of_phi(pv[c]);
          ov[c] = pick(a2[r][ci >> 1], ci);
        }
        st_vec<L::VW>(dkb + gb + L::col(tx, u), ok);
        st_vec<L::VW>(dvb + gb + L::col(tx, u), ov);
      }
    }
    __syncthreads();  // PK and Vs are rewritten by the next tile
  }
}

template <int D>
cudaError_t lin_bwd_t(const LinBwdArgs &a, int stage, cudaStream_t st) {
  using L = Lay<D>;
  const Dims &d = a.d;
  cudaError_t e = cudaSuccess;
  const size_t smem_outer = (size_t)(4 * KC * L::LD + 2 * KC) * sizeof(float);
  switch (stage) {
    case LIN_BWD_STATE:
      e = cudaFuncSetAttribute(lin_outer_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem_outer);
      if (e != cudaSuccess) return e;
      lin_outer_kernel<D, false><<<dim3(d.F + 1, d.H), BT, smem_outer, st>>>(
          d, (const __nv_bfloat16 *)a.k, a.v, (const __nv_bfloat16 *)a.kt, (const __nv_bfloat16 *)a.vt, nullptr, a.S,
          a.z, a.St, a.zt, d.F);
      break;
    case LIN_BWD_ROWS: {
      const size_t smem = (size_t)(2 * D * L::LD + 2 * BM * L::LD + D + 6 * BM) * sizeof(float);
      e = cudaFuncSetAttribute(lin_bwd_rows_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      lin_bwd_rows_kernel<D><<<dim3(d.F, d.H), BT, smem, st>>>(d, (const __nv_bfloat16 *)a.q, a.dO, a.Sf, a.Sb, a.zf,
                                                                a.zb, a.ftab, a.dq, a.dnum, a.dden);
      break;
    }
    case LIN_BWD_FRAMES:
      e = cudaFuncSetAttribute(lin_outer_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem_outer);
      if (e != cudaSuccess) return e;
      lin_outer_kernel<D, true><<<dim3(d.F, d.H), BT, smem_outer, st>>>(
          d, (const __nv_bfloat16 *)a.q, a.dnum, nullptr, nullptr, a.dden, a.part, a.zpart, nullptr, nullptr, d.F);
      break;
    case LIN_BWD_GROUPS:
      lin_bwd_group_sum_kernel<D><<<dim3(a.G, d.H), BT, 0, st>>>(d, a.part, a.zpart, a.gtab, a.dN, a.dZ);
      break;
    case LIN_BWD_KEYS: {
      const size_t smem = linear_bwd_keys_smem(D, a.G);
      e = cudaFuncSetAttribute(lin_bwd_keys_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      lin_bwd_keys_kernel<D><<<dim3(d.F + 1, d.H), BT, smem, st>>>(
          d, (const __nv_bfloat16 *)a.k, (const __nv_bfloat16 *)a.v, (const __nv_bfloat16 *)a.kt,
          (const __nv_bfloat16 *)a.vt, a.dN, a.dZ, a.gtab, a.G, a.dk, a.dv, a.dkt, a.dvt);
      break;
    }
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

size_t linear_bwd_keys_smem(int D, int G) {
  const size_t g = (size_t)((G + 15) & ~15);
  if (D == 32) return (size_t)(2 * D * Lay<32>::LD + 2 * BM * Lay<32>::LD + D) * sizeof(float) + g;
  if (D == 64) return (size_t)(2 * D * Lay<64>::LD + 2 * BM * Lay<64>::LD + D) * sizeof(float) + g;
  return (size_t)(2 * D * Lay<128>::LD + 2 * BM * Lay<128>::LD + D) * sizeof(float) + g;
}

cudaError_t launch_linear_bwd(const LinBwdArgs &a, int stage, cudaStream_t st) {
  if (a.d.D == 32) return lin_bwd_t<32>(a, stage, st);
  if (a.d.D == 64) return lin_bwd_t<64>(a, stage, st);
  if (a.d.D == 128) return lin_bwd_t<128>(a, stage, st);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
