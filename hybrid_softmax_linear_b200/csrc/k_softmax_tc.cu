// Softmax branch on the 5th-generation tensor cores: block-sparse flash attention over
// the key set of each query group ("VDN-MiniMax-H3 开源" article, 技术解读 /
// 局部精确计算: the chunk window, both anchor frames and every text token; the model
// card calls it the window softmax).
//
// One CTA owns 256 query rows of one group and one head, as two 128-row tiles Q0, Q1
// that share every K/V tile.  Warp 0 streams Q once and the group's K/V tiles (128 keys,
// text first, then the merged video segments) with TMA into 2-stage rings.  One thread
// of warp 1 issues tcgen05.mma: S_w = Q_w K_j^T (M=128, N=128) into tensor memory, then,
// once softmax warpgroup w has rescaled its output and written P_w (bf16 or e4m3, over
// S_w's columns; e4m3 in two pieces of 64 keys, each handed over as soon as it is
// written), O_w += P_w V_j (A operand from tensor memory, V as an MN-major operand).
// Warpgroups 1 and 2 (warps 4-7 and 8-11) run the online softmax of Q0 and Q1, one row
// per thread, so while one warpgroup exponentiates, the tensor cores work for the
// other.  Warpgroup 0 (the TMA and MMA warps and two idle ones) hands most of its
// registers to the softmax warpgroups (setmaxnreg), which keep a whole row of S in
// registers and work on pairs of values with the packed fp32 instructions of sm_100.
// (A share of the exponentials can run as a polynomial on the FMA pipe instead of the
// exponential unit, VDN_SOFTMAX_POLY_PAIRS; measured slower at every share, so off.)
// The running maximum is only moved (and O rescaled) when it grows by more than
// 2^8; the final normalisation uses the same stale maximum, so the result is exact.
// Keys past the end of a segment are masked in the last tile of that segment.
#include "tc_common.cuh"

#ifndef VDN_SOFTMAX_POLY_PAIRS
#define VDN_SOFTMAX_POLY_PAIRS 0
#endif

namespace vdn {
namespace {

using namespace tc;

constexpr int BM = 128;     // rows per Q tile
constexpr int BN = 128;     // keys per K/V tile
constexpr int NQ = 2;       // Q tiles per CTA
constexpr int KST = 2, VST = 2;
constexpr int THREADS = 384;      // 12 warps: warpgroup 0 = TMA, MMA, 2 idle; warpgroups 1, 2 = softmax
// registers per thread after the split: 128 x 64 + 256 x 216 = 63488, within the launch's 384 x 168
constexpr uint32_t REGS_CTRL = 64, REGS_SOFTMAX = 216;
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
// P of a tile is handed to the tensor cores in up to MAX_P_PARTS pieces (Cfg::P_PARTS)
constexpr int MAX_P_PARTS = 2;

// FP8 = false: bf16 Q/K/V and P (kind::f16, K = 16 per MMA).  FP8 = true: e4m3 Q/K/V
// with per-head scales and e4m3 P at unit scale (kind::f8f6f4, K = 32 per MMA).  A
// 128-byte swizzle row holds 64 bf16 or 128 e4m3 values; one MMA K-step is 32 bytes of a
// row either way, and one P column of tensor memory packs 2 bf16 or 4 e4m3 values.
template <int D, bool FP8>
struct Cfg {
  static constexpr int EB = FP8 ? 1 : 2;               // bytes per element
  static constexpr int BOX_ELEMS = 128 / EB;           // elements in a 128-byte box row
  static constexpr int BOXES = D * EB / 128;           // 128-byte boxes per row
  static constexpr int TILE_BYTES = BM * D * EB;       // one 128 x D tile
  static constexpr int KSTEP = 32 / EB;                // elements per MMA K-step
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + NQ * TILE_BYTES;
  static constexpr int V_OFF = K_OFF + KST * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + VST * TILE_BYTES;
  static constexpr uint32_t IDESC_S = FP8 ? idesc_e4m3(BM, BN, false, false) : idesc_bf16(BM, BN, false, false);
  static constexpr uint32_t IDESC_O = FP8 ? idesc_e4m3(BM, D, false, true) : idesc_bf16(BM, D, false, true);
  // e4m3: P goes to the tensor cores in two pieces of 64 keys, so the P.V MMA of the first
  // overlaps the exponentials of the second (5% faster, measured).  bf16: in one piece; its
  // P.V takes twice as long and a wait in its middle holds up the single MMA issuer (2%
  // slower in two pieces, 8% in four).
  static constexpr int P_PARTS = FP8 ? 2 : 1;
  static_assert(P_PARTS <= MAX_P_PARTS && (P_PARTS == 1 || P_PARTS == 2 || P_PARTS == 4), "P is written in 32-key chunks");
  // tensor memory columns: S_0, S_1, O_0, O_1
  __device__ static constexpr uint32_t s_col(int w) { return (uint32_t)w * 128u; }
  __device__ static constexpr uint32_t o_col(int w) { return 256u + (uint32_t)w * 128u; }
};

// The key tiles of a group: text rows first, then video rows, each merged segment of the
// group cut into 128-key tiles.
struct KvParts {
  int n;
  int text[5], lo[5], hi[5];
};

struct alignas(8) Bars {
  uint64_t q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[NQ], p_ready[NQ][MAX_P_PARTS], o_done,
      drain;
  uint32_t tmem_base;
  int abort;
  // this block's work, decoded once by thread 0; each role reads it after the register
  // split, so that nothing computed before the split stays live across it
  int h, row0, row_end, nkv;
  KvParts parts;
};

// dynamic shared memory of a block: the 1024-byte alignment pad, the Q, K and V tiles, and
// the barriers
template <int D, bool FP8>
constexpr size_t smem_bytes() { return 1024 + Cfg<D, FP8>::BAR_OFF + sizeof(Bars); }
static_assert(smem_bytes<128, false>() <= 227 * 1024 && smem_bytes<128, true>() <= 227 * 1024,
              "shared memory of a block");

__device__ __forceinline__ void kv_parts(const int32_t *g, int L, KvParts &p) {
  p.n = 0;
  for (int s = 0; s < g[2]; ++s) {
    const int lo = g[4 + 2 * s], hi = g[5 + 2 * s];
    if (lo < L) { p.text[p.n] = 1; p.lo[p.n] = lo; p.hi[p.n] = hi < L ? hi : L; ++p.n; }
    if (hi > L) { p.text[p.n] = 0; p.lo[p.n] = (lo > L ? lo : L) - L; p.hi[p.n] = hi - L; ++p.n; }
  }
}

__device__ __forceinline__ int kv_tiles(const KvParts &p) {
  int n = 0;
  for (int i = 0; i < p.n; ++i) n += (p.hi[i] - p.lo[i] + BN - 1) / BN;
  return n;
}

// cursor over the tiles: part index and row of the current tile
struct KvCursor {
  int part, row;
  __device__ void init(const KvParts &p) { part = 0; row = p.lo[0]; }
  __device__ void next(const KvParts &p) {
    row += BN;
    if (row >= p.hi[part]) { ++part; if (part < p.n) row = p.lo[part]; }
  }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA and integer pipes for a share of the exponentials (pairs of values,
// packed fp32 instructions), so that the hardware exponential unit is not the only path.
// Range reduction: x = n + f with n = round(x) (read from the low mantissa bits after
// adding 1.5 * 2^23) and f in [-1/2, 1/2]; 2^f is a degree-3 polynomial, fitted here for
// minimal relative error on [-1/2, 1/2] (iteratively reweighted least squares, Lawson's
// method; max relative error 7.5e-5, below bf16's 2^-9); 2^n is added to the exponent
// field.  x is clamped to -125 so that the result stays a normal float (~2e-38 there).
constexpr int POLY_PAIRS = VDN_SOFTMAX_POLY_PAIRS;  // pairs of every 16 computed this way
static_assert(POLY_PAIRS >= 0 && POLY_PAIRS <= 16, "pairs per 32-key chunk");

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 j = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
  const float2 n = __fadd2_rn(j, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(make_float2(0.05517132f, 0.05517132f), f, make_float2(0.24261054f, 0.24261054f));
  p = __ffma2_rn(p, f, make_float2(0.69326097f, 0.69326097f));
  p = __ffma2_rn(p, f, make_float2(0.99992812f, 0.99992812f));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(j.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(j.y) << 23)));
}

// pair i of a 16-pair chunk goes through the polynomial (spread evenly over the chunk;
// a compile-time constant once the loops are unrolled)
__device__ __forceinline__ constexpr bool poly_pair(int i) {
  return ((i + 1) * POLY_PAIRS) / 16 > (i * POLY_PAIRS) / 16;
}

__device__ __forceinline__ float2 exp2_pair(float2 x, int i) {
  if (poly_pair(i)) return exp2_poly2(x);
  return make_float2(ex2(x.x), ex2(x.y));
}

__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_CTRL));
}
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
}

// three-input max of sm_100 (half the instructions of a pairwise max tree)
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int D, bool FP8>
__global__ void __launch_bounds__(THREADS, 1)
    softmax_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKt,
                      const __grid_constant__ CUtensorMap tmVt, Dims d, float sl2, const float *__restrict__ scales,
                      void *__restrict__ out, int64_t out_row_stride, const float *__restrict__ w_gate_s,
                      float *__restrict__ lse, const int32_t *__restrict__ gtab, const int32_t *__restrict__ tiles,
                      int out8, DevStatus *st) {
  using C = Cfg<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  Bars *bars = reinterpret_cast<Bars *>(base + C::BAR_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int *abort_flag = &bars->abort;
  __shared__ int skip;  // an earlier block gave up: do no more work (block-uniform decision)
  if (threadIdx.x == 0) skip = *(volatile uint32_t *)&st->code != 0u;
  __syncthreads();
  if (skip) return;

  if (threadIdx.x == 0) {
    // Blocks [H*first, H*(first+count)) belong to the group whose tiles are
    // first..first+count-1 in the tile list; inside that range the head varies slowest, so
    // the blocks that run together share one head's keys and values in L2.
    const int32_t *t0 = tiles + (int64_t)(blockIdx.x / d.H) * TILE_REC;
    const int first = t0[4], count = t0[5];
    const int rel = (int)(blockIdx.x - (unsigned)first * d.H);
    const int64_t ti = first + rel % count;
    const int32_t *tr = tiles + ti * TILE_REC;
    bars->h = rel / count;
    bars->row0 = tr[1];
    bars->row_end = tr[2];
    kv_parts(gtab + tr[0] * 16, d.L, bars->parts);
    bars->nkv = kv_tiles(bars->parts);
    // range-check build: the tile, its group, its rows, its head and every key part must lie
    // inside their tensors; a block that fails does no work
    bool in = in_range(st, ti, max_tiles(d.F, d.T, d.C), K_SOFTMAX_TC, 1) &&
              in_range(st, tr[0], max_groups(d.F, d.C), K_SOFTMAX_TC, 2) &&
              in_range(st, bars->row0, d.Nv(), K_SOFTMAX_TC, 3) &&
              in_range(st, bars->row_end - 1, d.Nv(), K_SOFTMAX_TC, 4) &&
              in_range(st, bars->h, d.H, K_SOFTMAX_TC, 5) &&
              in_range(st, (int64_t)bars->h * D + D - 1, out_row_stride, K_SOFTMAX_TC, 6);
    for (int i = 0; in && i < bars->parts.n; ++i)
      in = in_range(st, bars->parts.lo[i], bars->parts.text[i] ? d.L : d.Nv(), K_SOFTMAX_TC, 7) &&
           in_range(st, bars->parts.hi[i] - 1, bars->parts.text[i] ? d.L : d.Nv(), K_SOFTMAX_TC, 8);
    if (!in) { bars->nkv = 0; bars->row_end = bars->row0; }
  }
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int s = 0; s < KST; ++s) { mbar_init(smem_u32(&bars->k_full[s]), 1); mbar_init(smem_u32(&bars->k_empty[s]), 1); }
    for (int s = 0; s < VST; ++s) { mbar_init(smem_u32(&bars->v_full[s]), 1); mbar_init(smem_u32(&bars->v_empty[s]), 1); }
    for (int w = 0; w < NQ; ++w) {
      mbar_init(smem_u32(&bars->s_full[w]), 1);
      for (int i = 0; i < C::P_PARTS; ++i) mbar_init(smem_u32(&bars->p_ready[w][i]), 4);
    }
    mbar_init(smem_u32(&bars->o_done), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
    tma_prefetch(&tmQ); tma_prefetch(&tmK); tma_prefetch(&tmV); tma_prefetch(&tmKt); tma_prefetch(&tmVt);
  }
  if (warp == 1) { tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
  reg_dealloc();
  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const int h = bars->h, row0 = bars->row0, nkv = bars->nkv;
      const KvParts &parts = bars->parts;
      uint32_t armed_k = 0, ph_k = 0, armed_v = 0, ph_v = 0;
      const uint32_t qb = smem_u32(&bars->q_full);
      mbar_arrive_expect_tx(qb, NQ * C::TILE_BYTES);
      for (int w = 0; w < NQ; ++w)
        for (int c = 0; c < C::BOXES; ++c)
          tma_load_2d(smem_u32(base + C::Q_OFF + w * C::TILE_BYTES + c * BM * 128), &tmQ, qb,
                      h * D + c * C::BOX_ELEMS, row0 + w * BM);
      // K runs one tile ahead of V: K_{j+1} is needed as soon as P_j V_j is issued, V_j only
      // after the softmax of tile j
      KvCursor ck, cv;
      ck.init(parts);
      cv.init(parts);
      auto load_k = [&](int j) -> bool {
        const int ks = j % KST;
        if (!mbar_wait(smem_u32(&bars->k_empty[ks]), ((j / KST) & 1) ^ 1, abort_flag, st, K_SOFTMAX_TC, 1))
          return false;
        const uint32_t kb = smem_u32(&bars->k_full[ks]);
        mbar_arrive_expect_tx(kb, C::TILE_BYTES);
        const CUtensorMap *mk = parts.text[ck.part] ? &tmKt : &tmK;
        for (int c = 0; c < C::BOXES; ++c)
          tma_load_2d(smem_u32(base + C::K_OFF + ks * C::TILE_BYTES + c * BN * 128), mk, kb, h * D + c * C::BOX_ELEMS,
                      ck.row);
        armed_k |= 1u << ks;
        ph_k = (ph_k & ~(1u << ks)) | (((j / KST) & 1u) << ks);
        ck.next(parts);
        return true;
      };
      bool go = nkv > 0 && load_k(0);
      for (int j = 0; go && j < nkv; ++j) {
        if (j + 1 < nkv && !load_k(j + 1)) break;
        const int vs = j % VST;
        if (!mbar_wait(smem_u32(&bars->v_empty[vs]), ((j / VST) & 1) ^ 1, abort_flag, st, K_SOFTMAX_TC, 2)) break;
        const uint32_t vb = smem_u32(&bars->v_full[vs]);
        mbar_arrive_expect_tx(vb, C::TILE_BYTES);
        const CUtensorMap *mv = parts.text[cv.part] ? &tmVt : &tmV;
        for (int c = 0; c < C::BOXES; ++c)
          tma_load_2d(smem_u32(base + C::V_OFF + vs * C::TILE_BYTES + c * BN * 128), mv, vb, h * D + c * C::BOX_ELEMS,
                      cv.row);
        armed_v |= 1u << vs;
        ph_v = (ph_v & ~(1u << vs)) | (((j / VST) & 1u) << vs);
        cv.next(parts);
      }
      // loads issued here land before the block leaves (bounded waits)
      int no_abort = 0;
      mbar_wait(qb, 0, &no_abort, st, K_SOFTMAX_TC, 10);
      for (int s = 0; s < KST; ++s)
        if (armed_k & (1u << s)) mbar_wait(smem_u32(&bars->k_full[s]), (ph_k >> s) & 1u, &no_abort, st, K_SOFTMAX_TC, 11);
      for (int s = 0; s < VST; ++s)
        if (armed_v & (1u << s)) mbar_wait(smem_u32(&bars->v_full[s]), (ph_v >> s) & 1u, &no_abort, st, K_SOFTMAX_TC, 12);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const int nkv = bars->nkv;
      const uint32_t qa = smem_u32(base + C::Q_OFF);
      auto issue_s = [&](int w, int j) {
        const uint32_t kbase = smem_u32(base + C::K_OFF + (j % KST) * C::TILE_BYTES);
        const uint32_t abase = qa + w * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / C::KSTEP; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;  // 32-byte K-steps, 4 per box row
          if (FP8)
            mma_ss_f8(tmem + C::s_col(w), sdesc(abase + off, 16, 1024), sdesc(kbase + off, 16, 1024), C::IDESC_S,
                      kk > 0);
          else
            mma_ss(tmem + C::s_col(w), sdesc(abase + off, 16, 1024), sdesc(kbase + off, 16, 1024), C::IDESC_S,
                   kk > 0);
        }
        mma_commit(smem_u32(&bars->s_full[w]));
      };
      bool ok = mbar_wait(smem_u32(&bars->q_full), 0, abort_flag, st, K_SOFTMAX_TC, 3);
      if (ok) ok = mbar_wait(smem_u32(&bars->k_full[0]), 0, abort_flag, st, K_SOFTMAX_TC, 4);
      // Q tile 1 starts half a step behind Q tile 0: its first S is issued only once P_0 of
      // tile 0 is ready.  In steady state each warpgroup then exponentiates while the tensor
      // cores run the other one's P.V and next S, instead of both competing for the
      // exponential units at the same time.
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int vs = j % VST;
        const bool more = j + 1 < nkv;
        const uint32_t vbase = smem_u32(base + C::V_OFF + vs * C::TILE_BYTES);
        for (int w = 0; w < NQ && ok; ++w) {
          // each wait sits right before the first MMA that needs it
          if (!mbar_wait(smem_u32(&bars->p_ready[w][0]), j & 1, abort_flag, st, K_SOFTMAX_TC, 7)) { ok = false; break; }
          if (w == 0 && !mbar_wait(smem_u32(&bars->v_full[vs]), (j / VST) & 1, abort_flag, st, K_SOFTMAX_TC, 5)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // O_w += P_w V_j: P_w (two bf16 or four e4m3 per column) sits over the first columns
          // of S_w; each K-step takes 8 of those columns and KSTEP rows of V (128 bytes each).
          // Each piece of P goes as soon as it is written, while the softmax warps still
          // exponentiate the next.
          constexpr int KSTEPS = BN / C::KSTEP, KPART = KSTEPS / C::P_PARTS;
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk) {
            if (kk > 0 && kk % KPART == 0) {
              if (!mbar_wait(smem_u32(&bars->p_ready[w][kk / KPART]), j & 1, abort_flag, st, K_SOFTMAX_TC, 15)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            const uint64_t bdesc = sdesc(vbase + kk * (C::KSTEP * 128), BM * 128, 1024);
            if (FP8)
              mma_ts_f8(tmem + C::o_col(w), tmem + C::s_col(w) + kk * 8, bdesc, C::IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
            else
              mma_ts(tmem + C::o_col(w), tmem + C::s_col(w) + kk * 8, bdesc, C::IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
          }
          if (!ok) break;
          if (j == 0 && w == 0) {
            issue_s(1, 0);                               // staggered start of Q tile 1
            mma_commit(smem_u32(&bars->k_empty[0]));     // K tile 0 is free once both S of it complete
          }
          if (more) {
            if (w == 0 && !mbar_wait(smem_u32(&bars->k_full[(j + 1) % KST]), ((j + 1) / KST) & 1, abort_flag, st,
                                     K_SOFTMAX_TC, 6)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(w, j + 1);
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&bars->v_empty[vs]));
        if (more) mma_commit(smem_u32(&bars->k_empty[(j + 1) % KST]));
      }
      mma_commit(smem_u32(&bars->o_done));
      mma_commit(smem_u32(&bars->drain));
      int no_abort = 0;
      mbar_wait(smem_u32(&bars->drain), 0, &no_abort, st, K_SOFTMAX_TC, 8);
    }
  }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    reg_alloc();
    const int h = bars->h, row0 = bars->row0, row_end = bars->row_end, nkv = bars->nkv;
    const KvParts &parts = bars->parts;
    // e4m3: scores carry s_q * s_k, the output s_v (per-head dequantisation scales)
    if (FP8) sl2 *= scales[h] * scales[d.H + h];
    const float out_scale = FP8 ? scales[2 * d.H + h] : 1.f;
    const int w = (warp >> 2) - 1;          // Q tile of this warpgroup
    const int quad = warp & 3;              // tensor-memory lane quadrant
    const int r = quad * 32 + lane;         // row within the Q tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + C::s_col(w);
    const uint32_t o_addr = tmem + lane_off + C::o_col(w);
    float m = -INFINITY, l = 0.f;
    KvCursor cur;
    cur.init(parts);
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int nvalid = min(BN, parts.hi[cur.part] - cur.row);
      cur.next(parts);
      // the warp proceeds (or gives up) as a whole: tensor-memory access is warp-collective
      const bool got = mbar_wait(smem_u32(&bars->s_full[w]), j & 1, abort_flag, st, K_SOFTMAX_TC, 9);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      float s[BN];
      float alpha = 1.f;
      float2 rs2[4];              // row sum in four independent pair chains
#pragma unroll
      for (int i = 0; i < 4; ++i) rs2[i] = make_float2(0.f, 0.f);
      const float2 sl2v = make_float2(sl2, sl2);
      // P of keys [0, c + 32) (and the rescaled O) handed to the MMA thread at the end of
      // each piece
      auto hand_piece = [&](int c) {
        if ((c + 32) % (BN / C::P_PARTS) == 0) {
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->p_ready[w][(c + 32) / (BN / C::P_PARTS) - 1]));
        }
      };
      // O_w was last written by P V of tile j-1, which completed before S_w of tile j; it is
      // rescaled before any P of tile j is handed to the tensor cores
      auto rescale_o = [&]() {
#pragma unroll 1
        for (int c = 0; c < D; c += 8) {  // 8 columns at a time: the row of S is still live
          uint32_t u[8];
          tmem_ld8(o_addr + c, u);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
          tmem_st8(o_addr + c, u);
        }
      };
      // bf16: x = s * scale - m, 2^x and the row sum of one 32-key chunk on pairs of values
      // (packed fp32 instructions), P over the chunk's first 16 columns
      auto exp_chunk_bf16 = [&](int c, float2 negm) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 p = exp2_pair(__ffma2_rn(make_float2(s[c + 2 * i], s[c + 2 * i + 1]), sl2v, negm), i);
          rs2[i & 3] = __fadd2_rn(rs2[i & 3], p);
          pk[i] = pack_bf16(p.x, p.y);
        }
        tmem_st16(s_addr + (c >> 1), pk);
      };
      {
      // the whole row of S in one round trip: four loads in flight, one wait
      {
        uint32_t u0[32], u1[32], u2[32], u3[32];
        tmem_ld32(s_addr + 0, u0);
        tmem_ld32(s_addr + 32, u1);
        tmem_ld32(s_addr + 64, u2);
        tmem_ld32(s_addr + 96, u3);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = __uint_as_float(u0[i]);
          s[32 + i] = __uint_as_float(u1[i]);
          s[64 + i] = __uint_as_float(u2[i]);
          s[96 + i] = __uint_as_float(u3[i]);
        }
      }
      if (nvalid < BN) {
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (i >= nvalid) s[i] = -INFINITY;
      }
      // row max as a tree of three-input maxima (eight independent chains)
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        mx8[k] = s[k];
#pragma unroll
        for (int t = 0; t < 7; ++t) mx8[k] = max3(mx8[k], s[8 + 16 * t + k], s[16 + 16 * t + k]);
        mx8[k] = fmaxf(mx8[k], s[120 + k]);
      }
      const float mx = fmaxf(max3(mx8[0], mx8[1], mx8[2]), max3(mx8[3], mx8[4], max3(mx8[5], mx8[6], mx8[7])));
      const float m_new = fmaxf(m, mx * sl2);
      const bool need = __any_sync(0xffffffffu, m_new > m + RESCALE_THRESHOLD);
      if (need) {
        alpha = ex2(m - m_new);   // 0 on the first tile (m = -inf)
        m = m_new;
      }
      if (need && j > 0) rescale_o();
      const float2 negm = make_float2(-m, -m);
      if (FP8) {
        // e4m3 P at unit scale, four per tensor-memory column (p <= 2^8 < 448)
#pragma unroll
        for (int c = 0; c < BN; c += 32) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 p0 = exp2_pair(__ffma2_rn(make_float2(s[c + 4 * i], s[c + 4 * i + 1]), sl2v, negm), 2 * i);
            const float2 p1 =
                exp2_pair(__ffma2_rn(make_float2(s[c + 4 * i + 2], s[c + 4 * i + 3]), sl2v, negm), 2 * i + 1);
            rs2[(2 * i) & 3] = __fadd2_rn(rs2[(2 * i) & 3], p0);
            rs2[(2 * i + 1) & 3] = __fadd2_rn(rs2[(2 * i + 1) & 3], p1);
            const uint32_t lo = __nv_cvt_float2_to_fp8x2(p0, __NV_SATFINITE, __NV_E4M3);
            const uint32_t hi = __nv_cvt_float2_to_fp8x2(p1, __NV_SATFINITE, __NV_E4M3);
            pk[i] = (lo & 0xffffu) | (hi << 16);
          }
          tmem_st8(s_addr + (c >> 2), pk);
          hand_piece(c);
        }
      } else {
#pragma unroll
        for (int c = 0; c < BN; c += 32) {
          exp_chunk_bf16(c, negm);
          hand_piece(c);
        }
      }
      }
      const float2 rsa = __fadd2_rn(__fadd2_rn(rs2[0], rs2[1]), __fadd2_rn(rs2[2], rs2[3]));
      const float rs = rsa.x + rsa.y;
      l = l * alpha + rs;
    }
    // ------------------------------------------------------------ epilogue
    const bool done = ok && mbar_wait(smem_u32(&bars->o_done), 0, abort_flag, st, K_SOFTMAX_TC, 13);
    if (__all_sync(0xffffffffu, done)) {
      tc_fence_after();
      const int row = row0 + w * BM + r;
      const bool valid = row < row_end;
      float inv = out_scale / l;
      if (w_gate_s != nullptr) {
        // softmax gate of the layer, g_s = sigmoid(q . w_s[h]) from this row of Q in shared
        // memory (128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r & 7))
        mbar_wait(smem_u32(&bars->q_full), 0, abort_flag, st, K_SOFTMAX_TC, 14);
        const uint8_t *qt = base + C::Q_OFF + w * C::TILE_BYTES;
        const float *ws_h = w_gate_s + h * D;
        float dot = 0.f;
        constexpr int PER_CHUNK = 16 / C::EB;  // elements per 16-byte chunk
#pragma unroll 1
        for (int cl = 0; cl < D / PER_CHUNK; ++cl) {
          const uint4 raw = *reinterpret_cast<const uint4 *>(qt + (cl >> 3) * (BM * 128) + r * 128 +
                                                               (((cl & 7) ^ (r & 7)) << 4));
          if (FP8) {
            // dequantised e4m3 q (the per-head scale is applied once below)
            const __nv_fp8x2_storage_t *pp = reinterpret_cast<const __nv_fp8x2_storage_t *>(&raw);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pp[e], __NV_E4M3);
              const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
              dot = fmaf(f.x, __ldg(ws_h + cl * 16 + 2 * e), dot);
              dot = fmaf(f.y, __ldg(ws_h + cl * 16 + 2 * e + 1), dot);
            }
          } else {
            const __nv_bfloat162 *hp = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(hp[e]);
              dot = fmaf(f.x, __ldg(ws_h + cl * 8 + 2 * e), dot);
              dot = fmaf(f.y, __ldg(ws_h + cl * 8 + 2 * e + 1), dot);
            }
          }
        }
        if (FP8) dot *= scales[h];  // s_q
        inv *= 1.f / (1.f + expf(-dot));
      }
      if (out8) {
        // e4m3 codes of g_s O / l in units of the V scale, which is then A_s's dequantisation
        // scale: |g_s O| <= amax(V), so the codes stay within e4m3's 448
        const float inv8 = inv / out_scale;
        uint8_t *orow = (uint8_t *)out + (int64_t)row * out_row_stride + (int64_t)h * D;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t u[32];
          tmem_ld32(o_addr + c, u);
          tmem_wait_ld();
          if (valid) {
            uint32_t w4[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t lo = __nv_cvt_float2_to_fp8x2(
                  make_float2(__uint_as_float(u[4 * i]) * inv8, __uint_as_float(u[4 * i + 1]) * inv8), __NV_SATFINITE,
                  __NV_E4M3);
              const uint32_t hi = __nv_cvt_float2_to_fp8x2(
                  make_float2(__uint_as_float(u[4 * i + 2]) * inv8, __uint_as_float(u[4 * i + 3]) * inv8),
                  __NV_SATFINITE, __NV_E4M3);
              w4[i] = (lo & 0xffffu) | (hi << 16);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
            dst[0] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            dst[1] = make_uint4(w4[4], w4[5], w4[6], w4[7]);
          }
        }
      } else {
        __nv_bfloat16 *orow = (__nv_bfloat16 *)out + (int64_t)row * out_row_stride + (int64_t)h * D;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t u[32];
          tmem_ld32(o_addr + c, u);
          tmem_wait_ld();
          if (valid) {
            uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o;
              o.x = pack_bf16(__uint_as_float(u[8 * v + 0]) * inv, __uint_as_float(u[8 * v + 1]) * inv);
              o.y = pack_bf16(__uint_as_float(u[8 * v + 2]) * inv, __uint_as_float(u[8 * v + 3]) * inv);
              o.z = pack_bf16(__uint_as_float(u[8 * v + 4]) * inv, __uint_as_float(u[8 * v + 5]) * inv);
              o.w = pack_bf16(__uint_as_float(u[8 * v + 6]) * inv, __uint_as_float(u[8 * v + 7]) * inv);
              dst[v] = o;
            }
          }
        }
      }
      if (valid && lse != nullptr) lse[(int64_t)row * d.H + h] = (m + __log2f(l)) * 0.69314718055994530942f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

template <int D, bool FP8>
cudaError_t launch_t(const Dims &d, const void *q, const void *k, const void *v, const void *kt, const void *vt,
                     const float *scales, float sl2, void *o, int64_t o_row_stride, const float *w_gate_s,
                     float *lse, char *ws, const WsPlan &p, cudaStream_t st, bool out8 = false) {
  using C = Cfg<D, FP8>;
  const uint64_t HD = (uint64_t)d.H * D;
  const CUtensorMapDataType dt = FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap mq, mk, mv, mkt, mvt;
  uint64_t strides[1] = {HD * C::EB};
  uint32_t box[2] = {(uint32_t)C::BOX_ELEMS, BM};
  uint64_t dims_v[2] = {HD, (uint64_t)d.Nv()};
  uint64_t dims_t[2] = {HD, (uint64_t)(d.L > 0 ? d.L : 1)};
  const void *kt_base = d.L > 0 ? kt : k, *vt_base = d.L > 0 ? vt : v;  // unused when there is no text
  if (!encode_tmap(&mq, dt, 2, q, dims_v, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&mk, dt, 2, k, dims_v, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&mv, dt, 2, v, dims_v, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&mkt, dt, 2, kt_base, dims_t, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&mvt, dt, 2, vt_base, dims_t, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int ntiles = host_tile_count(d);
  cudaError_t e = cudaFuncSetAttribute(softmax_tc_kernel<D, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem_bytes<D, FP8>());
  if (e != cudaSuccess) return e;
  softmax_tc_kernel<D, FP8><<<ntiles * d.H, THREADS, smem_bytes<D, FP8>(), st>>>(
      mq, mk, mv, mkt, mvt, d, sl2, scales, o, o_row_stride, w_gate_s, lse, (const int32_t *)(ws + p.gtab),
      (const int32_t *)(ws + p.tiles), out8 ? 1 : 0, (DevStatus *)(ws + p.status));
  return cudaGetLastError();
}

}  // namespace

bool softmax_tc_supported(const Dims &d, vdn_dtype dt) {
  return (dt == VDN_BF16 && (d.D == 64 || d.D == 128)) || (dt == VDN_E4M3 && d.D == 128);
}

cudaError_t launch_softmax_tc(const Dims &d, vdn_dtype dt, const void *q, const void *k, const void *v,
                              const void *kt, const void *vt, const float *scales, float sl2, void *o, float *lse,
                              char *ws, const WsPlan &p, cudaStream_t st) {
  const int64_t HD = (int64_t)d.H * d.D;
  if (dt == VDN_E4M3 && d.D == 128)
    return launch_t<128, true>(d, q, k, v, kt, vt, scales, sl2, o, HD, nullptr, lse, ws, p, st);
  if (dt != VDN_BF16) return cudaErrorInvalidValue;
  if (d.D == 128) return launch_t<128, false>(d, q, k, v, kt, vt, nullptr, sl2, o, HD, nullptr, lse, ws, p, st);
  if (d.D == 64) return launch_t<64, false>(d, q, k, v, kt, vt, nullptr, sl2, o, HD, nullptr, lse, ws, p, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_softmax_tc_gated(const Dims &d, vdn_dtype dt, const void *q, const void *k, const void *v,
                                    const void *kt, const void *vt, const float *scales, const float *w_gate_s,
                                    float sl2, void *a, char *ws, const WsPlan &p, cudaStream_t st, bool a8) {
  const int64_t stride = 2 * (int64_t)d.H * d.D;  // A = [A_s | A_l]: the softmax half of each row
  if (dt == VDN_E4M3 && d.D == 128)
    return launch_t<128, true>(d, q, k, v, kt, vt, scales, sl2, a, stride, w_gate_s, nullptr, ws, p, st, a8);
  if (a8) return cudaErrorInvalidValue;
  if (dt != VDN_BF16) return cudaErrorInvalidValue;
  if (d.D == 128) return launch_t<128, false>(d, q, k, v, kt, vt, nullptr, sl2, a, stride, w_gate_s, nullptr, ws, p, st);
  if (d.D == 64) return launch_t<64, false>(d, q, k, v, kt, vt, nullptr, sl2, a, stride, w_gate_s, nullptr, ws, p, st);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
