// Linear branch on the 5th-generation tensor cores (bf16 inputs, head dim 128).
// ("VDN-MiniMax-H3 开源" article, 技术解读 / 局部精确计算: a frame-wise linear branch
// whose forward and backward memories are read at the query position; 独立门控: the
// linear output is RMS-normalised and gated element-wise.)
//
// state_build_tc: S_f = phi(K_f)^T V_f and z_f = sum phi(K_f) for one (frame or text,
//   head) per CTA.  TMA streams 64-token K/V tiles into a 3-stage ring; eight warps apply
//   phi = elu+1 in place in shared memory (masking tokens past the frame) and sum z;
//   one thread issues tcgen05.mma with both operands MN-major (M = key feature, N =
//   value dim, K = tokens) into a 128x128 fp32 accumulator in tensor memory.
// read_stage: the linear-gate weights converted to bf16 and, where the scan left fp32
//   memories (step entry points, delta rule), S_fwd + S_bwd of every group summed into
//   bf16 (the MMA B operand) and the normalisers summed.
// read_tc: 128 query rows of one group and head per CTA, two CTAs per SM.  Two threads per
//   row (one per column half) build phi(q) (or q/|q| for the delta rule) and the
//   normaliser phi(q).z while thread 0's MMA forms the gate logits Q W_l, write the
//   features over Q, and after num = phi(Q) S_sum form o = num / den and store o or the
//   gated, RMS-normalised A_l (staged in shared memory, whole rows per store) into the
//   linear half of A.
#include "tc_common.cuh"

namespace vdn {
namespace {

using namespace tc;

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 16-byte chunk `cl` (8 bf16 of columns 8cl..8cl+7) of row r in a tile stored as
// 64-column boxes of `box_rows` rows with the 128-byte swizzle
__device__ __forceinline__ uint32_t swz_off(int r, int cl, int box_rows) {
  return (uint32_t)((cl >> 3) * box_rows * 128 + r * 128 + ((((cl & 7) ^ (r & 7))) << 4));
}

__device__ __forceinline__ uint4 pack8(const float *f) {
  uint4 u;
  u.x = pack_bf16(f[0], f[1]); u.y = pack_bf16(f[2], f[3]); u.z = pack_bf16(f[4], f[5]); u.w = pack_bf16(f[6], f[7]);
  return u;
}

// 2^x with the hardware approximation (flushes subnormal results to zero)
__device__ __forceinline__ float ex2_sb(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ============================================================================ state build
// Persistent: every CTA walks the (frame or text, head group) items blockIdx.x, blockIdx.x +
// gridDim.x, ... (head groups vary fastest, so the CTAs in flight read whole token rows of K
// and V), two CTAs per SM.  A head group is 128 features: one head of D = 128, or 128 / D
// heads of D = 64 or 32, whose states are the diagonal D x D blocks of the group's 128 x 128
// product (the tensor cores compute the off-diagonal blocks too, for free: the kernel is
// bound by HBM).  The TMA ring of 64-token chunks runs on across items, so no CTA
// waits for its first loads after the first item; the accumulator alternates between two
// 128-column halves of tensor memory, so the MMAs of an item start while the previous
// item's S is still being read out.
namespace sb {
constexpr int D = 128, TK = 64, NS = 3, THREADS = 320, PHI_WARPS = 8;
constexpr int BOX_BYTES = TK * 128;        // 64 tokens x 64 bf16
constexpr int TILE_BYTES = 2 * BOX_BYTES;  // 64 tokens x 128 features
constexpr int STAGE_BYTES = 2 * TILE_BYTES;
constexpr uint32_t IDESC = idesc_bf16(128, 128, true, true);
constexpr uint32_t TMEM_COLS = 256;        // two accumulators of 128 columns
struct alignas(8) Bars {
  uint64_t full[NS], phi[NS], empty[NS], acc_full[2], acc_empty[2], drain;
  uint32_t tmem;
  int abort;
  float zpart[PHI_WARPS][D];  // z of each phi warp, summed in a fixed order (repeatable bits)
};
constexpr size_t SMEM = 1024 + NS * STAGE_BYTES + sizeof(Bars);

// item x: frame fr = x / Hg (fr == F: the text), head group h = x % Hg; its rows and tokens
struct Item {
  int h, fr, row_base, ntok, nch;
  bool text;
};
__device__ __forceinline__ Item item_of(const Dims &d, int Hg, int x) {
  Item it;
  it.h = x % Hg;
  it.fr = x / Hg;
  it.text = it.fr == d.F;
  it.ntok = it.text ? d.L : d.T;
  it.row_base = it.text ? 0 : it.fr * d.T;
  it.nch = (it.ntok + TK - 1) / TK;
  return it;
}
}  // namespace sb

__global__ void __launch_bounds__(sb::THREADS, 2)
    state_build_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmKt, const __grid_constant__ CUtensorMap tmVt, Dims d,
                          float *__restrict__ S, float *__restrict__ z, float *__restrict__ St,
                          float *__restrict__ zt, DevStatus *st) {
  using namespace sb;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  Bars *bars = reinterpret_cast<Bars *>(base + NS * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int *abort_flag = &bars->abort;
  __shared__ int skip;
  if (threadIdx.x == 0) skip = *(volatile uint32_t *)&st->code != 0u;
  __syncthreads();
  if (skip) return;
  const int Hg = d.H * d.D / D;  // head groups of 128 features
  const int n_items = (d.F + 1) * Hg;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->phi[s]), PHI_WARPS);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->acc_full[b]), 1);
      mbar_init(smem_u32(&bars->acc_empty[b]), PHI_WARPS);
    }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(smem_u32(&bars->tmem), TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;

  // Every role walks the same items and chunks in the same order: the ring slot of global
  // chunk gc is gc % NS with phase (gc / NS) & 1, and the accumulator of the n-th item that
  // has chunks is n & 1 with phase (n >> 1) & 1.
  if (warp == 0) {
    if (lane == 0) {
      uint32_t armed = 0, armed_ph = 0;
      int gc = 0;
      bool go = true;
      for (int x = blockIdx.x; go && x < n_items; x += gridDim.x) {
        const Item it = item_of(d, Hg, x);
        const CUtensorMap *mk = it.text ? &tmKt : &tmK;
        const CUtensorMap *mv = it.text ? &tmVt : &tmV;
        for (int c = 0; c < it.nch; ++c, ++gc) {
          const int s = gc % NS;
          if (!mbar_wait(smem_u32(&bars->empty[s]), ((gc / NS) & 1) ^ 1, abort_flag, st, K_STATE_TC, 1)) {
            go = false;
            break;
          }
          const uint32_t fb = smem_u32(&bars->full[s]);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          uint8_t *stg = base + s * STAGE_BYTES;
          for (int bx = 0; bx < 2; ++bx) {
            tma_load_2d(smem_u32(stg + bx * BOX_BYTES), mk, fb, it.h * D + bx * 64, it.row_base + c * TK);
            tma_load_2d(smem_u32(stg + TILE_BYTES + bx * BOX_BYTES), mv, fb, it.h * D + bx * 64,
                        it.row_base + c * TK);
          }
          armed |= 1u << s;
          armed_ph = (armed_ph & ~(1u << s)) | (((gc / NS) & 1u) << s);
        }
      }
      int no_abort = 0;
      for (int s = 0; s < NS; ++s)
        if (armed & (1u << s)) mbar_wait(smem_u32(&bars->full[s]), (armed_ph >> s) & 1u, &no_abort, st, K_STATE_TC, 2);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int gc = 0, na = 0;
      bool ok = true;
      for (int x = blockIdx.x; ok && x < n_items; x += gridDim.x) {
        const Item it = item_of(d, Hg, x);
        if (it.nch == 0) continue;
        const int b = na & 1;
        // the accumulator's previous item has been read out
        if (!mbar_wait(smem_u32(&bars->acc_empty[b]), ((na >> 1) & 1) ^ 1, abort_flag, st, K_STATE_TC, 3)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(b * 128);
        for (int c = 0; c < it.nch; ++c, ++gc) {
          const int s = gc % NS;
          if (!mbar_wait(smem_u32(&bars->phi[s]), (gc / NS) & 1, abort_flag, st, K_STATE_TC, 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = smem_u32(base + s * STAGE_BYTES), vb = kb + TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < TK / 16; ++kk)
            mma_ss(acc, sdesc(kb + kk * 2048, BOX_BYTES, 1024), sdesc(vb + kk * 2048, BOX_BYTES, 1024), IDESC,
                   (c | kk) != 0);
          mma_commit(smem_u32(&bars->empty[s]));
        }
        if (!ok) break;
        mma_commit(smem_u32(&bars->acc_full[b]));
        ++na;
      }
      mma_commit(smem_u32(&bars->drain));
      int no_abort = 0;
      mbar_wait(smem_u32(&bars->drain), 0, &no_abort, st, K_STATE_TC, 5);
    }
  } else {
    // ---------------- phi pass (in place, masked) and z; then each item's epilogue
    const int tid = threadIdx.x - 64;
    const int cl = tid & 15, rg = tid >> 4;  // column chunk 8cl..8cl+7; rows rg + 16i
    const int quad = warp & 3, c_lo = ((warp - 2) >> 2) * (D / 2);  // lane quarter; column half
    const int i_row = quad * 32 + lane;  // key feature = accumulator row = tensor-memory lane
    int gc = 0, na = 0;
    bool ok = true;
    for (int x = blockIdx.x; x < n_items; x += gridDim.x) {
      const Item it = item_of(d, Hg, x);
      float zacc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) zacc[e] = 0.f;
      for (int c = 0; c < it.nch; ++c, ++gc) {
        const int s = gc % NS;
        if (ok) ok = mbar_wait(smem_u32(&bars->full[s]), (gc / NS) & 1, abort_flag, st, K_STATE_TC, 6);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        uint8_t *kt = base + s * STAGE_BYTES;
        // all four rows' loads first, so their latencies overlap (the stores below go to the
        // same tile, which the compiler would otherwise keep in order with the next load)
        constexpr int RI = TK / 16;
        uint4 raw[RI];
#pragma unroll
        for (int i = 0; i < RI; ++i) raw[i] = *reinterpret_cast<const uint4 *>(kt + swz_off(rg + 16 * i, cl, TK));
#pragma unroll
        for (int i = 0; i < RI; ++i) {
          const int r = rg + 16 * i;
          const bool valid = c * TK + r < it.ntok;
          const __nv_bfloat162 *hp = reinterpret_cast<const __nv_bfloat162 *>(&raw[i]);
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // phi = max(x, 0) + 2^(min(x, 0) log2 e) on pairs; phi enters the MMA in bf16, so
            // the hardware exponential is accurate enough
            const float2 x = __bfloat1622float2(hp[e]);
            const float2 t = __fmul2_rn(make_float2(fminf(x.x, 0.f), fminf(x.y, 0.f)),
                                        make_float2(1.4426950408889634f, 1.4426950408889634f));
            float2 ph = __fadd2_rn(make_float2(fmaxf(x.x, 0.f), fmaxf(x.y, 0.f)), make_float2(ex2_sb(t.x), ex2_sb(t.y)));
            if (!valid) ph = make_float2(0.f, 0.f);
            zacc[2 * e] += ph.x;
            zacc[2 * e + 1] += ph.y;
            w4[e] = pack_bf16(ph.x, ph.y);
          }
          *reinterpret_cast<uint4 *>(kt + swz_off(r, cl, TK)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->phi[s]));
      }
      // lanes l and l ^ 16 hold the same columns: pair them, then one row per warp
#pragma unroll
      for (int e = 0; e < 8; ++e) zacc[e] += __shfl_xor_sync(0xffffffffu, zacc[e], 16);
      named_bar_sync(1, 32 * PHI_WARPS);  // the previous item's z sums are read
      if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e) bars->zpart[warp - 2][cl * 8 + e] = zacc[e];
      }
      // this thread's accumulator row is key feature ii of head ph of the group
      const int dh = d.D, ph = i_row / dh, ii = i_row % dh, hh = it.h * (D / dh) + ph;
      float *So = (it.text ? St + (int64_t)hh * dh * dh : S + ((int64_t)it.fr * d.H + hh) * dh * dh) + (int64_t)ii * dh;
      if (it.nch > 0) {
        const int b = na & 1;
        const bool done = ok && mbar_wait(smem_u32(&bars->acc_full[b]), (na >> 1) & 1, abort_flag, st, K_STATE_TC, 7);
        ok = __all_sync(0xffffffffu, done);
        if (ok) {
          tc_fence_after();
          const uint32_t acc = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(b * 128) + c_lo;
          uint32_t u0[32], u1[32];
          tmem_ld32(acc, u0);
          tmem_ld32(acc + 32, u1);
          tmem_wait_ld();
          // this accumulator may take the next item's MMAs once every phi warp has read it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty[b]));
          // the 32-column chunks c_lo and c_lo + 32 that belong to head ph (the diagonal block)
          if (c_lo / dh == ph) {
            float4 *dst = reinterpret_cast<float4 *>(So + (c_lo - ph * dh));
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(__uint_as_float(u0[4 * v]), __uint_as_float(u0[4 * v + 1]),
                                   __uint_as_float(u0[4 * v + 2]), __uint_as_float(u0[4 * v + 3]));
          }
          if ((c_lo + 32) / dh == ph) {
            float4 *dst = reinterpret_cast<float4 *>(So + (c_lo + 32 - ph * dh));
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(__uint_as_float(u1[4 * v]), __uint_as_float(u1[4 * v + 1]),
                                   __uint_as_float(u1[4 * v + 2]), __uint_as_float(u1[4 * v + 3]));
          }
        }
        ++na;
      } else {
        // no tokens (an empty text): the head's block is zero
        for (int cc = 0; cc < D / 2; ++cc)
          if ((c_lo + cc) / dh == ph) So[c_lo + cc - ph * dh] = 0.f;
      }
      // every phi warp has written its share of z; their states are ANDed, so that all eight
      // leave the item loop together and their named barriers always pair up
      ok = named_bar_and(1, 32 * PHI_WARPS, ok);
      float *zo = it.text ? zt : z;
      if (zo != nullptr && tid < D) {
        float zs = 0.f;
#pragma unroll
        for (int pw = 0; pw < PHI_WARPS; ++pw) zs += bars->zpart[pw][tid];
        // the group's 128 features are its heads' z vectors back to back
        zo[(it.text ? (int64_t)it.h * D : (int64_t)it.fr * d.H * d.D + (int64_t)it.h * D) + tid] = zs;
      }
      if (!ok) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// ============================================================================ read staging
// Destination of the 8 consecutive entries starting at (row i, column j) of head h's D x D
// block in the block-diagonal bf16 layout [..][H / P][128][128] (P = 128 / D heads per head
// group); `lead` selects the leading index (group g for S_sum, nothing for W_l).  With
// D = 128 this is the plain [..][H][D][D] index.
__device__ __forceinline__ int64_t bdiag_index(int64_t lead, int H, int D, int h, int i, int j) {
  const int P = 128 / D, hg = h / P, pp = h % P;
  return ((lead * (H / P) + hg) * 128 + pp * D + i) * 128 + pp * D + j;
}

__global__ void __launch_bounds__(256) read_stage_kernel(int64_t n_s8, int64_t n_z, int64_t n_w8, int H, int D,
                                                         const float *__restrict__ Sf, const float *__restrict__ Sb,
                                                         const float *__restrict__ zf, const float *__restrict__ zb,
                                                         const float *__restrict__ wgl, __nv_bfloat16 *__restrict__ ssum,
                                                         float *__restrict__ zsum, __nv_bfloat16 *__restrict__ wl) {
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  const int64_t DD = (int64_t)D * D;
  if (i < n_s8) {
    const float4 *a = reinterpret_cast<const float4 *>(Sf + 8 * i), *b = reinterpret_cast<const float4 *>(Sb + 8 * i);
    const float4 a0 = a[0], a1 = a[1], b0 = b[0], b1 = b[1];
    const float f[8] = {a0.x + b0.x, a0.y + b0.y, a0.z + b0.z, a0.w + b0.w,
                        a1.x + b1.x, a1.y + b1.y, a1.z + b1.z, a1.w + b1.w};
    const int64_t e = 8 * i, gh = e / DD, rem = e % DD;
    *reinterpret_cast<uint4 *>(ssum + bdiag_index(gh / H, H, D, (int)(gh % H), (int)(rem / D), (int)(rem % D))) =
        pack8(f);
  } else if (i < n_s8 + n_z) {
    const int64_t j = i - n_s8;
    zsum[j] = zf[j] + zb[j];
  } else if (i < n_s8 + n_z + n_w8) {
    const int64_t e = 8 * (i - n_s8 - n_z), h = e / DD, rem = e % DD;
    const float4 *a = reinterpret_cast<const float4 *>(wgl + e);
    const float4 a0 = a[0], a1 = a[1];
    const float f[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    *reinterpret_cast<uint4 *>(wl + bdiag_index(0, H, D, (int)h, (int)(rem / D), (int)(rem % D))) = pack8(f);
  }
}

// ============================================================================ read (+ gate, RMSNorm)
// Persistent, one CTA per SM; CTA c takes a contiguous range of the work list.  An item is
// the 128-row half of a query tile for one head, listed head by head (a CTA keeps one
// head's gate weights W_l for long runs) and, inside a head, tile by tile in row order (so
// consecutive items of one group share the group memory S_sum).  Roles:
//   warp 0      TMA: Q tiles into a 3-stage ring, then W_l and S_sum into one slot each
//               when the item's head or group changes (each slot is a one-stage ring whose
//               refill waits for the release of the previous fill)
//   warp 1      one thread issues the MMAs: the gate logits Q W_l into tensor memory as
//               soon as the Q tile has landed, then num = feature * S_sum once the feature
//               rows are written; two accumulator sets of 256 columns
//   warps 4-11  two threads per query row, one per column half: that half of the feature
//               row phi(q), written over the Q tile once the gate MMA has read it, and its
//               share of the normaliser phi(q).z (delta rule: of |q|^2; the MMAs read q and
//               the epilogue divides by |q|) and (G_l = 1) of the scalar gate logit; then
//               (G_l = D) that half of the gate sigmoid(Q W_l), in place over its logits
//               in tensor memory
//   warps 12-19 epilogue, two threads per row: o = num / den from tensor memory, then o or
//               A_l = g_l * gamma * o / rms(o) (the halves' sums of squares meet in shared
//               memory), staged in shared memory and written by a TMA store that runs on
//               while the next item is computed (a short last tile of a group, whose box
//               would reach the next group's rows, with plain stores instead)
// (warps 2 and 3 have no role.)  Eight warps per role keep two of them on each scheduler,
// so that one covers the exponential-unit and memory latencies of the other.  The TMA loads of later tiles, the tensor cores, the feature
// rows of one item and the epilogue of the previous one overlap.  Every wait names the fill
// or use it expects with a phase parity that cannot be two phases behind: a slot is refilled
// only after its previous contents are released, and no release is issued before a use.
namespace rd {
constexpr int D = 128, BM = 128, HC = D / 2, NQ = 3, THREADS = 640;
constexpr int FEAT_WARP0 = 4, EPI_WARP0 = 12, ROLE_WARPS = 8;  // two threads per row: one per column half
constexpr int TILE_BYTES = BM * D * 2;  // 32 KB: one 128-row bf16 tile (two 64-column boxes)
// staged output tile: the TMA store's boxes with the 128-byte swizzle (bf16: two boxes of 64
// columns, 16 KB each; e4m3: one box of 128 columns)
constexpr int Q_OFF = 0, S_OFF = NQ * TILE_BYTES, W_OFF = S_OFF + TILE_BYTES, O_OFF = W_OFF + TILE_BYTES;
constexpr int BAR_OFF = O_OFF + TILE_BYTES;
constexpr uint32_t IDESC_NUM = idesc_bf16(BM, D, false, true);   // A K-major, B MN-major
constexpr uint32_t TMEM_COLS = 512;                               // set a: num at 256a, gate logits at 256a + 128
struct alignas(16) Bars {
  // with S_sum (one fill per group and head): the normaliser z and the scalar-gate weights
  float zs[D], wg1[D];
  float gam[D];                 // gamma of the epilogue's current head (staged by the epilogue)
  // per accumulator set and 32-column block of the row: shares of the normaliser (delta
  // rule: of |q|^2) and of the scalar-gate logit; the epilogue's sums of squares.  A head
  // of D features takes D / 32 consecutive blocks.
  float den[2][4][BM], g1[2][4][BM];
  float ssq[4][BM];
  uint64_t q_full[NQ], q_empty[NQ], gate_done[NQ], feat_full[NQ], den_full[2], acc_full[2], acc_empty[2];
  uint64_t s_full, s_empty, w_full, w_empty, drain;
  uint32_t tmem;
  int abort;
};
constexpr size_t SMEM = 1024 + BAR_OFF + sizeof(Bars);
static_assert(SMEM <= 227 * 1024, "shared memory of a block");
static_assert(BAR_OFF % 16 == 0, "barrier alignment");
}  // namespace rd

// 1 / (1 + 2^(-x log2 e)) with the hardware exp2 and reciprocal approximations (relative
// error near 2^-21); the result goes to bf16
__device__ __forceinline__ float fast_sigmoid(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

// The element-wise linear gate, sigmoid(x) = (1 + tanh(x/2)) / 2, with the hardware tanh
// approximation (relative error below 2^-10.9): within 2.5e-4 of sigmoid(x), about half a
// bf16 step of a gate of 1/8 and a tenth of one at 1/2, at one exponential-unit operation
// per element instead of two
__device__ __forceinline__ float tanh_fast(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(x));
  return t;
}
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct ReadItem {
  int g, h, row0, row_end;
};

// Item x of the work list: head x / (2 n_tiles), then the tiles in row order, two halves
// each.  False for the empty second half of a short tile, and (range-check build) for an
// item whose group or rows fall outside their tensors; every role decodes the same list,
// so all of them skip the same items.
__device__ __forceinline__ bool read_item(const int32_t *__restrict__ tiles, int n_tiles, const Dims &d,
                                          DevStatus *st, int64_t x, ReadItem &it) {
  const int64_t per_head = 2 * (int64_t)n_tiles;
  it.h = (int)(x / per_head);
  const int rem = (int)(x - (int64_t)it.h * per_head);
  const int32_t *tr = tiles + (int64_t)(rem >> 1) * TILE_REC;
  it.g = tr[0];
  it.row0 = tr[1] + (rem & 1) * rd::BM;
  it.row_end = tr[2];
  return it.row0 < it.row_end && in_range(st, it.g, max_groups(d.F, d.C), K_READ_TC, 2) &&
         in_range(st, it.row0, d.Nv(), K_READ_TC, 3) && in_range(st, it.row_end - 1, d.Nv(), K_READ_TC, 4);
}

// DELTA: q/|q| features and no normaliser; FUSED: RMSNorm and the linear gate (GATE_MMA:
// element-wise, G_l = D, on the tensor cores; otherwise the scalar gate, G_l = 1); AMAX:
// also the per-head max |q| into amax_q (for the e4m3 quantisation that follows); NB: the
// 32-column blocks of one head (D / 32: 4 for D = 128, whose halves of a row belong to one
// head; 2 or 1 for the 128 / D heads of a head group of D = 64 or 32)
template <bool DELTA, bool FUSED, bool GATE_MMA, bool AMAX, int NB>
__global__ void __launch_bounds__(rd::THREADS, 1)
    read_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS,
                   const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmO, Dims d,
                   const float *__restrict__ zsum, const float *__restrict__ wgl, int G_l,
                   const float *__restrict__ gamma, float eps, void *__restrict__ out, int64_t out_stride,
                   const int32_t *__restrict__ tiles, int n_tiles,
                   int64_t n_items, const float *__restrict__ a8_scale, uint32_t *__restrict__ amax_q,
                   DevStatus *st) {
  using namespace rd;
  constexpr bool delta = DELTA, fused = FUSED, gate_mma = FUSED && GATE_MMA, scalar_gate = FUSED && !GATE_MMA;
  constexpr bool amax = AMAX;
  static_assert(NB == 4 || NB == 2 || NB == 1, "32-column blocks per head");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  Bars *bars = reinterpret_cast<Bars *>(base + BAR_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int *abort_flag = &bars->abort;
  __shared__ int skip;
  if (threadIdx.x == 0) skip = *(volatile uint32_t *)&st->code != 0u;
  __syncthreads();
  if (skip) return;
  const int64_t per = (n_items + gridDim.x - 1) / gridDim.x;
  const int64_t x0 = (int64_t)blockIdx.x * per;
  const int64_t x1 = x0 + per < n_items ? x0 + per : n_items;
  if (x0 >= x1) return;  // block-uniform
  // range-check build: the last head's columns lie inside an output row (block-uniform)
  if (!in_range(st, (int64_t)d.H * d.D - 1, out_stride, K_READ_TC, 5)) return;
  const int Hg = d.H * d.D / D;  // head groups of 128 features (one head when D = 128)

  if (threadIdx.x == 0) {
    for (int s = 0; s < NQ; ++s) {
      mbar_init(smem_u32(&bars->q_full[s]), 1);
      mbar_init(smem_u32(&bars->q_empty[s]), 1);
      mbar_init(smem_u32(&bars->gate_done[s]), 1);
      mbar_init(smem_u32(&bars->feat_full[s]), ROLE_WARPS);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&bars->den_full[a]), ROLE_WARPS);
      mbar_init(smem_u32(&bars->acc_full[a]), 1);
      mbar_init(smem_u32(&bars->acc_empty[a]), ROLE_WARPS);
    }
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->s_empty), 1);
    mbar_init(smem_u32(&bars->w_full), 1);
    mbar_init(smem_u32(&bars->w_empty), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
    tma_prefetch(&tmQ);
    tma_prefetch(&tmS);
    if (gate_mma) tma_prefetch(&tmW);
    tma_prefetch(&tmO);
  }
  if (warp == 0) { tmem_alloc(smem_u32(&bars->tmem), TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      // Per item: its Q tile first, then a refill of W_l / S_sum if the head / group
      // changed.  The MMA thread releases a slot at the first item of the next head or
      // group, before it waits for anything of that item, so these waits never wait on a
      // load that comes after them.
      int k = 0, ns = 0, nw = 0, cur_s = -1, cur_w = -1;
      for (int64_t x = x0; x < x1; ++x) {
        ReadItem it;
        if (!read_item(tiles, n_tiles, d, st, x, it)) continue;
        const int s = k % NQ;
        if (!mbar_wait(smem_u32(&bars->q_empty[s]), ((k / NQ) & 1) ^ 1, abort_flag, st, K_READ, 1)) break;
        const uint32_t qb = smem_u32(&bars->q_full[s]);
        mbar_arrive_expect_tx(qb, TILE_BYTES);
        for (int b = 0; b < 2; ++b)
          tma_load_2d(smem_u32(base + Q_OFF + s * TILE_BYTES + b * BM * 128), &tmQ, qb, it.h * D + b * 64, it.row0);
        ++k;
        if (gate_mma && it.h != cur_w) {
          if (!mbar_wait(smem_u32(&bars->w_empty), (nw & 1) ^ 1, abort_flag, st, K_READ, 2)) break;
          const uint32_t wb = smem_u32(&bars->w_full);
          mbar_arrive_expect_tx(wb, TILE_BYTES);
          for (int b = 0; b < 2; ++b) tma_load_2d(smem_u32(base + W_OFF + b * BM * 128), &tmW, wb, b * 64, it.h * D);
          ++nw;
          cur_w = it.h;
        }
        const int key = it.g * Hg + it.h;
        if (key != cur_s) {
          if (!mbar_wait(smem_u32(&bars->s_empty), (ns & 1) ^ 1, abort_flag, st, K_READ, 3)) break;
          const uint32_t sb = smem_u32(&bars->s_full);
          mbar_arrive_expect_tx(sb, TILE_BYTES + (delta ? 0u : D * 4u) + (scalar_gate ? D * 4u : 0u));
          for (int b = 0; b < 2; ++b) tma_load_2d(smem_u32(base + S_OFF + b * BM * 128), &tmS, sb, b * 64, key * D);
          if (!delta) bulk_load(smem_u32(bars->zs), zsum + (int64_t)key * D, D * 4u, sb);
          if (scalar_gate) bulk_load(smem_u32(bars->wg1), wgl + (int64_t)it.h * D, D * 4u, sb);
          ++ns;
          cur_s = key;
        }
      }
      // every copy issued here lands before the block may exit (bounded waits)
      int no_abort = 0;
      for (int s = 0; s < NQ && s < k; ++s) {
        const int fills = (k - s + NQ - 1) / NQ;
        mbar_wait(smem_u32(&bars->q_full[s]), (fills - 1) & 1, &no_abort, st, K_READ, 4);
      }
      if (ns > 0) mbar_wait(smem_u32(&bars->s_full), (ns - 1) & 1, &no_abort, st, K_READ, 4);
      if (nw > 0) mbar_wait(smem_u32(&bars->w_full), (nw - 1) & 1, &no_abort, st, K_READ, 4);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      int k = 0, ns = 0, nw = 0, cur_s = -1, cur_w = -1;
      const uint32_t sb_ = smem_u32(base + S_OFF), wb = smem_u32(base + W_OFF);
      for (int64_t x = x0; x < x1; ++x) {
        ReadItem it;
        if (!read_item(tiles, n_tiles, d, st, x, it)) continue;
        const int s = k % NQ, a = k & 1;
        const int key = it.g * Hg + it.h;
        const bool new_w = gate_mma && it.h != cur_w, new_s = key != cur_s;
        // releases first: every MMA on the previous W_l / S_sum has been issued
        if (new_w && nw > 0) mma_commit(smem_u32(&bars->w_empty));
        if (new_s && ns > 0) mma_commit(smem_u32(&bars->s_empty));
        if (new_w) {
          if (!mbar_wait(smem_u32(&bars->w_full), nw & 1, abort_flag, st, K_READ, 5)) break;
          ++nw;
          cur_w = it.h;
        }
        if (!mbar_wait(smem_u32(&bars->q_full[s]), (k / NQ) & 1, abort_flag, st, K_READ, 6)) break;
        if (!mbar_wait(smem_u32(&bars->acc_empty[a]), ((k >> 1) & 1) ^ 1, abort_flag, st, K_READ, 7)) break;
        tc_fence_after();
        const uint32_t qa = smem_u32(base + Q_OFF + s * TILE_BYTES);
        const uint32_t acc = tmem + (uint32_t)a * 256;
        if (gate_mma) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(acc + 128, sdesc(qa + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024),
                   sdesc(wb + kk * 2048, BM * 128, 1024), IDESC_NUM, kk > 0);
        }
        // Q may be overwritten by the features, and den/g1 of set a reused, once this arrives
        mma_commit(smem_u32(&bars->gate_done[s]));
        if (new_s) {
          if (!mbar_wait(smem_u32(&bars->s_full), ns & 1, abort_flag, st, K_READ, 8)) break;
          ++ns;
          cur_s = key;
        }
        if (!mbar_wait(smem_u32(&bars->feat_full[s]), (k / NQ) & 1, abort_flag, st, K_READ, 9)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(acc, sdesc(qa + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024),
                 sdesc(sb_ + kk * 2048, BM * 128, 1024), IDESC_NUM, kk > 0);
        mma_commit(smem_u32(&bars->acc_full[a]));
        mma_commit(smem_u32(&bars->q_empty[s]));
        ++k;
      }
      // no MMA of this block may be in flight when it exits
      mma_commit(smem_u32(&bars->drain));
      int no_abort = 0;
      mbar_wait(smem_u32(&bars->drain), 0, &no_abort, st, K_READ, 10);
    }
  } else if (warp >= FEAT_WARP0 && warp < FEAT_WARP0 + ROLE_WARPS) {
    // ---------------------------------------------------------------- feature rows
    const int r = (warp & 3) * 32 + lane, hf = (warp - FEAT_WARP0) >> 2, c0 = hf * HC;
    int k = 0, ns = 0, cur_s = -1;
    // amax_q: this warp's max |q| over the items of head qh, flushed (one atomicMax per warp)
    // when the head changes and at the end
    float qmax = 0.f;
    int qh = -1;
    auto flush_qmax = [&]() {
      float m = qmax;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0 && qh >= 0) atomicMax(&amax_q[qh], __float_as_uint(m));
      qmax = 0.f;
    };
    for (int64_t x = x0; x < x1; ++x) {
      ReadItem it;
      if (!read_item(tiles, n_tiles, d, st, x, it)) continue;
      const int s = k % NQ, a = k & 1;
      // z (and the scalar-gate weights) of a new group come with its S_sum; the slot is
      // refilled only after the last item of the previous group has been handed over
      const int key = it.g * Hg + it.h;
      if (key != cur_s && (!delta || scalar_gate)) {
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full), ns & 1, abort_flag, st, K_READ, 15))) break;
        ++ns;
        cur_s = key;
      }
      if (amax && it.h != qh) {  // warp-uniform
        flush_qmax();
        qh = it.h;
      }
      // the warp proceeds (or gives up) as a whole
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->q_full[s]), (k / NQ) & 1, abort_flag, st, K_READ, 11)))
        break;
      uint8_t *qt = base + Q_OFF + s * TILE_BYTES;
      // ELU1: this half of phi(q) and of the normaliser phi(q).z.  Delta rule: no feature
      // rows at all; the MMAs take q itself (q/|q| . S = (q . S) / |q|), and this half's
      // share of |q|^2 goes where the normaliser would, for the epilogue to apply 1/|q|.
      // (Each half reads only its own columns of the tile: the other half's thread may
      // already be writing its features over the rest.)
      uint32_t fr[HC / 2];
      float2 den2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // per 32-column block
      float gate1[2] = {0.f, 0.f};
      const float2 l2e = make_float2(1.4426950408889634f, 1.4426950408889634f);
#pragma unroll
      for (int i = 0; i < HC / 8; ++i) {
        const int cl = c0 / 8 + i, bk = i >> 2;  // 16-byte chunk, and its block in this half
        const uint4 raw = *reinterpret_cast<const uint4 *>(qt + swz_off(r, cl, BM));
        const __nv_bfloat162 *hp = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 xv = __bfloat1622float2(hp[e]);
          if (amax) qmax = fmaxf(qmax, fmaxf(fabsf(xv.x), fabsf(xv.y)));
          // D = 128: one share per half row; otherwise one per 32-column block
          const int ab = NB == 4 ? 0 : bk;
          if (scalar_gate) {
            const float2 wv = *reinterpret_cast<const float2 *>(&bars->wg1[cl * 8 + 2 * e]);
            gate1[ab] = fmaf(xv.x, wv.x, fmaf(xv.y, wv.y, gate1[ab]));
          }
          if (delta) {
            den2[ab] = __ffma2_rn(xv, xv, den2[ab]);
          } else {
            // elu + 1 as max(x, 0) + 2^(min(x, 0) log2 e): no branch
            const float2 e2 = __fmul2_rn(make_float2(fminf(xv.x, 0.f), fminf(xv.y, 0.f)), l2e);
            xv = __fadd2_rn(make_float2(fmaxf(xv.x, 0.f), fmaxf(xv.y, 0.f)), make_float2(ex2f(e2.x), ex2f(e2.y)));
            den2[ab] = __ffma2_rn(xv, *reinterpret_cast<const float2 *>(&bars->zs[cl * 8 + 2 * e]), den2[ab]);
            fr[i * 4 + e] = pack_bf16(xv.x, xv.y);
          }
        }
      }
      // Q is the A operand of the gate MMA: the features go over it only afterwards.
      // gate_done also means the epilogue has released accumulator set a, and with it den[a]
      // and g1[a].
      if (!__all_sync(0xffffffffu,
                      mbar_wait(smem_u32(&bars->gate_done[s]), (k / NQ) & 1, abort_flag, st, K_READ, 12)))
        break;
      if (!delta) {
#pragma unroll
        for (int i = 0; i < HC / 8; ++i)
          *reinterpret_cast<uint4 *>(qt + swz_off(r, c0 / 8 + i, BM)) =
              make_uint4(fr[i * 4], fr[i * 4 + 1], fr[i * 4 + 2], fr[i * 4 + 3]);
      }
      if constexpr (NB == 4) {
        bars->den[a][hf][r] = den2[0].x + den2[0].y;
        bars->g1[a][hf][r] = gate1[0];
      } else {
#pragma unroll
        for (int bk = 0; bk < 2; ++bk) {
          bars->den[a][2 * hf + bk][r] = den2[bk].x + den2[bk].y;
          bars->g1[a][2 * hf + bk][r] = gate1[bk];
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->feat_full[s]));
      if (gate_mma) {
        // the element-wise gate sigmoid(Q W_l) in place over its logits in tensor memory (the
        // gate MMA has completed: gate_done), so the epilogue only multiplies
        const uint32_t ga = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)a * 256 + 128 + (uint32_t)c0;
        tc_fence_after();  // the logits were written by the gate MMA that gate_done saw complete
#pragma unroll
        for (int c = 0; c < HC; c += 32) {
          uint32_t ug[32];
          tmem_ld32(ga + c, ug);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 t = __fmul2_rn(make_float2(__uint_as_float(ug[i]), __uint_as_float(ug[i + 1])),
                                        make_float2(0.5f, 0.5f));
            const float2 g = __ffma2_rn(make_float2(0.5f, 0.5f), make_float2(tanh_fast(t.x), tanh_fast(t.y)),
                                        make_float2(0.5f, 0.5f));
            ug[i] = __float_as_uint(g.x);
            ug[i + 1] = __float_as_uint(g.y);
          }
          tmem_st32(ga + c, ug);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
      }
      if (lane == 0) mbar_arrive(smem_u32(&bars->den_full[a]));
      ++k;
    }
    if (amax) flush_qmax();
  } else if (warp >= EPI_WARP0) {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3, r = quad * 32 + lane, hf = (warp - EPI_WARP0) >> 2, c0 = hf * HC;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint8_t *stage = base + O_OFF;
    const bool out8 = fused && a8_scale != nullptr;  // e4m3 codes of A_l in units of a8_scale[h]
    const int et = threadIdx.x - EPI_WARP0 * 32;     // 0 .. 255
    constexpr int NT = ROLE_WARPS * 32;
    int k = 0, cur_h = -1;
    for (int64_t x = x0; x < x1; ++x) {
      ReadItem it;
      if (!read_item(tiles, n_tiles, d, st, x, it)) continue;
      const int a = k & 1;
      // gamma of a new head: every epilogue thread has passed the previous item's last
      // barrier, so nobody reads the old values any more; the next barrier publishes these
      if (fused && it.h != cur_h) {
        if (et < D) bars->gam[et] = gamma[(int64_t)it.h * D + et];
        cur_h = it.h;
      }
      // the previous item's TMA store has read the staged tile once this returns; the
      // barrier below tells the others
      if (et == 0) bulk_wait_read_all();
      const bool got = mbar_wait(smem_u32(&bars->acc_full[a]), (k >> 1) & 1, abort_flag, st, K_READ, 13) &&
                       mbar_wait(smem_u32(&bars->den_full[a]), (k >> 1) & 1, abort_flag, st, K_READ, 14);
      // the epilogue warps go on (or give up) together: they share the staging buffer, which
      // the previous item's stores have finished reading once all of them are here
      if (!named_bar_and(1, NT, got)) break;
      tc_fence_after();
      // The row's two 32-column chunks (blocks 2hf and 2hf + 1) and the heads they belong
      // to: D = 128, the row's one head over both halves; otherwise the NB blocks of each head.
      auto head_sum = [&](const float (*arr)[BM], int b) {
        const int b0 = (b / NB) * NB;
        float t = 0.f;
#pragma unroll
        for (int j = 0; j < NB; ++j) t += arr[b0 + j][r];
        return t;
      };
      // ELU1: the normaliser phi(q).z; delta rule: |q|^2 (o = (q . S) / |q|)
      float scale[2], gs[2];
      if constexpr (NB == 4) {
        const float den = bars->den[a][0][r] + bars->den[a][1][r];
        scale[0] = scale[1] = delta ? (den > 0.f ? rsqrtf(den) : 0.f) : (den > 0.f ? 1.f / den : 0.f);
        gs[0] = gs[1] = fast_sigmoid(bars->g1[a][0][r] + bars->g1[a][1][r]);
      } else {
#pragma unroll
        for (int bk = 0; bk < 2; ++bk) {
          const float den = head_sum(bars->den[a], 2 * hf + bk);
          scale[bk] = delta ? (den > 0.f ? rsqrtf(den) : 0.f) : (den > 0.f ? 1.f / den : 0.f);
          gs[bk] = fast_sigmoid(head_sum(bars->g1[a], 2 * hf + bk));
        }
      }
      const uint32_t acc = tmem + lane_off + (uint32_t)a * 256 + (uint32_t)c0;
      float rinv[2] = {1.f, 1.f};
      if (fused) {
        uint32_t u0[32], u1[32];
        tmem_ld32(acc, u0);
        tmem_ld32(acc + 32, u1);
        tmem_wait_ld();
        float2 ss2 = make_float2(0.f, 0.f);  // .x: block 2hf, .y: block 2hf + 1
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 ab = make_float2(__uint_as_float(u0[i]), __uint_as_float(u1[i]));
          ss2 = __ffma2_rn(ab, ab, ss2);
        }
        if constexpr (NB == 4) {
          bars->ssq[hf][r] = ss2.x + ss2.y;
          named_bar_sync(1, NT);  // both halves' sums of squares are in
          rinv[0] = rinv[1] = rsqrtf((bars->ssq[0][r] + bars->ssq[1][r]) * (scale[0] * scale[0]) / (float)D + eps);
        } else {
          bars->ssq[2 * hf][r] = ss2.x;
          bars->ssq[2 * hf + 1][r] = ss2.y;
          named_bar_sync(1, NT);  // every block's sum of squares is in
#pragma unroll
          for (int bk = 0; bk < 2; ++bk)
            rinv[bk] = rsqrtf(head_sum(bars->ssq, 2 * hf + bk) * (scale[bk] * scale[bk]) / (float)(32 * NB) + eps);
        }
      }
      // this thread's 64 columns: bf16, box hf, chunks 0-7 of row r; e4m3, chunks 4hf .. 4hf+3
      uint8_t *srow = stage + (out8 ? 0 : hf * (BM * 128)) + r * 128;
#pragma unroll
      for (int c = 0; c < HC; c += 32) {
        const int bk = c >> 5;
        const float f_row = scale[bk] * rinv[bk];  // o / rms(o) = num * scale * rinv
        const float f_out = out8 ? f_row / a8_scale[it.h] : f_row;
        uint32_t u[32], ug[32];
        tmem_ld32(acc + c, u);
        if (gate_mma) tmem_ld32(acc + 128 + c, ug);
        tmem_wait_ld();
#pragma unroll
        for (int v = 0; v < 32; v += 8) {
          float o8[8];
          if (fused) {
            const float2 *gg = reinterpret_cast<const float2 *>(&bars->gam[c0 + c + v]);
            const float2 fo = make_float2(f_out, f_out);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              float2 gl;
              if (gate_mma) {
                gl = make_float2(__uint_as_float(ug[v + e]), __uint_as_float(ug[v + e + 1]));  // sigmoid, in place
              } else {
                gl = make_float2(gs[bk], gs[bk]);
              }
              const float2 o = __fmul2_rn(__fmul2_rn(gl, gg[e >> 1]),
                                          __fmul2_rn(make_float2(__uint_as_float(u[v + e]), __uint_as_float(u[v + e + 1])), fo));
              o8[e] = o.x;
              o8[e + 1] = o.y;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) o8[e] = __uint_as_float(u[v + e]) * f_out;
          }
          if (out8) {
            uint32_t w2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(o8[4 * e], o8[4 * e + 1]), __NV_SATFINITE, __NV_E4M3);
              const uint32_t hi =
                  __nv_cvt_float2_to_fp8x2(make_float2(o8[4 * e + 2], o8[4 * e + 3]), __NV_SATFINITE, __NV_E4M3);
              w2[e] = (lo & 0xffffu) | (hi << 16);
            }
            const int byte = c0 + c + v;  // 8 bytes inside 16-byte chunk byte / 16
            *reinterpret_cast<uint2 *>(srow + ((((byte >> 4) ^ (r & 7))) << 4) + (byte & 15)) =
                make_uint2(w2[0], w2[1]);
          } else {
            *reinterpret_cast<uint4 *>(srow + ((((c + v) >> 3) ^ (r & 7)) << 4)) = pack8(o8);
          }
        }
      }
      // accumulator set a is free once every warp's tensor-memory reads are done
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty[a]));
      fence_proxy_async();    // the staged values, for the TMA store
      named_bar_sync(1, NT);  // the staged rows are complete
      const int nrows = min(BM, it.row_end - it.row0);
      if (nrows == BM) {
        if (et == 0) {
          if (out8) {
            tma_store_2d(&tmO, smem_u32(stage), it.h * D, it.row0);
          } else {
            tma_store_2d(&tmO, smem_u32(stage), it.h * D, it.row0);
            tma_store_2d(&tmO, smem_u32(stage + BM * 128), it.h * D + 64, it.row0);
          }
          bulk_commit_group();
        }
      } else if (out8) {
        // four rows per warp instruction: eight lanes per 128-byte row
        for (int rr = (et >> 5) * 4 + (lane >> 3); rr < nrows; rr += 4 * ROLE_WARPS) {
          const int j = lane & 7;
          const uint4 val = *reinterpret_cast<const uint4 *>(stage + rr * 128 + ((j ^ (rr & 7)) << 4));
          *reinterpret_cast<uint4 *>((uint8_t *)out + (int64_t)(it.row0 + rr) * out_stride + (int64_t)it.h * D +
                                     j * 16) = val;
        }
      } else {
        // two rows per warp instruction: lanes 0-15 one row, 16-31 the next (256 bytes each)
        for (int rr = (et >> 5) * 2 + (lane >> 4); rr < nrows; rr += 2 * ROLE_WARPS) {
          const int j = lane & 15;
          const uint4 val =
              *reinterpret_cast<const uint4 *>(stage + (j >> 3) * (BM * 128) + rr * 128 + (((j & 7) ^ (rr & 7)) << 4));
          *reinterpret_cast<uint4 *>((__nv_bfloat16 *)out + (int64_t)(it.row0 + rr) * out_stride + (int64_t)it.h * D +
                                     j * 8) = val;
        }
      }
      ++k;
    }
    if (et == 0) bulk_wait_all();  // every TMA store of this block has completed
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace

// bf16 with D = 128, or D = 64 or 32 whose heads fill whole 128-feature groups
bool linear_tc_supported(const Dims &d, vdn_dtype dt) {
  return dt == VDN_BF16 && (d.D == 128 || ((d.D == 64 || d.D == 32) && (d.H * d.D) % 128 == 0));
}

cudaError_t launch_state_build_tc(const Dims &d, const void *k, const void *v, const void *kt, const void *vt,
                                  float *S, float *z, float *St, float *zt, char *ws, const WsPlan &p,
                                  cudaStream_t st) {
  using namespace sb;
  const uint64_t HD = (uint64_t)d.H * d.D;
  CUtensorMap mk, mv, mkt, mvt;
  uint64_t strides[1] = {HD * 2};
  uint32_t box[2] = {64, TK};
  uint64_t dims_v[2] = {HD, (uint64_t)d.Nv()};
  uint64_t dims_t[2] = {HD, (uint64_t)(d.L > 0 ? d.L : 1)};
  const void *ktb = d.L > 0 ? kt : k, *vtb = d.L > 0 ? vt : v;
  if (!encode_tmap(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, dims_v, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, dims_v, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&mkt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ktb, dims_t, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&mvt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, vtb, dims_t, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(state_build_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
  if (e != cudaSuccess) return e;
  const int n_items = (d.F + 1) * (int)(HD / D);  // (frames + text) x head groups
  const int grid = n_items < 2 * sm_count() ? n_items : 2 * sm_count();  // persistent: two CTAs per SM
  state_build_tc_kernel<<<(unsigned)grid, THREADS, SMEM, st>>>(mk, mv, mkt, mvt, d, S, z, St, zt,
                                                               (DevStatus *)(ws + p.status));
  return cudaGetLastError();
}

cudaError_t launch_read_stage(const Dims &d, vdn_lin_kind kind, const float *Sf, const float *Sb, const float *zf,
                              const float *zb, const float *wgl, int G_l, char *ws, const WsPlan &p,
                              cudaStream_t st) {
  const int64_t G = host_group_count(d), DD = (int64_t)d.D * d.D;
  const int64_t n_s8 = Sf != nullptr ? G * d.H * DD / 8 : 0;
  const int64_t n_z = (Sf != nullptr && kind == VDN_LIN_ELU1) ? G * d.H * d.D : 0;
  const int64_t n_w8 = (wgl != nullptr && G_l == d.D) ? (int64_t)d.H * DD / 8 : 0;
  const int64_t n = n_s8 + n_z + n_w8;
  if (n == 0) return cudaSuccess;
  if (d.D < 128) {
    // the off-diagonal blocks of the head groups' 128 x 128 operands are zero
    const size_t hd128 = (size_t)d.H * d.D * 128 * 2;
    cudaError_t e = cudaSuccess;
    if (n_s8 > 0) e = cudaMemsetAsync(ws + p.ssum, 0, (size_t)G * hd128, st);
    if (e == cudaSuccess && n_w8 > 0) e = cudaMemsetAsync(ws + p.wl, 0, hd128, st);
    if (e != cudaSuccess) return e;
  }
  read_stage_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
      n_s8, n_z, n_w8, d.H, d.D, Sf, Sb, zf, zb, wgl, (__nv_bfloat16 *)(ws + p.ssum), (float *)(ws + p.zsum),
      (__nv_bfloat16 *)(ws + p.wl));
  return cudaGetLastError();
}

cudaError_t launch_read_tc(const Dims &d, vdn_lin_kind kind, const void *q, void *out, const float *wgl, int G_l,
                           const float *gamma, float eps, char *ws, const WsPlan &p, cudaStream_t st,
                           const float *a8_scale, uint32_t *amax_q) {
  using namespace rd;
  const uint64_t HD = (uint64_t)d.H * d.D;
  const int G = host_group_count(d);
  const bool fused = wgl != nullptr;
  const bool gate_mma = fused && G_l == D;
  if (a8_scale != nullptr && !fused) return cudaErrorInvalidValue;
  CUtensorMap mq, ms, mw;
  {
    uint64_t dims[2] = {HD, (uint64_t)d.Nv()}, strides[1] = {HD * 2};
    uint32_t box[2] = {64, BM};
    if (!encode_tmap(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    // block-diagonal S_sum [G][head groups][128][128] and W_l [head groups][128][128]
    uint64_t dims[2] = {(uint64_t)D, (uint64_t)G * HD}, strides[1] = {(uint64_t)D * 2};
    uint32_t box[2] = {64, (uint32_t)D};
    if (!encode_tmap(&ms, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.ssum, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    uint64_t dimsw[2] = {(uint64_t)D, HD};
    if (!encode_tmap(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + p.wl, dimsw, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const int64_t stride = fused ? 2 * (int64_t)HD : (int64_t)HD;
  // fused: the linear half of A (bf16, or e4m3 codes with a8_scale)
  void *o = (a8_scale != nullptr) ? (void *)((uint8_t *)out + HD) : (void *)((__nv_bfloat16 *)out + (fused ? HD : 0));
  CUtensorMap mo;  // the output rows' H*D columns (the linear half of A when fused)
  {
    uint64_t dims[2] = {HD, (uint64_t)d.Nv()};
    uint64_t strides[1] = {(uint64_t)stride * (a8_scale != nullptr ? 1 : 2)};
    uint32_t box[2] = {a8_scale != nullptr ? 128u : 64u, (uint32_t)BM};
    if (!encode_tmap(&mo, a8_scale != nullptr ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, o,
                     dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const int n_tiles = host_tile_count(d);
  const int64_t n_items = (int64_t)2 * n_tiles * (int64_t)(HD / D);  // tile halves x head groups
  const int grid = (int)(n_items < sm_count() ? n_items : sm_count());  // persistent: one CTA per SM
  const float *zs = (const float *)(ws + p.zsum);
  const int32_t *tl = (const int32_t *)(ws + p.tiles);
  DevStatus *sp = (DevStatus *)(ws + p.status);
  const bool delta = kind == VDN_LIN_DELTA;
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e != cudaSuccess) return e;
    kern<<<grid, THREADS, SMEM, st>>>(mq, ms, mw, mo, d, zs, fused ? wgl : nullptr, G_l, gamma, eps, o, stride, tl,
                                      n_tiles, n_items, a8_scale, amax_q, sp);
    return cudaGetLastError();
  };
  if (d.D < 128) {
    // heads of D = 64 or 32 in 128-feature head groups: the plain read (the layer applies the
    // gates and RMSNorm in its own pass at these sizes)
    if (fused || amax_q != nullptr) return cudaErrorInvalidValue;
    if (d.D == 64) return delta ? go(read_tc_kernel<true, false, false, false, 2>) : go(read_tc_kernel<false, false, false, false, 2>);
    return delta ? go(read_tc_kernel<true, false, false, false, 1>) : go(read_tc_kernel<false, false, false, false, 1>);
  }
  if (amax_q != nullptr) {  // the max |q| by-product: the delta rule's gated layer only
    if (!(delta && gate_mma)) return cudaErrorInvalidValue;
    return go(read_tc_kernel<true, true, true, true, 4>);
  }
  if (delta) {
    if (!fused) return go(read_tc_kernel<true, false, false, false, 4>);
    return gate_mma ? go(read_tc_kernel<true, true, true, false, 4>) : go(read_tc_kernel<true, true, false, false, 4>);
  }
  if (!fused) return go(read_tc_kernel<false, false, false, false, 4>);
  return gate_mma ? go(read_tc_kernel<false, true, true, false, 4>) : go(read_tc_kernel<false, true, false, false, 4>);
}

}  // namespace vdn
