// Output projections on the 5th-generation tensor cores:
//   y[M][N] = A[M][2N'] Wcat^T,  Wcat = [W_os | W_ol]  (N = N' = H*D)
// ("VDN-MiniMax-H3 开源" article, 独立门控，融合两条注意力分支: separate output
// projections of the two branches, summed).  One GEMM with K = 2*H*D: the K loop reads
// W_os for the first H*D columns of A and W_ol for the rest.
//
// Persistent, warp-specialised: warp 0 issues TMA loads of 128x64 A and 256x64 W tiles
// (128-byte swizzle) into a 4-stage ring; one thread of warp 1 issues tcgen05.mma
// (M=128, N=256, K=16) into one of two 128x256 fp32 accumulators in tensor memory;
// warps 2-5 drain the other accumulator (tcgen05.ld), round to bf16 and store y, so the
// epilogue of tile i overlaps the main loop of tile i+1.  Tiles are visited in groups of
// 16 row blocks so that concurrently running CTAs share A rows and W columns in L2.
#include <mutex>

#include "tc_common.cuh"

namespace vdn {
namespace tc {

bool encode_tmap(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *base, const uint64_t *dims,
                 const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swz) {
  static PFN_cuTensorMapEncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled)p;
  });
  if (fn == nullptr) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) { gd[i] = dims[i]; bx[i] = box[i]; }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void *>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  static int n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (n[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    n[dev] = v;
  }
  return n[dev];
}

}  // namespace tc

namespace {

using namespace tc;

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4, GROUP_M = 16;
constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_bf16(BM, BN, false, false);

struct alignas(8) Bars {
  uint64_t full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + sizeof(Bars);

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int &m, int &n) {
  const int per_group = GROUP_M * num_n;
  const int g = t / per_group, idx = t % per_group;
  const int gm = min(GROUP_M, num_m - g * GROUP_M);
  m = g * GROUP_M + idx % gm;
  n = idx / gm;
}

__global__ void __launch_bounds__(THREADS, 1)
    out_proj_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW1,
                       const __grid_constant__ CUtensorMap tmW2, __nv_bfloat16 *__restrict__ y, int M, int N,
                       int KH, DevStatus *st) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t *base = smem_raw + ((1024 - (raw & 1023)) & 1023);
  uint8_t *sa = base;                                // STAGES x A tile
  uint8_t *sb = base + STAGES * A_BYTES;             // STAGES x B tile
  Bars *bars = reinterpret_cast<Bars *>(base + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int *abort_flag = &bars->abort;
  __shared__ int skip;  // an earlier block gave up: do no more work (block-uniform decision)
  if (threadIdx.x == 0) skip = *(volatile uint32_t *)&st->code != 0u;
  __syncthreads();
  if (skip) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(smem_u32(&bars->full[s]), 1); mbar_init(smem_u32(&bars->empty[s]), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(smem_u32(&bars->tfull[b]), 1); mbar_init(smem_u32(&bars->tempty[b]), 4); }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
    tma_prefetch(&tmA); tma_prefetch(&tmW1); tma_prefetch(&tmW2);
  }
  if (warp == 1) { tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN, tiles = num_m * num_n;
  const int ktiles = 2 * KH / BK;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    int s = 0;
    uint32_t ph = 0;
    uint32_t armed = 0, armed_ph = 0;  // per stage: armed at least once, parity of the last arming
    for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
      int m, n;
      tile_coords(t, num_m, num_n, m, n);
      for (int kt = 0; kt < ktiles; ++kt) {
        if (!mbar_wait(smem_u32(&bars->empty[s]), ph ^ 1, abort_flag, st, K_GEMM_TC, 1)) break;
        const uint32_t fb = smem_u32(&bars->full[s]);
        mbar_arrive_expect_tx(fb, STAGE_BYTES);
        const int kx = kt * BK;
        tma_load_2d(smem_u32(sa + s * A_BYTES), &tmA, fb, kx, m * BM);
        if (kx < KH) tma_load_2d(smem_u32(sb + s * B_BYTES), &tmW1, fb, kx, n * BN);
        else tma_load_2d(smem_u32(sb + s * B_BYTES), &tmW2, fb, kx - KH, n * BN);
        armed |= 1u << s;
        armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
    }
    // every load issued here has landed before the block leaves (bounded waits)
    int no_abort = 0;
    for (int i = 0; i < STAGES; ++i)
      if (armed & (1u << i)) mbar_wait(smem_u32(&bars->full[i]), (armed_ph >> i) & 1u, &no_abort, st, K_GEMM_TC, 6);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int s = 0, b = 0;
    uint32_t ph = 0, tph = 0;
    for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
      if (!mbar_wait(smem_u32(&bars->tempty[b]), tph ^ 1, abort_flag, st, K_GEMM_TC, 2)) break;
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(b * BN);
      bool ok = true;
      for (int kt = 0; kt < ktiles; ++kt) {
        if (!mbar_wait(smem_u32(&bars->full[s]), ph, abort_flag, st, K_GEMM_TC, 3)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sa + s * A_BYTES), b0 = smem_u32(sb + s * B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          mma_ss(d, sdesc(a0 + k * 32, 16, 1024), sdesc(b0 + k * 32, 16, 1024), IDESC, (kt | k) != 0);
        }
        mma_commit(smem_u32(&bars->empty[s]));
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) break;
      mma_commit(smem_u32(&bars->tfull[b]));
      if (++b == 2) { b = 0; tph ^= 1; }
    }
    // all MMAs issued by this thread complete before the block leaves (bounded wait)
    mma_commit(smem_u32(&bars->drain));
    int no_abort = 0;
    mbar_wait(smem_u32(&bars->drain), 0, &no_abort, st, K_GEMM_TC, 4);
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> registers -> bf16 -> global
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    int b = 0;
    uint32_t tph = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      int m, n;
      tile_coords(t, num_m, num_n, m, n);
      // the warp proceeds (or gives up) as a whole: tensor-memory loads are warp-collective
      const bool got = mbar_wait(smem_u32(&bars->tfull[b]), tph, abort_flag, st, K_GEMM_TC, 5);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int row = m * BM + q * 32 + lane;
      __nv_bfloat16 *yr = y + (int64_t)row * N + n * BN;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * BN + c0), r);
        tmem_wait_ld();
        if (row < M && n * BN + c0 < N) {
          uint4 *dst = reinterpret_cast<uint4 *>(yr + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 o;
            o.x = pack_bf16(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
            o.y = pack_bf16(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
            o.z = pack_bf16(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
            o.w = pack_bf16(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
            dst[v] = o;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->tempty[b]));
      if (++b == 2) { b = 0; tph ^= 1; }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace

bool out_proj_tc_supported(const Dims &d) {
  const int HD = d.H * d.D;
  return HD % BK == 0 && HD % 8 == 0 && HD >= BK;
}

cudaError_t launch_out_proj_tc(const Dims &d, const void *a, const void *wos, const void *wol, void *y, char *ws,
                               const WsPlan &p, cudaStream_t st) {
  const int HD = d.H * d.D;
  const int64_t M = d.Nv();
  CUtensorMap tmA, tmW1, tmW2;
  {
    uint64_t dims[2] = {(uint64_t)(2 * HD), (uint64_t)M}, strides[1] = {(uint64_t)(2 * HD) * 2};
    uint32_t box[2] = {BK, BM};
    if (!encode_tmap(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[2] = {(uint64_t)HD, (uint64_t)HD}, strides[1] = {(uint64_t)HD * 2};
    uint32_t box[2] = {BK, BN};
    if (!encode_tmap(&tmW1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wos, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap(&tmW2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wol, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(out_proj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int tiles = (int)((M + BM - 1) / BM) * ((HD + BN - 1) / BN);
  const int grid = tiles < sm_count() ? tiles : sm_count();
  out_proj_tc_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tmA, tmW1, tmW2, (__nv_bfloat16 *)y, (int)M, HD, HD,
                                                        (DevStatus *)(ws + p.status));
  return cudaGetLastError();
}

}  // namespace vdn
