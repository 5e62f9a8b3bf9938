// Output projections on the 5th-generation tensor cores:
//   y[M][N] = A[M][2N'] Wcat^T,  Wcat = [W_os | W_ol]  (N = N' = H*D)
// ("VDN-MiniMax-H3 开源" article, 独立门控，融合两条注意力分支: separate output
// projections of the two branches, summed).  One GEMM with K = 2*H*D: the K loop reads
// W_os for the first H*D columns of A and W_ol for the rest.
//
// Persistent, warp-specialised: warp 0 issues TMA loads of 128-row A and 256-row W tiles
// of 128 bytes per row (64 bf16 or 128 e4m3; 128-byte swizzle) into a 4-stage ring; one
// thread of warp 1 issues tcgen05.mma (M=128, N=256, K=16 bf16 or K=32 e4m3) into one of
// two 128x256 fp32 accumulators in tensor memory; warps 2-5 drain the other accumulator
// (tcgen05.ld), round to bf16 and store y, so the epilogue of tile i overlaps the main
// loop of tile i+1.  Tiles are visited in groups of 16 row blocks so that concurrently
// running CTAs share A rows and W columns in L2.
//
// e4m3 form (the model card's "Inference with Diffusers" runs every wide Linear in fp8
// e4m3): A holds e4m3 codes whose dequantisation scale depends only on the column's
// branch and head; w8_prep folds those scales into a copy of [W_os | W_ol], which it
// quantises with one scale per output column n (its amax / 448), so that one fp32
// accumulator sums both halves and the epilogue multiplies column n by that scale.
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

constexpr int BM = 128, BN = 256, BKB = 128, STAGES = 4, GROUP_M = 16;  // BKB: bytes of a K tile row
constexpr int A_BYTES = BM * BKB, B_BYTES = BN * BKB, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;

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

// FP8 = false: bf16 A and W, the K loop switching from W_os (tmW1) to W_ol (tmW2) at HD.
// FP8 = true: e4m3 A and the prepared e4m3 [W_os | W_ol] copy (tmW1 only); column scales
// wsc[N] applied in the epilogue.
template <bool FP8>
__global__ void __launch_bounds__(THREADS, 1)
    out_proj_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW1,
                       const __grid_constant__ CUtensorMap tmW2, void *__restrict__ y, int M, int N,
                       int KH, const float *__restrict__ wsc, int y_f32, DevStatus *st) {
  constexpr int EB = FP8 ? 1 : 2;          // bytes per element
  constexpr int BK = BKB / EB;             // K elements per stage
  constexpr int KSTEP = 32 / EB;           // K elements per MMA (32 bytes of a row)
  constexpr uint32_t IDESC = FP8 ? idesc_e4m3(BM, BN, false, false) : idesc_bf16(BM, BN, false, false);
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
  const int ktiles = 2 * KH / BK;  // K = 2 * KH elements

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
        if (FP8 || kx < KH) tma_load_2d(smem_u32(sb + s * B_BYTES), &tmW1, fb, kx, n * BN);
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
        for (int k = 0; k < BK / KSTEP; ++k) {
          if (FP8)
            mma_ss_f8(d, sdesc(a0 + k * 32, 16, 1024), sdesc(b0 + k * 32, 16, 1024), IDESC, (kt | k) != 0);
          else
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
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * BN + c0), r);
        tmem_wait_ld();
        if (row < M && n * BN + c0 < N) {
          float f[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(r[i]);
          if (FP8) {
            const float4 *sc = reinterpret_cast<const float4 *>(wsc + n * BN + c0);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 c = __ldg(sc + i);
              f[4 * i] *= c.x; f[4 * i + 1] *= c.y; f[4 * i + 2] *= c.z; f[4 * i + 3] *= c.w;
            }
          }
          const int64_t o = (int64_t)row * N + n * BN + c0;
          if (y_f32) {
            // float partial sums (the head-sharded layer reduces them across ranks)
            float4 *dst = reinterpret_cast<float4 *>((float *)y + o);
#pragma unroll
            for (int v = 0; v < 8; ++v) dst[v] = make_float4(f[4 * v], f[4 * v + 1], f[4 * v + 2], f[4 * v + 3]);
          } else {
            uint4 *dst = reinterpret_cast<uint4 *>((__nv_bfloat16 *)y + o);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w4;
              w4.x = pack_bf16(f[8 * v + 0], f[8 * v + 1]);
              w4.y = pack_bf16(f[8 * v + 2], f[8 * v + 3]);
              w4.z = pack_bf16(f[8 * v + 4], f[8 * v + 5]);
              w4.w = pack_bf16(f[8 * v + 6], f[8 * v + 7]);
              dst[v] = w4;
            }
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


// w8[n][c] = e4m3(w'[n][c] / wsc[n]) with w'[n][c] = [W_os | W_ol][n][c] * ascale[c / D] (the
// dequantisation scale of A's column c: its branch half and head) and wsc[n] =
// max_c |w'[n][c]| / 448 (1 for an all-zero row).  One block per output row.
__global__ void __launch_bounds__(256) w8_prep_kernel(const __nv_bfloat16 *__restrict__ wos,
                                                      const __nv_bfloat16 *__restrict__ wol, int HD, int D,
                                                      const float *__restrict__ ascale, uint8_t *__restrict__ w8,
                                                      float *__restrict__ wsc) {
  __shared__ float red[8];
  const int n = blockIdx.x, tid = threadIdx.x;
  const int K = 2 * HD;
  float mx = 0.f;
  // pass 1: amax of the scaled row (8 elements per step: 16-byte loads of each half)
  for (int c = tid * 8; c < K; c += 256 * 8) {
    const __nv_bfloat16 *src = c < HD ? wos + (int64_t)n * HD + c : wol + (int64_t)n * HD + (c - HD);
    const float sc = ascale[c / D];
    const uint4 raw = *reinterpret_cast<const uint4 *>(src);
    const __nv_bfloat162 *hp = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(hp[e]);
      mx = fmaxf(mx, fmaxf(fabsf(f.x * sc), fabsf(f.y * sc)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) mx = fmaxf(mx, red[i]);
  const float scale = mx > 0.f ? mx / 448.f : 1.f;
  const float inv = 1.f / scale;
  if (tid == 0) wsc[n] = scale;
  // pass 2: the codes (the row is in L1/L2 from pass 1)
  for (int c = tid * 8; c < K; c += 256 * 8) {
    const __nv_bfloat16 *src = c < HD ? wos + (int64_t)n * HD + c : wol + (int64_t)n * HD + (c - HD);
    const float sc = ascale[c / D] * inv;
    const uint4 raw = *reinterpret_cast<const uint4 *>(src);
    const __nv_bfloat162 *hp = reinterpret_cast<const __nv_bfloat162 *>(&raw);
    uint32_t q[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 f0 = __bfloat1622float2(hp[2 * e]), f1 = __bfloat1622float2(hp[2 * e + 1]);
      const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(f0.x * sc, f0.y * sc), __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(f1.x * sc, f1.y * sc), __NV_SATFINITE, __NV_E4M3);
      q[e] = (lo & 0xffffu) | (hi << 16);
    }
    *reinterpret_cast<uint2 *>(w8 + (int64_t)n * K + c) = make_uint2(q[0], q[1]);
  }
}

// Per-(branch half, head) dequantisation scales of A in the e4m3 layer, from static bounds:
// A_s = g_s O_s is a gated convex combination of V rows, so |A_s| <= amax(V_h), the e4m3
// V scale's 448 (its scale is then that of V); A_l = g_l gamma O_l / rms(O_l) has
// |A_l| <= max|gamma_h| sqrt(D), so its scale is that / 448.
// halves: bit 0 the A_s scales (the V scales), bit 1 the A_l scales (from gamma alone)
__global__ void a8_scale_kernel(int H, int D, const float *__restrict__ vscale, const float *__restrict__ gamma,
                                float *__restrict__ ascale, int halves) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  if (halves & 1) ascale[h] = vscale[h];
  if (halves & 2) {
    float g = 0.f;
    for (int i = 0; i < D; ++i) g = fmaxf(g, fabsf(gamma[(int64_t)h * D + i]));
    const float b = g * sqrtf((float)D) / 448.f;
    ascale[H + h] = b > 0.f ? b : 1.f;
  }
}

}  // namespace

bool out_proj_tc_supported(const Dims &d) {
  const int HD = d.H * d.D;
  return HD % 64 == 0 && HD % 8 == 0 && HD >= 64;
}

cudaError_t launch_out_proj_tc(const Dims &d, const void *a, const void *wos, const void *wol, void *y, char *ws,
                               const WsPlan &p, cudaStream_t st, int n_out, bool y_f32) {
  const int HD = d.H * d.D;                 // K of each projection (this call's heads)
  const int N = n_out > 0 ? n_out : HD;     // output features
  const int64_t M = d.Nv();
  CUtensorMap tmA, tmW1, tmW2;
  {
    uint64_t dims[2] = {(uint64_t)(2 * HD), (uint64_t)M}, strides[1] = {(uint64_t)(2 * HD) * 2};
    uint32_t box[2] = {BKB / 2, BM};
    if (!encode_tmap(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[2] = {(uint64_t)HD, (uint64_t)N}, strides[1] = {(uint64_t)HD * 2};
    uint32_t box[2] = {BKB / 2, BN};
    if (!encode_tmap(&tmW1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wos, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap(&tmW2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wol, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(out_proj_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int tiles = (int)((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = tiles < sm_count() ? tiles : sm_count();
  out_proj_tc_kernel<false><<<grid, THREADS, SMEM_BYTES, st>>>(tmA, tmW1, tmW2, y, (int)M, N, HD, nullptr,
                                                               y_f32 ? 1 : 0, (DevStatus *)(ws + p.status));
  return cudaGetLastError();
}

bool out_proj_e4m3_supported(const Dims &d) {
  const int HD = d.H * d.D;
  return HD % 256 == 0 && HD >= 256;
}

cudaError_t launch_a8_scales(const Dims &d, const float *vscale, const float *gamma, float *ascale, cudaStream_t st,
                             int halves) {
  a8_scale_kernel<<<(d.H + 127) / 128, 128, 0, st>>>(d.H, d.D, vscale, gamma, ascale, halves);
  return cudaGetLastError();
}

cudaError_t launch_out_proj_e4m3(const Dims &d, const void *a8, const float *ascale, const void *wos, const void *wol,
                                 void *y, uint8_t *w8, float *wsc, DevStatus *status, cudaStream_t st) {
  const int HD = d.H * d.D;
  const int64_t M = d.Nv();
  w8_prep_kernel<<<HD, 256, 0, st>>>((const __nv_bfloat16 *)wos, (const __nv_bfloat16 *)wol, HD, d.D, ascale, w8, wsc);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tmA, tmW;
  {
    uint64_t dims[2] = {(uint64_t)(2 * HD), (uint64_t)M}, strides[1] = {(uint64_t)(2 * HD)};
    uint32_t box[2] = {BKB, BM};
    if (!encode_tmap(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a8, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[2] = {(uint64_t)(2 * HD), (uint64_t)HD}, strides[1] = {(uint64_t)(2 * HD)};
    uint32_t box[2] = {BKB, BN};
    if (!encode_tmap(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w8, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  e = cudaFuncSetAttribute(out_proj_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int tiles = (int)((M + BM - 1) / BM) * ((HD + BN - 1) / BN);
  const int grid = tiles < sm_count() ? tiles : sm_count();
  out_proj_tc_kernel<true><<<grid, THREADS, SMEM_BYTES, st>>>(tmA, tmW, tmW, y, (int)M, HD, HD, wsc, 0, status);
  return cudaGetLastError();
}

}  // namespace vdn
