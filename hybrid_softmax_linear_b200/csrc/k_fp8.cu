// Per-head FP8 (e4m3) quantisation of Q, K and V for the softmax branch (model card
// "Video DeltaNet: ...", "Inference with Diffusers": fp8 e4m3 inference).
//
// Scale per head and tensor: s = amax / 448, with amax over the video rows and, for K
// and V, the text rows too (text shares the video scale).  Values are stored as
// round-to-nearest-even, saturating e4m3 of x / s; the softmax kernel multiplies the
// scales back in.  Two passes: an amax reduction (per-block maxima in shared memory,
// then one atomicMax per head and block on the float bit pattern, which orders like
// the value for non-negative floats) and the cast.  Where the layer's linear branch
// reads every value of Q, K and V anyway (the delta rule's frame statistics, text init
// and read), those kernels leave the per-head maxima behind and only the cast runs here
// (launch_fp8_cast): one pass over the bf16 inputs.
#include "vdn_internal.cuh"

namespace vdn {
namespace {

constexpr float E4M3_MAX = 448.f;

// Tensor t of the three (0 q, 1 k, 2 v); row r of the concatenation [video | text]
// (q has no text rows).
struct Src {
  const __nv_bfloat16 *video[3];
  const __nv_bfloat16 *text[3];
  uint8_t *video8[3];
  uint8_t *text8[3];
};

__device__ __forceinline__ int64_t rows_of(int t, const Dims &d) { return d.Nv() + (t == 0 ? 0 : d.L); }

// Each thread owns up to SLOTS fixed 8-value column chunks (chunk threadIdx.x + 256 j) and
// keeps their running max in registers while the block strides over rows (coalesced
// 16-byte loads); at the end one shared-memory atomicMax per slot, then one global
// atomicMax per head.  grid.y = tensor.  Needs H*D <= 256 * 8 * SLOTS.
constexpr int AMAX_SLOTS = 8;

__global__ void __launch_bounds__(256) fp8_amax_kernel(Dims d, Src s, uint32_t *__restrict__ amax_bits) {
  extern __shared__ uint32_t sm_max[];  // [H]
  const int t = blockIdx.y;
  const int HD = d.H * d.D, n8 = HD / 8;
  for (int h = threadIdx.x; h < d.H; h += blockDim.x) sm_max[h] = 0u;
  __syncthreads();
  float m[AMAX_SLOTS];
#pragma unroll
  for (int j = 0; j < AMAX_SLOTS; ++j) m[j] = 0.f;
  const int64_t rows = rows_of(t, d);
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const __nv_bfloat16 *row = r < d.Nv() ? s.video[t] + r * HD : s.text[t] + (r - d.Nv()) * HD;
#pragma unroll
    for (int j = 0; j < AMAX_SLOTS; ++j) {
      const int c = threadIdx.x + 256 * j;
      if (c < n8) {
        const uint4 u = *reinterpret_cast<const uint4 *>(row + 8 * c);
        const __nv_bfloat162 *hp = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(hp[i]);
          m[j] = fmaxf(m[j], fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < AMAX_SLOTS; ++j) {
    const int c = threadIdx.x + 256 * j;
    if (c < n8) atomicMax(&sm_max[(8 * c) / d.D], __float_as_uint(m[j]));
  }
  __syncthreads();
  for (int h = threadIdx.x; h < d.H; h += blockDim.x) atomicMax(&amax_bits[t * d.H + h], sm_max[h]);
}

__global__ void __launch_bounds__(256) fp8_scale_kernel(int n, const uint32_t *__restrict__ amax_bits,
                                                       float *__restrict__ scales) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float a = __uint_as_float(amax_bits[i]);
    scales[i] = a > 0.f ? a / E4M3_MAX : 1.f;
  }
}

__global__ void __launch_bounds__(256) fp8_cast_kernel(Dims d, Src s, const float *__restrict__ scales) {
  const int t = blockIdx.y;
  const int HD = d.H * d.D, n8 = HD / 8;
  const int64_t rows = rows_of(t, d);
  const int64_t total = rows * n8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / n8;
    const int c = (int)(i % n8);
    const bool vid = r < d.Nv();
    const __nv_bfloat16 *src = vid ? s.video[t] + r * HD : s.text[t] + (r - d.Nv()) * HD;
    uint8_t *dst = vid ? s.video8[t] + r * HD : s.text8[t] + (r - d.Nv()) * HD;
    const float inv = 1.f / scales[t * d.H + (8 * c) / d.D];
    const uint4 u = *reinterpret_cast<const uint4 *>(src + 8 * c);
    const __nv_bfloat162 *hp = reinterpret_cast<const __nv_bfloat162 *>(&u);
    uint32_t w[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float2 a = __bfloat1622float2(hp[2 * j]), b = __bfloat1622float2(hp[2 * j + 1]);
      const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a.x * inv, a.y * inv), __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(b.x * inv, b.y * inv), __NV_SATFINITE, __NV_E4M3);
      w[j] = (lo & 0xffffu) | (hi << 16);
    }
    *reinterpret_cast<uint2 *>(dst + 8 * c) = make_uint2(w[0], w[1]);
  }
}

}  // namespace

cudaError_t launch_fp8_quant(const Dims &d, const void *q, const void *k, const void *v, const void *kt,
                             const void *vt, void *q8, void *k8, void *v8, void *kt8, void *vt8, float *scales,
                             uint32_t *amax_bits, cudaStream_t st) {
  Src s;
  s.video[0] = (const __nv_bfloat16 *)q; s.video[1] = (const __nv_bfloat16 *)k; s.video[2] = (const __nv_bfloat16 *)v;
  s.text[0] = nullptr; s.text[1] = (const __nv_bfloat16 *)kt; s.text[2] = (const __nv_bfloat16 *)vt;
  s.video8[0] = (uint8_t *)q8; s.video8[1] = (uint8_t *)k8; s.video8[2] = (uint8_t *)v8;
  s.text8[0] = nullptr; s.text8[1] = (uint8_t *)kt8; s.text8[2] = (uint8_t *)vt8;
  cudaError_t e = cudaMemsetAsync(amax_bits, 0, 3 * d.H * sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  fp8_amax_kernel<<<dim3(2048, 3), 256, d.H * sizeof(uint32_t), st>>>(d, s, amax_bits);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fp8_scale_kernel<<<(3 * d.H + 255) / 256, 256, 0, st>>>(3 * d.H, amax_bits, scales);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fp8_cast_kernel<<<dim3(4096, 3), 256, 0, st>>>(d, s, scales);
  return cudaGetLastError();
}

cudaError_t launch_fp8_cast(const Dims &d, const void *q, const void *k, const void *v, const void *kt,
                            const void *vt, void *q8, void *k8, void *v8, void *kt8, void *vt8, float *scales,
                            const uint32_t *amax_bits, cudaStream_t st) {
  Src s;
  s.video[0] = (const __nv_bfloat16 *)q; s.video[1] = (const __nv_bfloat16 *)k; s.video[2] = (const __nv_bfloat16 *)v;
  s.text[0] = nullptr; s.text[1] = (const __nv_bfloat16 *)kt; s.text[2] = (const __nv_bfloat16 *)vt;
  s.video8[0] = (uint8_t *)q8; s.video8[1] = (uint8_t *)k8; s.video8[2] = (uint8_t *)v8;
  s.text8[0] = nullptr; s.text8[1] = (uint8_t *)kt8; s.text8[2] = (uint8_t *)vt8;
  fp8_scale_kernel<<<(3 * d.H + 255) / 256, 256, 0, st>>>(3 * d.H, amax_bits, scales);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fp8_cast_kernel<<<dim3(4096, 3), 256, 0, st>>>(d, s, scales);
  return cudaGetLastError();
}

}  // namespace vdn
