// vdn_softmax_branch_fwd_noalloc: the softmax branch for callers that cannot allocate
// device memory.  Such callers include plug-ins that only ever see tensors handed to
// them by a host framework that owns all device memory and offers no scratch hook,
// and code that must not allocate once it is running.  These callers cannot size and
// pass a workspace.  This entry point keeps the branch's small scratch (status word,
// layout tables, query-tile list) in a fixed array in the library's own device memory
// instead.
//
// The array is a file-scope __device__ array: each GPU that loads the library holds
// it until the process exits.  Host code cannot use the array's name as a device
// address, so the address is looked up once per device with cudaGetSymbolAddress
// (on the first call made on that device) and passed to the kernels.
#include <cstdio>
#include <mutex>

#include "vdn_internal.cuh"

namespace vdn {
void set_last_error(const char *msg);  // vdn_api.cu

namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = 256u * 1024u;  // 256 KiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
void *g_scratch_ptr[MAX_DEVICES] = {nullptr};

// messages go to the library's vdn_last_error()
vdn_status noalloc_fail(vdn_status code, const char *msg, cudaError_t e = cudaSuccess) {
  char buf[384];
  if (e != cudaSuccess)
    snprintf(buf, sizeof(buf), "%s: %s", msg, cudaGetErrorString(e));
  else
    snprintf(buf, sizeof(buf), "%s", msg);
  set_last_error(buf);
  return code;
}

// Device address of the scratch array on the current device (looked up once per device).
vdn_status scratch_address(char **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(VDN_ERR_CUDA, "cudaGetDevice", e);
  if (dev < 0 || dev >= MAX_DEVICES) return noalloc_fail(VDN_ERR_UNSUPPORTED, "device index out of range");
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return noalloc_fail(VDN_ERR_CUDA, "cudaGetSymbolAddress of the static scratch array", e);
    g_scratch_ptr[dev] = p;
  }
  *out = (char *)g_scratch_ptr[dev];
  return VDN_OK;
}

}  // namespace
}  // namespace vdn

using namespace vdn;

extern "C" VDN_API vdn_status vdn_softmax_branch_fwd_noalloc(const vdn_shape *shape, vdn_dtype dtype, const void *q,
                                                             const void *k, const void *v, const void *kt,
                                                             const void *vt, float sm_scale, void *o_s, float *lse,
                                                             vdn_stream stream) {
  set_last_error("");
  if (shape == nullptr) return noalloc_fail(VDN_ERR_INVALID_ARG, "shape is NULL");
  const vdn_shape &s = *shape;
  if (s.frames < 1 || s.tokens_per_frame < 1 || s.chunk_frames < 1 || s.text_tokens < 0 || s.heads < 1)
    return noalloc_fail(VDN_ERR_INVALID_ARG, "shape out of range");
  if (s.head_dim != 32 && s.head_dim != 64 && s.head_dim != 128)
    return noalloc_fail(VDN_ERR_UNSUPPORTED, "head_dim not in {32, 64, 128}");
  if ((int64_t)s.frames * s.tokens_per_frame + s.text_tokens >= ((int64_t)1 << 31))
    return noalloc_fail(VDN_ERR_INVALID_ARG, "shape too large");
  if (dtype != VDN_F32 && dtype != VDN_BF16)
    return noalloc_fail(VDN_ERR_UNSUPPORTED, "dtype must be VDN_F32 or VDN_BF16");
  auto bad = [](const void *p) { return p == nullptr || ((uintptr_t)p & 15u) != 0; };
  if (bad(q) || bad(k) || bad(v) || bad(o_s) || (s.text_tokens > 0 && (bad(kt) || bad(vt))))
    return noalloc_fail(VDN_ERR_INVALID_ARG, "a tensor pointer is NULL or not 16-byte aligned");
  const WsPlan p = plan_workspace(s, VDN_LIN_ELU1, VDN_BF16);
  if (p.step_end > NOALLOC_SCRATCH_BYTES)
    return noalloc_fail(VDN_ERR_WORKSPACE,
                        "shape needs more scratch than the fixed 256 KiB array (tables and query-tile list); "
                        "use vdn_softmax_branch_fwd with a workspace");
  int dev = 0, major = 0, minor = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (e != cudaSuccess) return noalloc_fail(VDN_ERR_CUDA, "device query", e);
  if (major != 10 || minor != 0) return noalloc_fail(VDN_ERR_UNSUPPORTED, "libvdn is built for sm_100a (B200) only");
  char *scratch = nullptr;
  vdn_status rs = scratch_address(&scratch);
  if (rs != VDN_OK) return rs;
  cudaStream_t st = (cudaStream_t)stream;
  const Dims d = dims_of(s);
  // the status word must start at zero; the tables and tile list are rewritten below
  e = cudaMemsetAsync(scratch + p.status, 0, 256, st);
  if (e != cudaSuccess) return noalloc_fail(VDN_ERR_CUDA, "clearing the scratch status word", e);
  e = launch_tables(d, scratch, p, st);
  if (e != cudaSuccess) return noalloc_fail(VDN_ERR_CUDA, "tables launch", e);
  const float scale = sm_scale > 0.f ? sm_scale : 1.f / sqrtf((float)s.head_dim);
  const float sl2 = scale * 1.4426950408889634f;
  if (softmax_tc_supported(d, dtype))
    e = launch_softmax_tc(d, dtype, q, k, v, kt, vt, nullptr, sl2, o_s, lse, scratch, p, st);
  else
    e = launch_softmax_simt(d, dtype, q, k, v, kt, vt, sl2, o_s, lse, scratch, p, st);
  if (e != cudaSuccess) return noalloc_fail(VDN_ERR_CUDA, "softmax branch launch", e);
  return VDN_OK;
}
