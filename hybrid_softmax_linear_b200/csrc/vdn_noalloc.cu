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
// address: every call looks the address up with cudaGetSymbolAddress in the context
// current at that moment (a host-side lookup) and passes it to the kernels, so a caller
// that switches contexts never gets an address that belongs to another one.  The first
// call on a device (or in a new context) also loads the library's device code there,
// which is why that first call should come before any stream capture.
#include <cstdio>

#include "vdn_internal.cuh"

namespace vdn {
void set_last_error(const char *msg);  // vdn_api.cu
vdn_status softmax_args_check(const vdn_shape *shape, vdn_dtype dtype, const void *q, const void *k, const void *v,
                              const void *kt, const void *vt, const float *scales, float sm_scale, const void *o_s);
vdn_status device_check();
float softmax_scale_log2(float sm_scale, int D);

namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = 256u * 1024u;  // 256 KiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

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

// Device address of the scratch array in the current context.
vdn_status scratch_address(char **out) {
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr)
    return noalloc_fail(VDN_ERR_CUDA, "cudaGetSymbolAddress of the static scratch array", e);
  *out = (char *)p;
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
  // the same argument checks as vdn_softmax_branch_fwd; e4m3 needs its scales, which this
  // entry point does not take
  if (dtype != VDN_F32 && dtype != VDN_BF16)
    return noalloc_fail(VDN_ERR_UNSUPPORTED, "dtype must be VDN_F32 or VDN_BF16");
  vdn_status rs = softmax_args_check(shape, dtype, q, k, v, kt, vt, nullptr, sm_scale, o_s);
  if (rs != VDN_OK) return rs;
  const vdn_shape &s = *shape;
  const WsPlan p = plan_workspace(s, VDN_LIN_ELU1, VDN_BF16);
  if (p.step_end > NOALLOC_SCRATCH_BYTES)
    return noalloc_fail(VDN_ERR_WORKSPACE,
                        "shape needs more scratch than the fixed 256 KiB array (tables and query-tile list); "
                        "use vdn_softmax_branch_fwd with a workspace");
  rs = device_check();
  if (rs != VDN_OK) return rs;
  char *scratch = nullptr;
  rs = scratch_address(&scratch);
  if (rs != VDN_OK) return rs;
  cudaStream_t st = (cudaStream_t)stream;
  const Dims d = dims_of(s);
  // the status word must start at zero; the tables and tile list are rewritten below
  cudaError_t e = cudaMemsetAsync(scratch + p.status, 0, 256, st);
  if (e != cudaSuccess) return noalloc_fail(VDN_ERR_CUDA, "clearing the scratch status word", e);
  e = launch_tables(d, scratch, p, st);
  if (e != cudaSuccess) return noalloc_fail(VDN_ERR_CUDA, "tables launch", e);
  const float sl2 = softmax_scale_log2(sm_scale, s.head_dim);
  if (softmax_tc_supported(d, dtype))
    e = launch_softmax_tc(d, dtype, q, k, v, kt, vt, nullptr, sl2, o_s, lse, scratch, p, st);
  else
    e = launch_softmax_simt(d, dtype, q, k, v, kt, vt, sl2, o_s, lse, scratch, p, st);
  if (e != cudaSuccess) return noalloc_fail(VDN_ERR_CUDA, "softmax branch launch", e);
  return VDN_OK;
}
