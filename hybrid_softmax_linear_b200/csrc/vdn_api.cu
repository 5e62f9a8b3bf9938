// The C ABI of libvdn (declared in include/vdn.h): argument checks, workspace plan,
// and the order in which the layer's kernels are enqueued.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "vdn_internal.cuh"

using namespace vdn;

namespace {

thread_local char g_err[512] = "";

vdn_status fail(vdn_status code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

vdn_status ok() {
  g_err[0] = '\0';
  return VDN_OK;
}

vdn_status cuda_fail(cudaError_t e, const char *what) {
  return fail(VDN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

vdn_status check_shape(const vdn_shape *s) {
  if (s == nullptr) return fail(VDN_ERR_INVALID_ARG, "shape is NULL");
  if (s->frames < 1 || s->tokens_per_frame < 1 || s->chunk_frames < 1 || s->text_tokens < 0 || s->heads < 1)
    return fail(VDN_ERR_INVALID_ARG, "shape out of range (F=%d T=%d C=%d L=%d H=%d)", s->frames,
                s->tokens_per_frame, s->chunk_frames, s->text_tokens, s->heads);
  if (s->head_dim != 32 && s->head_dim != 64 && s->head_dim != 128)
    return fail(VDN_ERR_UNSUPPORTED, "head_dim %d not in {32, 64, 128}", s->head_dim);
  const int64_t nv = (int64_t)s->frames * s->tokens_per_frame;
  if (nv + s->text_tokens >= (int64_t)1 << 31 || (int64_t)s->heads * s->head_dim > 65536)
    return fail(VDN_ERR_INVALID_ARG, "shape too large (F*T + L must stay below 2^31, H*D <= 65536)");
  return VDN_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

vdn_status need(const void *p, const char *name) {
  if (p == nullptr) return fail(VDN_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(VDN_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return VDN_OK;
}

#define VDN_TRY(x)                     \
  do {                                 \
    vdn_status _s = (x);               \
    if (_s != VDN_OK) return _s;       \
  } while (0)

// sm_100 check, once per device
vdn_status check_device() {
  static int cached[64];  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(VDN_ERR_UNSUPPORTED, "device index %d", dev);
  if (cached[dev] == 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  if (cached[dev] != 1) return fail(VDN_ERR_UNSUPPORTED, "libvdn is built for sm_100a (B200) only");
  return VDN_OK;
}

vdn_status check_ws(void *ws, size_t ws_bytes, size_t needed) {
  if (ws == nullptr) return fail(VDN_ERR_WORKSPACE, "workspace is NULL");
  if (((uintptr_t)ws & (WS_ALIGN - 1)) != 0) return fail(VDN_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < needed) return fail(VDN_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, needed);
  return VDN_OK;
}

vdn_status check_act_dtype(vdn_dtype dt) {
  if (dt != VDN_F32 && dt != VDN_BF16) return fail(VDN_ERR_UNSUPPORTED, "dtype %d not supported here", (int)dt);
  return VDN_OK;
}

vdn_status check_kind(vdn_lin_kind kind) {
  if (kind != VDN_LIN_ELU1 && kind != VDN_LIN_DELTA) return fail(VDN_ERR_INVALID_ARG, "unknown kind %d", (int)kind);
  return VDN_OK;
}

#define VDN_CUDA(x, what)                               \
  do {                                                  \
    cudaError_t _e = (x);                               \
    if (_e != cudaSuccess) return cuda_fail(_e, what);  \
  } while (0)

// ---- per-kernel event timing (host state; off unless vdn_profile_begin was called)
struct Prof {
  bool on = false;
  int cap = 0, n = 0;
  cudaEvent_t *ev = nullptr;  // 2 per launch
  int *kid = nullptr;
} g_prof;

void prof_mark(int kid, bool start, cudaStream_t st) {
  if (!g_prof.on) return;
  if (start) {
    if (g_prof.n >= g_prof.cap) return;
    g_prof.kid[g_prof.n] = kid;
    cudaEventRecord(g_prof.ev[2 * g_prof.n], st);
  } else {
    if (g_prof.n >= g_prof.cap) return;
    cudaEventRecord(g_prof.ev[2 * g_prof.n + 1], st);
    ++g_prof.n;
  }
}

struct ProfScope {
  int kid;
  cudaStream_t st;
  ProfScope(int k, cudaStream_t s) : kid(k), st(s) { prof_mark(kid, true, st); }
  ~ProfScope() { prof_mark(kid, false, st); }
};

constexpr uint32_t DEBUG_MAX_POLLS = 1000000u;

float scale_log2_of(float sm_scale, int D) {
  const float s = sm_scale > 0.f ? sm_scale : 1.f / std::sqrt((float)D);
  return s * 1.4426950408889634f;
}

vdn_status softmax_dispatch(const Dims &d, vdn_dtype dt, const void *q, const void *k, const void *v,
                            const void *kt, const void *vt, const float *scales, float sl2, void *o, float *lse,
                            char *ws, const WsPlan &p, cudaStream_t st) {
  if (dt == VDN_E4M3 && !softmax_tc_supported(d, dt))
    return fail(VDN_ERR_UNSUPPORTED, "the e4m3 softmax branch needs head_dim 128");
  if (softmax_tc_supported(d, dt)) {
    ProfScope ps(K_SOFTMAX_TC, st);
    VDN_CUDA(launch_softmax_tc(d, dt, q, k, v, kt, vt, scales, sl2, o, lse, ws, p, st),
             "softmax branch (tensor cores) launch");
  } else {
    ProfScope ps(K_SOFTMAX_SIMT, st);
    VDN_CUDA(launch_softmax_simt(d, dt, q, k, v, kt, vt, sl2, o, lse, ws, p, st), "softmax branch launch");
  }
  return VDN_OK;
}

vdn_status state_build_dispatch(const Dims &d, vdn_lin_kind kind, vdn_dtype act, const void *k, const void *v,
                                const void *kt, const void *vt, float *S, float *z, float *St, float *zt, char *ws,
                                const WsPlan &p, cudaStream_t st, uint32_t *amax = nullptr) {
  if (kind == VDN_LIN_ELU1 && linear_tc_supported(d, act)) {
    ProfScope ps(K_STATE_TC, st);
    VDN_CUDA(launch_state_build_tc(d, k, v, kt, vt, S, z, St, zt, ws, p, st), "state build (tensor cores) launch");
  } else {
    ProfScope ps(K_STATE, st);
    VDN_CUDA(launch_state_build(d, kind, act, k, v, kt, vt, S, z, St, zt, st, amax), "state build launch");
  }
  return VDN_OK;
}

vdn_status out_proj_dispatch(const Dims &d, vdn_dtype act, const void *a, const void *w_os, const void *w_ol, void *y,
                             char *ws, const WsPlan &p, cudaStream_t st) {
  if (act == VDN_BF16 && out_proj_tc_supported(d)) {
    ProfScope ps(K_GEMM_TC, st);
    VDN_CUDA(launch_out_proj_tc(d, a, w_os, w_ol, y, ws, p, st), "out-proj (tensor cores) launch");
  } else {
    ProfScope ps(K_GEMM_SIMT, st);
    VDN_CUDA(launch_out_proj_simt(d, act, a, w_os, w_ol, y, st), "out-proj launch");
  }
  return VDN_OK;
}

}  // namespace

namespace vdn {
// lets entry points defined in other files report through vdn_last_error()
void set_last_error(const char *msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }
// the checks every softmax-branch entry point applies, shared so that they accept exactly
// the same arguments (each reports through vdn_last_error())
vdn_status softmax_args_check(const vdn_shape *shape, vdn_dtype dtype, const void *q, const void *k, const void *v,
                              const void *kt, const void *vt, const float *scales, float sm_scale, const void *o_s) {
  VDN_TRY(check_shape(shape));
  if (dtype != VDN_F32 && dtype != VDN_BF16 && dtype != VDN_E4M3)
    return fail(VDN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  VDN_TRY(need(q, "q")); VDN_TRY(need(k, "k")); VDN_TRY(need(v, "v")); VDN_TRY(need(o_s, "o_s"));
  if (shape->text_tokens > 0) { VDN_TRY(need(kt, "kt")); VDN_TRY(need(vt, "vt")); }
  if ((dtype == VDN_E4M3) != (scales != nullptr))
    return fail(VDN_ERR_INVALID_ARG, "scales must be given exactly when dtype is VDN_E4M3");
  if (!std::isfinite(sm_scale)) return fail(VDN_ERR_INVALID_ARG, "sm_scale is not finite");
  return VDN_OK;
}
vdn_status device_check() { return check_device(); }
float softmax_scale_log2(float sm_scale, int D) { return scale_log2_of(sm_scale, D); }
}  // namespace vdn

namespace vdn {
// workspace of the linear branch's backward: the step tables, then the per-frame states,
// the groups' memories, and the per-row and per-group scratch
struct LinBwdPlan {
  WsPlan p;
  size_t dnum, dden, dN, dZ, total;
};
LinBwdPlan plan_lin_bwd(const vdn_shape &s) {
  LinBwdPlan b;
  b.p = plan_workspace(s, VDN_LIN_ELU1, VDN_F32);
  const size_t F = s.frames, H = s.heads, D = s.head_dim, Nv = (size_t)s.frames * s.tokens_per_frame;
  const size_t G = (size_t)max_groups(s.frames, s.chunk_frames);
  size_t off = b.p.step_end;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
  b.p.S = take(F * H * D * D * 4);
  b.p.z = take(F * H * D * 4);
  b.p.St = take(H * D * D * 4);
  b.p.zt = take(H * D * 4);
  b.p.Sf = take(G * H * D * D * 4);
  b.p.Sb = take(G * H * D * D * 4);
  b.p.zf = take(G * H * D * 4);
  b.p.zb = take(G * H * D * 4);
  b.dnum = take(Nv * H * D * 4);
  b.dden = take(Nv * H * 4);
  b.dN = take(G * H * D * D * 4);
  b.dZ = take(G * H * D * 4);
  b.total = off;
  return b;
}
}  // namespace vdn

extern "C" {

int vdn_version(void) { return 100; }

const char *vdn_last_error(void) { return g_err; }

int32_t vdn_max_groups(const vdn_shape *shape) {
  if (check_shape(shape) != VDN_OK) return 0;
  return max_groups(shape->frames, shape->chunk_frames);
}

vdn_status vdn_mask_layout_build(const vdn_shape *shape, int32_t *frame_tab, int32_t *group_tab, int32_t *n_groups,
                                 size_t group_tab_cap) {
  VDN_TRY(check_shape(shape));
  if (frame_tab == nullptr || group_tab == nullptr || n_groups == nullptr)
    return fail(VDN_ERR_INVALID_ARG, "frame_tab, group_tab and n_groups must be non-NULL");
  const int cap = group_tab_cap > (size_t)1 << 30 ? 1 << 30 : (int)group_tab_cap;
  const int G = build_layout(shape->frames, shape->tokens_per_frame, shape->chunk_frames, shape->text_tokens,
                             frame_tab, group_tab, cap);
  if (G < 0) return fail(VDN_ERR_INVALID_ARG, "group_tab_cap %zu is below the group count", group_tab_cap);
  *n_groups = G;
  return ok();
}

size_t vdn_hybrid_attn_workspace_size(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype) {
  if (check_shape(shape) != VDN_OK || check_kind(kind) != VDN_OK) return 0;
  return plan_workspace(*shape, kind, dtype).total;
}

size_t vdn_step_workspace_size(const vdn_shape *shape) {
  if (check_shape(shape) != VDN_OK) return 0;
  return plan_workspace(*shape, VDN_LIN_ELU1, VDN_BF16).stage_end;
}

vdn_status vdn_workspace_init(void *ws, size_t ws_bytes, vdn_stream stream) {
  VDN_TRY(check_ws(ws, ws_bytes, 256));
  VDN_CUDA(cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream), "workspace init");
  return ok();
}

vdn_status vdn_softmax_branch_fwd(const vdn_shape *shape, vdn_dtype dtype, const void *q, const void *k,
                                  const void *v, const void *kt, const void *vt, const float *scales, float sm_scale,
                                  void *o_s, float *lse, void *ws, size_t ws_bytes, vdn_stream stream) {
  VDN_TRY(softmax_args_check(shape, dtype, q, k, v, kt, vt, scales, sm_scale, o_s));
  const WsPlan p = plan_workspace(*shape, VDN_LIN_ELU1, VDN_BF16);
  VDN_TRY(check_ws(ws, ws_bytes, p.step_end));
  VDN_TRY(check_device());
  const Dims d = dims_of(*shape);
  cudaStream_t st = (cudaStream_t)stream;
  VDN_CUDA(launch_tables(d, (char *)ws, p, st), "tables launch");
  VDN_TRY(softmax_dispatch(d, dtype, q, k, v, kt, vt, scales, scale_log2_of(sm_scale, d.D), o_s, lse, (char *)ws, p,
                           st));
  return ok();
}

vdn_status vdn_fp8_quant_per_head(const vdn_shape *shape, const void *q, const void *k, const void *v, const void *kt,
                                  const void *vt, void *q8, void *k8, void *v8, void *kt8, void *vt8, float *scales,
                                  void *ws, size_t ws_bytes, vdn_stream stream) {
  VDN_TRY(check_shape(shape));
  if ((int64_t)shape->heads * shape->head_dim > FP8_MAX_HD)
    return fail(VDN_ERR_UNSUPPORTED, "H*D above %d", FP8_MAX_HD);
  VDN_TRY(need(q, "q")); VDN_TRY(need(k, "k")); VDN_TRY(need(v, "v"));
  VDN_TRY(need(q8, "q8")); VDN_TRY(need(k8, "k8")); VDN_TRY(need(v8, "v8")); VDN_TRY(need(scales, "scales"));
  if (shape->text_tokens > 0) {
    VDN_TRY(need(kt, "kt")); VDN_TRY(need(vt, "vt")); VDN_TRY(need(kt8, "kt8")); VDN_TRY(need(vt8, "vt8"));
  }
  const WsPlan p = plan_workspace(*shape, VDN_LIN_ELU1, VDN_BF16);
  VDN_TRY(check_ws(ws, ws_bytes, p.step_end));
  VDN_TRY(check_device());
  cudaStream_t st = (cudaStream_t)stream;
  ProfScope ps(K_QUANT, st);
  VDN_CUDA(launch_fp8_quant(dims_of(*shape), q, k, v, kt, vt, q8, k8, v8, kt8, vt8, scales,
                            (uint32_t *)((char *)ws + p.qamax), st),
           "fp8 quantisation launch");
  return ok();
}

vdn_status vdn_linear_state_build(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, const void *k,
                                  const void *v, const void *kt, const void *vt, float *S, float *z, float *S_txt,
                                  float *z_txt, void *ws, size_t ws_bytes, vdn_stream stream) {
  VDN_TRY(check_shape(shape));
  VDN_TRY(check_kind(kind));
  VDN_TRY(check_act_dtype(dtype));
  VDN_TRY(need(k, "k")); VDN_TRY(need(v, "v")); VDN_TRY(need(S, "S")); VDN_TRY(need(z, "z"));
  VDN_TRY(need(S_txt, "S_txt"));
  if (kind == VDN_LIN_ELU1) VDN_TRY(need(z_txt, "z_txt"));
  if (shape->text_tokens > 0) { VDN_TRY(need(kt, "kt")); VDN_TRY(need(vt, "vt")); }
  const WsPlan p = plan_workspace(*shape, VDN_LIN_ELU1, VDN_BF16);
  VDN_TRY(check_ws(ws, ws_bytes, p.step_end));
  VDN_TRY(check_device());
  VDN_TRY(state_build_dispatch(dims_of(*shape), kind, dtype, k, v, kt, vt, S, z, S_txt, z_txt, (char *)ws, p,
                               (cudaStream_t)stream));
  return ok();
}

vdn_status vdn_linear_state_scan(const vdn_shape *shape, vdn_lin_kind kind, const float *S, const float *z,
                                 const float *S_txt, const float *z_txt, const float *beta, float *S_fwd,
                                 float *S_bwd, float *z_fwd, float *z_bwd, void *ws, size_t ws_bytes,
                                 vdn_stream stream) {
  VDN_TRY(check_shape(shape));
  VDN_TRY(check_kind(kind));
  VDN_TRY(need(S, "S")); VDN_TRY(need(S_txt, "S_txt")); VDN_TRY(need(S_fwd, "S_fwd")); VDN_TRY(need(S_bwd, "S_bwd"));
  if (kind == VDN_LIN_ELU1) {
    VDN_TRY(need(z, "z")); VDN_TRY(need(z_txt, "z_txt")); VDN_TRY(need(z_fwd, "z_fwd")); VDN_TRY(need(z_bwd, "z_bwd"));
  } else {
    VDN_TRY(need(z, "z (vbar)")); VDN_TRY(need(beta, "beta"));
  }
  const WsPlan p = plan_workspace(*shape, VDN_LIN_ELU1, VDN_BF16);
  VDN_TRY(check_ws(ws, ws_bytes, p.step_end));
  VDN_TRY(check_device());
  const Dims d = dims_of(*shape);
  cudaStream_t st = (cudaStream_t)stream;
  VDN_CUDA(launch_tables(d, (char *)ws, p, st), "tables launch");
  VDN_CUDA(launch_state_scan(d, kind, S, z, S_txt, z_txt, beta, S_fwd, S_bwd, z_fwd, z_bwd, (char *)ws, p, st),
           "scan launch");
  return ok();
}

vdn_status vdn_linear_read(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, const void *q,
                           const float *S_fwd, const float *S_bwd, const float *z_fwd, const float *z_bwd, void *o_l,
                           void *ws, size_t ws_bytes, vdn_stream stream) {
  VDN_TRY(check_shape(shape));
  VDN_TRY(check_kind(kind));
  VDN_TRY(check_act_dtype(dtype));
  VDN_TRY(need(q, "q")); VDN_TRY(need(S_fwd, "S_fwd")); VDN_TRY(need(S_bwd, "S_bwd")); VDN_TRY(need(o_l, "o_l"));
  if (kind == VDN_LIN_ELU1) { VDN_TRY(need(z_fwd, "z_fwd")); VDN_TRY(need(z_bwd, "z_bwd")); }
  const WsPlan p = plan_workspace(*shape, VDN_LIN_ELU1, VDN_BF16);
  VDN_TRY(check_ws(ws, ws_bytes, p.stage_end));
  VDN_TRY(check_device());
  const Dims d = dims_of(*shape);
  cudaStream_t st = (cudaStream_t)stream;
  VDN_CUDA(launch_tables(d, (char *)ws, p, st), "tables launch");
  if (linear_tc_supported(d, dtype)) {
    {
      ProfScope ps(K_READ_STAGE, st);
      VDN_CUDA(launch_read_stage(d, kind, S_fwd, S_bwd, z_fwd, z_bwd, nullptr, 0, (char *)ws, p, st), "read staging");
    }
    ProfScope ps(K_READ_TC, st);
    VDN_CUDA(launch_read_tc(d, kind, q, o_l, nullptr, 0, nullptr, 0.f, (char *)ws, p, st), "read launch");
  } else {
    ProfScope ps(K_READ, st);
    VDN_CUDA(launch_linear_read(d, kind, dtype, q, S_fwd, S_bwd, z_fwd, z_bwd, o_l, (char *)ws, p, st),
             "read launch");
  }
  return ok();
}

size_t vdn_linear_branch_bwd_workspace_size(const vdn_shape *shape) {
  if (check_shape(shape) != VDN_OK) return 0;
  return plan_lin_bwd(*shape).total;
}

vdn_status vdn_linear_branch_bwd(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, const void *q,
                                 const void *k, const void *v, const void *kt, const void *vt, const float *do_l,
                                 float *dq, float *dk, float *dv, float *dkt, float *dvt, void *ws, size_t ws_bytes,
                                 vdn_stream stream) {
  VDN_TRY(check_shape(shape));
  VDN_TRY(check_kind(kind));
  if (kind != VDN_LIN_ELU1) return fail(VDN_ERR_UNSUPPORTED, "the linear branch's backward is built for ELU1 only");
  if (dtype != VDN_BF16) return fail(VDN_ERR_UNSUPPORTED, "the linear branch's backward takes bf16 inputs");
  const int G = host_group_count(dims_of(*shape));
  if (linear_bwd_keys_smem(shape->head_dim, G) > MAX_DYN_SMEM)
    return fail(VDN_ERR_UNSUPPORTED, "%d groups: the backward's key kernel keeps one flag per group in shared "
                "memory, which this many groups overflow", G);
  VDN_TRY(need(q, "q")); VDN_TRY(need(k, "k")); VDN_TRY(need(v, "v")); VDN_TRY(need(do_l, "do_l"));
  VDN_TRY(need(dq, "dq")); VDN_TRY(need(dk, "dk")); VDN_TRY(need(dv, "dv"));
  if (shape->text_tokens > 0) {
    VDN_TRY(need(kt, "kt")); VDN_TRY(need(vt, "vt")); VDN_TRY(need(dkt, "dkt")); VDN_TRY(need(dvt, "dvt"));
  }
  const LinBwdPlan b = plan_lin_bwd(*shape);
  VDN_TRY(check_ws(ws, ws_bytes, b.total));
  VDN_TRY(check_device());
  const Dims d = dims_of(*shape);
  cudaStream_t st = (cudaStream_t)stream;
  char *w = (char *)ws;
  const WsPlan &p = b.p;
  VDN_CUDA(launch_tables(d, w, p, st), "tables launch");
  LinBwdArgs a{};
  a.d = d;
  a.q = q; a.k = k; a.v = v; a.kt = kt; a.vt = vt; a.dO = do_l;
  a.S = (float *)(w + p.S); a.z = (float *)(w + p.z); a.St = (float *)(w + p.St); a.zt = (float *)(w + p.zt);
  a.Sf = (float *)(w + p.Sf); a.Sb = (float *)(w + p.Sb); a.zf = (float *)(w + p.zf); a.zb = (float *)(w + p.zb);
  a.ftab = (const int32_t *)(w + p.ftab); a.gtab = (const int32_t *)(w + p.gtab);
  a.G = G;
  a.dnum = (float *)(w + b.dnum); a.dden = (float *)(w + b.dden);
  a.part = a.S; a.zpart = a.z;  // the per-frame states are dead once the scan has read them
  a.dN = (float *)(w + b.dN); a.dZ = (float *)(w + b.dZ);
  a.dq = dq; a.dk = dk; a.dv = dv; a.dkt = dkt; a.dvt = dvt;
  {
    ProfScope ps(K_STATE, st);
    VDN_CUDA(launch_linear_bwd(a, LIN_BWD_STATE, st), "state rebuild launch");
  }
  {
    ProfScope ps(K_SCAN, st);
    VDN_CUDA(launch_state_scan(d, VDN_LIN_ELU1, a.S, a.z, a.St, a.zt, nullptr, a.Sf, a.Sb, a.zf, a.zb, w, p, st),
             "scan launch");
  }
  static const int stages[4] = {LIN_BWD_ROWS, LIN_BWD_FRAMES, LIN_BWD_GROUPS, LIN_BWD_KEYS};
  static const int kids[4] = {K_LIN_BWD_ROWS, K_LIN_BWD_FRAMES, K_LIN_BWD_GROUPS, K_LIN_BWD_KEYS};
  for (int i = 0; i < 4; ++i) {
    ProfScope ps(kids[i], st);
    VDN_CUDA(launch_linear_bwd(a, stages[i], st), "linear branch backward launch");
  }
  return ok();
}

vdn_status vdn_hybrid_fuse(const vdn_shape *shape, vdn_dtype dtype, const void *q, const void *o_s, const void *o_l,
                           const float *w_gate_s, const float *w_gate_l, int32_t G_l, const float *gamma, float eps,
                           void *a, vdn_stream stream) {
  VDN_TRY(check_shape(shape));
  VDN_TRY(check_act_dtype(dtype));
  VDN_TRY(need(q, "q")); VDN_TRY(need(o_s, "o_s")); VDN_TRY(need(o_l, "o_l")); VDN_TRY(need(a, "a"));
  VDN_TRY(need(w_gate_s, "w_gate_s")); VDN_TRY(need(w_gate_l, "w_gate_l")); VDN_TRY(need(gamma, "gamma"));
  if (G_l != 1 && G_l != shape->head_dim) return fail(VDN_ERR_INVALID_ARG, "G_l must be 1 or D");
  if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(VDN_ERR_INVALID_ARG, "eps must be finite and >= 0");
  VDN_TRY(check_device());
  VDN_CUDA(launch_fuse(dims_of(*shape), dtype, q, o_s, o_l, w_gate_s, w_gate_l, G_l, gamma, eps, a,
                       (cudaStream_t)stream),
           "fuse launch");
  return ok();
}

vdn_status vdn_out_proj(const vdn_shape *shape, vdn_dtype dtype, const void *a, const void *w_os, const void *w_ol,
                        void *y, void *ws, size_t ws_bytes, vdn_stream stream) {
  VDN_TRY(check_shape(shape));
  VDN_TRY(check_act_dtype(dtype));
  VDN_TRY(need(a, "a")); VDN_TRY(need(w_os, "w_os")); VDN_TRY(need(w_ol, "w_ol")); VDN_TRY(need(y, "y"));
  const WsPlan p = plan_workspace(*shape, VDN_LIN_ELU1, VDN_BF16);
  VDN_TRY(check_ws(ws, ws_bytes, p.step_end));
  VDN_TRY(check_device());
  VDN_TRY(out_proj_dispatch(dims_of(*shape), dtype, a, w_os, w_ol, y, (char *)ws, p, (cudaStream_t)stream));
  return ok();
}

}  // extern "C"

namespace {
// The layer for this call's heads.  n_out = 0: y [N_v][HD] in the activation dtype (the
// whole layer).  n_out > 0: W_os, W_ol [n_out][HD] are these heads' input columns of a
// projection with n_out outputs, and y [N_v][n_out] receives float partial sums (the
// head-sharded layer; tensor-core path only).
vdn_status layer_impl(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, const void *q, const void *k,
                      const void *v, const void *kt, const void *vt, const float *beta, const float *w_gate_s,
                      const float *w_gate_l, int32_t G_l, const float *gamma, float eps, const void *w_os,
                      const void *w_ol, void *y, void *ws, size_t ws_bytes, vdn_stream stream, int32_t n_out) {
  VDN_TRY(check_shape(shape));
  VDN_TRY(check_kind(kind));
  if (dtype != VDN_F32 && dtype != VDN_BF16 && !dtype_e4m3_softmax(dtype))
    return fail(VDN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  VDN_TRY(need(q, "q")); VDN_TRY(need(k, "k")); VDN_TRY(need(v, "v")); VDN_TRY(need(y, "y"));
  if (shape->text_tokens > 0) { VDN_TRY(need(kt, "kt")); VDN_TRY(need(vt, "vt")); }
  VDN_TRY(need(w_gate_s, "w_gate_s")); VDN_TRY(need(w_gate_l, "w_gate_l")); VDN_TRY(need(gamma, "gamma"));
  VDN_TRY(need(w_os, "w_os")); VDN_TRY(need(w_ol, "w_ol"));
  if (kind == VDN_LIN_DELTA) VDN_TRY(need(beta, "beta"));
  else if (beta != nullptr) return fail(VDN_ERR_INVALID_ARG, "beta must be NULL for VDN_LIN_ELU1");
  if (G_l != 1 && G_l != shape->head_dim) return fail(VDN_ERR_INVALID_ARG, "G_l must be 1 or D");
  if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(VDN_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (dtype_e4m3_softmax(dtype) && (shape->head_dim != 128 || (int64_t)shape->heads * shape->head_dim > FP8_MAX_HD))
    return fail(VDN_ERR_UNSUPPORTED, "the e4m3 layer needs head_dim 128 and H*D <= %d", FP8_MAX_HD);
  if (dtype_e4m3_proj(dtype) && !out_proj_e4m3_supported(dims_of(*shape)))
    return fail(VDN_ERR_UNSUPPORTED, "the e4m3 projection needs H*D a multiple of 256");
  if (n_out > 0) {
    if (dtype_e4m3_proj(dtype) || !layer_fused(*shape, dtype) || !out_proj_tc_supported(dims_of(*shape)))
      return fail(VDN_ERR_UNSUPPORTED, "the partial layer runs bf16 or e4m3-softmax layers with head_dim 128");
    if (n_out % 32 != 0) return fail(VDN_ERR_INVALID_ARG, "out_features must be a multiple of 32");
  }
  const WsPlan p = plan_workspace(*shape, kind, dtype);
  VDN_TRY(check_ws(ws, ws_bytes, p.total));
  VDN_TRY(check_device());
  const Dims d = dims_of(*shape);
  cudaStream_t st = (cudaStream_t)stream;
  char *w = (char *)ws;
  const vdn_dtype act = dtype_e4m3_softmax(dtype) ? VDN_BF16 : dtype;
  const bool a8 = dtype_e4m3_proj(dtype);  // A in e4m3 for the e4m3 projection
  float *ascale = a8 ? (float *)(w + p.ascale) : nullptr;
  float *S = (float *)(w + p.S), *z = (float *)(w + p.z), *St = (float *)(w + p.St), *zt = (float *)(w + p.zt);
  float *Sf = (float *)(w + p.Sf), *Sb = (float *)(w + p.Sb), *zf = (float *)(w + p.zf), *zb = (float *)(w + p.zb);
  void *Os = w + p.Os, *Ol = w + p.Ol, *A = w + p.A;
  {
    ProfScope ps(K_TABLES, st);
    VDN_CUDA(launch_tables(d, w, p, st), "tables launch");
  }
  if (layer_fused(*shape, dtype)) {
    // tensor-core path: the softmax epilogue writes A_s = g_s * O_s and the linear read
    // writes A_l = g_l * gamma * RMSNorm(O_l), both straight into A.
    // e4m3 softmax with the delta rule: the frame statistics, the text init and the read
    // read every value of Q, K and V anyway, so they leave the per-head maxima behind, the
    // read runs before the softmax, and the quantisation is a single cast pass.
    const bool fold_amax = dtype_e4m3_softmax(dtype) && kind == VDN_LIN_DELTA && act == VDN_BF16 && d.D == 128 &&
                           linear_tc_supported(d, act) && w_gate_l != nullptr && G_l == d.D;
    uint32_t *amax = (uint32_t *)(w + p.amax);
    if (fold_amax) VDN_CUDA(cudaMemsetAsync(amax, 0, 3 * (size_t)d.H * sizeof(uint32_t), st), "amax clear");
    VDN_TRY(state_build_dispatch(d, kind, act, k, v, kt, vt, S, z, St, kind == VDN_LIN_ELU1 ? zt : nullptr, w, p,
                                 st, fold_amax ? amax : nullptr));
    const bool seg = layer_seg_scan(*shape, kind);
    {
      ProfScope ps(K_SCAN, st);
      if (seg)
        VDN_CUDA(launch_state_scan_sum(d, S, z, St, zt, w, p, st), "scan launch");
      else
        VDN_CUDA(launch_state_scan(d, kind, S, z, St, zt, beta, Sf, Sb, zf, zb, w, p, st), "scan launch");
    }
    if (!seg || (w_gate_l != nullptr && G_l == d.D)) {
      ProfScope ps(K_READ_STAGE, st);
      VDN_CUDA(launch_read_stage(d, kind, seg ? nullptr : Sf, Sb, zf, zb, w_gate_l, G_l, w, p, st), "read staging");
    }
    if (fold_amax) {
      // e4m3 projection: A_l's scales come from gamma alone (before the read); A_s's are
      // the V scales (after the cast)
      if (a8) VDN_CUDA(launch_a8_scales(d, nullptr, gamma, ascale, st, 2), "A scale launch");
      {
        ProfScope ps(K_READ_TC, st);
        VDN_CUDA(launch_read_tc(d, kind, q, A, w_gate_l, G_l, gamma, eps, w, p, st, a8 ? ascale + d.H : nullptr, amax),
                 "read launch");
      }
      {
        ProfScope ps(K_QUANT, st);
        VDN_CUDA(launch_fp8_cast(d, q, k, v, kt, vt, w + p.q8, w + p.k8, w + p.v8, w + p.kt8, w + p.vt8,
                                 (float *)(w + p.scales), amax, st),
                 "fp8 cast launch");
        if (a8)
          VDN_CUDA(launch_a8_scales(d, (const float *)(w + p.scales) + 2 * d.H, gamma, ascale, st, 1),
                   "A scale launch");
      }
      ProfScope ps(K_SOFTMAX_TC, st);
      VDN_CUDA(launch_softmax_tc_gated(d, VDN_E4M3, w + p.q8, w + p.k8, w + p.v8, w + p.kt8, w + p.vt8,
                                       (const float *)(w + p.scales), w_gate_s, scale_log2_of(0.f, d.D), A, w, p, st,
                                       a8),
               "softmax branch (tensor cores, e4m3) launch");
    } else if (dtype_e4m3_softmax(dtype)) {
      // per-head e4m3 Q/K/V for the softmax branch; the linear branch keeps the bf16 inputs
      {
        ProfScope ps(K_QUANT, st);
        VDN_CUDA(launch_fp8_quant(d, q, k, v, kt, vt, w + p.q8, w + p.k8, w + p.v8, w + p.kt8, w + p.vt8,
                                  (float *)(w + p.scales), (uint32_t *)(w + p.amax), st),
                 "fp8 quantisation launch");
        if (a8)
          VDN_CUDA(launch_a8_scales(d, (const float *)(w + p.scales) + 2 * d.H, gamma, ascale, st),
                   "A scale launch");
      }
      ProfScope ps(K_SOFTMAX_TC, st);
      VDN_CUDA(launch_softmax_tc_gated(d, VDN_E4M3, w + p.q8, w + p.k8, w + p.v8, w + p.kt8, w + p.vt8,
                                       (const float *)(w + p.scales), w_gate_s, scale_log2_of(0.f, d.D), A, w, p, st,
                                       a8),
               "softmax branch (tensor cores, e4m3) launch");
    } else {
      ProfScope ps(K_SOFTMAX_TC, st);
      VDN_CUDA(launch_softmax_tc_gated(d, VDN_BF16, q, k, v, kt, vt, nullptr, w_gate_s, scale_log2_of(0.f, d.D), A, w,
                                       p, st),
               "softmax branch (tensor cores) launch");
    }
    if (!fold_amax) {
      ProfScope ps(K_READ_TC, st);
      VDN_CUDA(launch_read_tc(d, kind, q, A, w_gate_l, G_l, gamma, eps, w, p, st, a8 ? ascale + d.H : nullptr),
               "read launch");
    }
  } else {
    VDN_TRY(softmax_dispatch(d, dtype, q, k, v, kt, vt, nullptr, scale_log2_of(0.f, d.D), Os, nullptr, w, p, st));
    VDN_TRY(state_build_dispatch(d, kind, act, k, v, kt, vt, S, z, St, kind == VDN_LIN_ELU1 ? zt : nullptr, w, p,
                                 st));
    {
      ProfScope ps(K_SCAN, st);
      VDN_CUDA(launch_state_scan(d, kind, S, z, St, zt, beta, Sf, Sb, zf, zb, w, p, st), "scan launch");
    }
    if (linear_tc_supported(d, act)) {
      {
        ProfScope ps(K_READ_STAGE, st);
        VDN_CUDA(launch_read_stage(d, kind, Sf, Sb, zf, zb, nullptr, 0, w, p, st), "read staging");
      }
      ProfScope ps(K_READ_TC, st);
      VDN_CUDA(launch_read_tc(d, kind, q, Ol, nullptr, 0, nullptr, 0.f, w, p, st), "read launch");
    } else {
      ProfScope ps(K_READ, st);
      VDN_CUDA(launch_linear_read(d, kind, act, q, Sf, Sb, zf, zb, Ol, w, p, st), "read launch");
    }
    {
      ProfScope ps(K_FUSE, st);
      VDN_CUDA(launch_fuse(d, act, q, Os, Ol, w_gate_s, w_gate_l, G_l, gamma, eps, A, st), "fuse launch");
    }
  }
  if (a8) {
    ProfScope ps(K_GEMM_TC, st);
    VDN_CUDA(launch_out_proj_e4m3(d, A, ascale, w_os, w_ol, y, (uint8_t *)(w + p.w8), (float *)(w + p.wsc),
                                  (DevStatus *)(w + p.status), st),
             "out-proj (tensor cores, e4m3) launch");
  } else if (n_out > 0) {
    ProfScope ps(K_GEMM_TC, st);
    VDN_CUDA(launch_out_proj_tc(d, A, w_os, w_ol, y, w, p, st, n_out, true), "out-proj (tensor cores) launch");
  } else {
    VDN_TRY(out_proj_dispatch(d, act, A, w_os, w_ol, y, w, p, st));
  }
  return ok();
}
}  // namespace

extern "C" {

vdn_status vdn_hybrid_attn_fwd(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, const void *q,
                               const void *k, const void *v, const void *kt, const void *vt, const float *beta,
                               const float *w_gate_s, const float *w_gate_l, int32_t G_l, const float *gamma,
                               float eps, const void *w_os, const void *w_ol, void *y, void *ws, size_t ws_bytes,
                               vdn_stream stream) {
  return layer_impl(shape, kind, dtype, q, k, v, kt, vt, beta, w_gate_s, w_gate_l, G_l, gamma, eps, w_os, w_ol, y,
                    ws, ws_bytes, stream, 0);
}

vdn_status vdn_hybrid_attn_fwd_partial(const vdn_shape *shape, int32_t out_features, vdn_lin_kind kind,
                                       vdn_dtype dtype, const void *q, const void *k, const void *v, const void *kt,
                                       const void *vt, const float *beta, const float *w_gate_s,
                                       const float *w_gate_l, int32_t G_l, const float *gamma, float eps,
                                       const void *w_os, const void *w_ol, float *y_partial, void *ws,
                                       size_t ws_bytes, vdn_stream stream) {
  if (out_features < 1) return fail(VDN_ERR_INVALID_ARG, "out_features must be >= 1");
  return layer_impl(shape, kind, dtype, q, k, v, kt, vt, beta, w_gate_s, w_gate_l, G_l, gamma, eps, w_os, w_ol,
                    y_partial, ws, ws_bytes, stream, out_features);
}

namespace {
// workspace of vdn_out_proj_e4m3: status word, the e4m3 weight copy, its column scales
struct ProjE4m3Plan {
  size_t status, w8, wsc, total;
};
ProjE4m3Plan plan_proj_e4m3(const vdn_shape &s) {
  ProjE4m3Plan pp{};
  const size_t hd = (size_t)s.heads * s.head_dim;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
  pp.status = take(256);
  pp.w8 = take(hd * 2 * hd);
  pp.wsc = take(hd * 4);
  pp.total = off;
  return pp;
}
}  // namespace

size_t vdn_out_proj_e4m3_workspace_size(const vdn_shape *shape) {
  if (check_shape(shape) != VDN_OK) return 0;
  return plan_proj_e4m3(*shape).total;
}

vdn_status vdn_out_proj_e4m3(const vdn_shape *shape, const void *a8, const float *a_scales, const void *w_os,
                             const void *w_ol, void *y, void *ws, size_t ws_bytes, vdn_stream stream) {
  VDN_TRY(check_shape(shape));
  VDN_TRY(need(a8, "a8")); VDN_TRY(need(a_scales, "a_scales")); VDN_TRY(need(w_os, "w_os"));
  VDN_TRY(need(w_ol, "w_ol")); VDN_TRY(need(y, "y"));
  const Dims d = dims_of(*shape);
  if (!out_proj_e4m3_supported(d)) return fail(VDN_ERR_UNSUPPORTED, "the e4m3 projection needs H*D a multiple of 256");
  const ProjE4m3Plan pp = plan_proj_e4m3(*shape);
  VDN_TRY(check_ws(ws, ws_bytes, pp.total));
  VDN_TRY(check_device());
  char *w = (char *)ws;
  cudaStream_t st = (cudaStream_t)stream;
  ProfScope ps(K_GEMM_TC, st);
  VDN_CUDA(launch_out_proj_e4m3(d, a8, a_scales, w_os, w_ol, y, (uint8_t *)(w + pp.w8), (float *)(w + pp.wsc),
                                (DevStatus *)(w + pp.status), st),
           "out-proj (tensor cores, e4m3) launch");
  return ok();
}

namespace {
// Staging area of the host entry point, after the layer's workspace.
struct HostStage {
  size_t q, k, v, kt, vt, beta, y, total;
};
HostStage plan_host_stage(const vdn_shape &s, vdn_lin_kind kind, vdn_dtype dtype) {
  HostStage h{};
  const size_t act = dtype == VDN_F32 ? 4 : 2;
  const size_t nv = (size_t)s.frames * s.tokens_per_frame, hd = (size_t)s.heads * s.head_dim;
  size_t off = plan_workspace(s, kind, dtype).total;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
  h.q = take(nv * hd * act);
  h.k = take(nv * hd * act);
  h.v = take(nv * hd * act);
  h.kt = take((size_t)s.text_tokens * hd * act);
  h.vt = take((size_t)s.text_tokens * hd * act);
  h.beta = take(kind == VDN_LIN_DELTA ? (size_t)s.frames * s.heads * 4 : 0);
  h.y = take(nv * hd * act);
  h.total = off;
  return h;
}
}  // namespace

size_t vdn_hybrid_attn_host_workspace_size(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype) {
  if (check_shape(shape) != VDN_OK || check_kind(kind) != VDN_OK) return 0;
  return plan_host_stage(*shape, kind, dtype).total;
}

vdn_status vdn_hybrid_attn_fwd_host(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, const void *q_host,
                                    const void *k_host, const void *v_host, const void *kt_host,
                                    const void *vt_host, const float *beta_host, const float *w_gate_s,
                                    const float *w_gate_l, int32_t G_l, const float *gamma, float eps,
                                    const void *w_os, const void *w_ol, void *y_host, void *ws, size_t ws_bytes,
                                    vdn_stream stream) {
  VDN_TRY(check_shape(shape));
  VDN_TRY(check_kind(kind));
  if (dtype != VDN_F32 && dtype != VDN_BF16 && !dtype_e4m3_softmax(dtype))
    return fail(VDN_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  const bool text = shape->text_tokens > 0;
  if (q_host == nullptr || k_host == nullptr || v_host == nullptr || y_host == nullptr ||
      (text && (kt_host == nullptr || vt_host == nullptr)))
    return fail(VDN_ERR_INVALID_ARG, "a host tensor pointer is NULL");
  if (kind == VDN_LIN_DELTA && beta_host == nullptr) return fail(VDN_ERR_INVALID_ARG, "beta is NULL");
  const HostStage h = plan_host_stage(*shape, kind, dtype);
  VDN_TRY(check_ws(ws, ws_bytes, h.total));
  VDN_TRY(check_device());
  cudaStream_t st = (cudaStream_t)stream;
  char *w = (char *)ws;
  const size_t act = dtype == VDN_F32 ? 4 : 2;
  const size_t nv = (size_t)shape->frames * shape->tokens_per_frame, hd = (size_t)shape->heads * shape->head_dim;
  const size_t big = nv * hd * act, small = (size_t)shape->text_tokens * hd * act;
  VDN_CUDA(cudaMemcpyAsync(w + h.q, q_host, big, cudaMemcpyHostToDevice, st), "copy of q to the device");
  VDN_CUDA(cudaMemcpyAsync(w + h.k, k_host, big, cudaMemcpyHostToDevice, st), "copy of k to the device");
  VDN_CUDA(cudaMemcpyAsync(w + h.v, v_host, big, cudaMemcpyHostToDevice, st), "copy of v to the device");
  if (text) {
    VDN_CUDA(cudaMemcpyAsync(w + h.kt, kt_host, small, cudaMemcpyHostToDevice, st), "copy of kt to the device");
    VDN_CUDA(cudaMemcpyAsync(w + h.vt, vt_host, small, cudaMemcpyHostToDevice, st), "copy of vt to the device");
  }
  if (kind == VDN_LIN_DELTA)
    VDN_CUDA(cudaMemcpyAsync(w + h.beta, beta_host, (size_t)shape->frames * shape->heads * 4,
                             cudaMemcpyHostToDevice, st),
             "copy of beta to the device");
  VDN_TRY(vdn_hybrid_attn_fwd(shape, kind, dtype, w + h.q, w + h.k, w + h.v, text ? w + h.kt : nullptr,
                              text ? w + h.vt : nullptr, kind == VDN_LIN_DELTA ? (const float *)(w + h.beta) : nullptr,
                              w_gate_s, w_gate_l, G_l, gamma, eps, w_os, w_ol, w + h.y, ws, ws_bytes, stream));
  VDN_CUDA(cudaMemcpyAsync(y_host, w + h.y, big, cudaMemcpyDeviceToHost, st), "copy of y to the host");
  return ok();
}

void *vdn_hybrid_attn_intermediate(const vdn_shape *shape, vdn_lin_kind kind, vdn_dtype dtype, void *ws, int which) {
  if (check_shape(shape) != VDN_OK || ws == nullptr) return nullptr;
  const WsPlan p = plan_workspace(*shape, kind, dtype);
  char *w = (char *)ws;
  const bool fused = layer_fused(*shape, dtype);
  switch (which) {
    case 0: return fused ? nullptr : w + p.Os;
    case 1: return fused ? nullptr : w + p.Ol;
    case 2: return w + p.A;
    case 3: return (fused && layer_seg_scan(*shape, kind)) ? nullptr : w + p.Sf;
    case 4: return (fused && layer_seg_scan(*shape, kind)) ? nullptr : w + p.Sb;
    case 5: return w + p.ftab;
    case 6: return w + p.gtab;
    case 7: return w + p.tiles;
    case 8: return w + p.meta;
    case 9: return w + p.splan;
    default: return nullptr;
  }
}

vdn_status vdn_check_device_status(void *ws, size_t ws_bytes, vdn_stream stream) {
  VDN_TRY(check_ws(ws, ws_bytes, 256));
  cudaStream_t st = (cudaStream_t)stream;
  VDN_CUDA(cudaStreamSynchronize(st), "stream synchronize");
  DevStatus h{};
  VDN_CUDA(cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost), "status read");
  VDN_CUDA(cudaMemset(ws, 0, sizeof(h)), "status clear");
  if (h.code == 0) return ok();
  const vdn_status code = h.code == VDN_ERR_TIMEOUT ? VDN_ERR_TIMEOUT : VDN_ERR_DEVICE;
  return fail(code, "device status %u from kernel %u, block %u, detail %u", h.code, h.where, h.block, h.detail);
}

vdn_status vdn_profile_begin(int32_t max_launches) {
  if (max_launches < 1 || max_launches > (1 << 20)) return fail(VDN_ERR_INVALID_ARG, "max_launches out of range");
  if (g_prof.cap < max_launches) {
    for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
    delete[] g_prof.ev;
    delete[] g_prof.kid;
    g_prof.ev = new cudaEvent_t[2 * max_launches];
    g_prof.kid = new int[max_launches];
    g_prof.cap = 0;
    for (int i = 0; i < 2 * max_launches; ++i) VDN_CUDA(cudaEventCreate(&g_prof.ev[i]), "event create");
    g_prof.cap = max_launches;
  }
  g_prof.n = 0;
  g_prof.on = true;
  return ok();
}

vdn_status vdn_profile_end(float *ms, int32_t *launches, int32_t n) {
  if (ms == nullptr || launches == nullptr || n < 1) return fail(VDN_ERR_INVALID_ARG, "bad output arrays");
  for (int i = 0; i < n; ++i) { ms[i] = 0.f; launches[i] = 0; }
  g_prof.on = false;
  for (int i = 0; i < g_prof.n; ++i) {
    VDN_CUDA(cudaEventSynchronize(g_prof.ev[2 * i + 1]), "event sync");
    float t = 0.f;
    VDN_CUDA(cudaEventElapsedTime(&t, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]), "event elapsed");
    const int k = g_prof.kid[i];
    if (k >= 0 && k < n) { ms[k] += t; launches[k] += 1; }
  }
  g_prof.n = 0;
  return ok();
}

vdn_status vdn_debug_unset_flag_wait(void *ws, size_t ws_bytes, uint32_t max_polls, vdn_stream stream) {
  VDN_TRY(check_ws(ws, ws_bytes, 256));
  // at about 64 ns a poll, 10^6 polls keep the test wait near 64 ms
  if (max_polls == 0 || max_polls > DEBUG_MAX_POLLS)
    return fail(VDN_ERR_INVALID_ARG, "max_polls must be in [1, %u]", DEBUG_MAX_POLLS);
  VDN_TRY(check_device());
  VDN_CUDA(launch_debug_wait((char *)ws, max_polls, (cudaStream_t)stream), "debug wait launch");
  return ok();
}

}  // extern "C"
