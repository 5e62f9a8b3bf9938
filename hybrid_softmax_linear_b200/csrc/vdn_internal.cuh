// Internal declarations of libvdn: layout rules (host and device), workspace plan,
// device status word, element conversions and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/vdn.h"

#define VDN_HD __host__ __device__ __forceinline__

namespace vdn {

// ---------------------------------------------------------------- layout rules
// Window of a query frame: its chunk and the chunks on either side ("VDN-MiniMax-H3
// 开源" article, 技术解读 / 局部精确计算 para. 1); chunks start at frame 0.
VDN_HD void chunk_window(int f, int F, int C, int *lo, int *hi) {
  int c = f / C;
  int a = (c - 1) * C, b = (c + 2) * C;
  *lo = a < 0 ? 0 : a;
  *hi = b > F ? F : b;
}

VDN_HD bool is_anchor(int f, int F) { return f == 0 || f == F - 1; }

struct FrameSets {
  int nseg;
  int seg[4][2];  // softmax key segments in [text | video] index space
  int fwd[2];     // forward-memory frames, empty = (0, 0)
  int bwd[2];     // backward-memory frames, empty = (0, 0)
  int win[2];
  int anchor;
};

// Key sets of query frame f.  Anchors read every frame by softmax and have empty
// memories; other frames read {0} + window + {F-1} by softmax, the frames in
// [1, win_lo) through the forward memory and [win_hi, F-1) through the backward one.
VDN_HD void frame_sets(int f, int F, int T, int C, int L, FrameSets *s) {
  int lo, hi;
  s->anchor = is_anchor(f, F) ? 1 : 0;
  if (s->anchor) { lo = 0; hi = F; } else { chunk_window(f, F, C, &lo, &hi); }
  s->win[0] = lo; s->win[1] = hi;
  // candidate token ranges, already in ascending order
  int cand[4][2];
  int nc = 0;
  if (L > 0) { cand[nc][0] = 0; cand[nc][1] = L; ++nc; }
  if (s->anchor) {
    cand[nc][0] = L; cand[nc][1] = L + F * T; ++nc;
  } else {
    cand[nc][0] = L; cand[nc][1] = L + T; ++nc;                       // frame 0
    cand[nc][0] = L + lo * T; cand[nc][1] = L + hi * T; ++nc;         // window
    cand[nc][0] = L + (F - 1) * T; cand[nc][1] = L + F * T; ++nc;     // frame F-1
  }
  s->nseg = 0;
  for (int i = 0; i < 4; ++i) { s->seg[i][0] = 0; s->seg[i][1] = 0; }
  for (int i = 0; i < nc; ++i) {
    if (s->nseg > 0 && cand[i][0] <= s->seg[s->nseg - 1][1]) {
      if (cand[i][1] > s->seg[s->nseg - 1][1]) s->seg[s->nseg - 1][1] = cand[i][1];
    } else {
      s->seg[s->nseg][0] = cand[i][0]; s->seg[s->nseg][1] = cand[i][1]; ++s->nseg;
    }
  }
  s->fwd[0] = s->fwd[1] = s->bwd[0] = s->bwd[1] = 0;
  if (!s->anchor) {
    int a = 1, b = lo;            // [1, lo): before the window, frame 0 excluded
    if (b > a) { s->fwd[0] = a; s->fwd[1] = b; }
    a = hi; b = F - 1;            // [hi, F-1): after the window, frame F-1 excluded
    if (b > a) { s->bwd[0] = a; s->bwd[1] = b; }
  }
}

VDN_HD bool same_sets(const FrameSets &x, const FrameSets &y) {
  if (x.nseg != y.nseg) return false;
  for (int i = 0; i < 4; ++i)
    if (x.seg[i][0] != y.seg[i][0] || x.seg[i][1] != y.seg[i][1]) return false;
  return x.fwd[0] == y.fwd[0] && x.fwd[1] == y.fwd[1] && x.bwd[0] == y.bwd[0] && x.bwd[1] == y.bwd[1];
}

VDN_HD int max_groups(int F, int C) { return (F + C - 1) / C + 2; }

// Fills frame_tab [F][8] and group_tab [cap][16]; returns G, or -1 if cap < G.
VDN_HD int build_layout(int F, int T, int C, int L, int32_t *ftab, int32_t *gtab, int cap) {
  FrameSets prev, cur;
  int G = 0;
  for (int f = 0; f < F; ++f) {
    frame_sets(f, F, T, C, L, &cur);
    bool extend = f > 0 && same_sets(cur, prev);
    if (extend) {
      gtab[(G - 1) * 16 + 1] = f + 1;
    } else {
      if (G >= cap) return -1;
      int32_t *r = gtab + G * 16;
      r[0] = f; r[1] = f + 1; r[2] = cur.nseg; r[3] = 0;
      for (int i = 0; i < 4; ++i) { r[4 + 2 * i] = cur.seg[i][0]; r[5 + 2 * i] = cur.seg[i][1]; }
      r[12] = cur.fwd[0]; r[13] = cur.fwd[1]; r[14] = cur.bwd[0]; r[15] = cur.bwd[1];
      ++G;
    }
    int32_t *fr = ftab + f * 8;
    fr[0] = G - 1; fr[1] = cur.win[0]; fr[2] = cur.win[1]; fr[3] = cur.anchor;
    fr[4] = cur.fwd[0]; fr[5] = cur.fwd[1]; fr[6] = cur.bwd[0]; fr[7] = cur.bwd[1];
    prev = cur;
  }
  return G;
}

VDN_HD int group_keys(const int32_t *grow) {
  int n = 0;
  for (int i = 0; i < grow[2]; ++i) n += grow[5 + 2 * i] - grow[4 + 2 * i];
  return n;
}

// ---------------------------------------------------------------- query tiles
// Query rows are cut into tiles of TILE_M rows that never straddle a group, so every
// row of a tile shares one key set.  Tiles are listed longest key set first.
constexpr int TILE_M = 256;
constexpr int TILE_REC = 8;  // {group, row_lo, row_hi, n_keys, first tile of the group, tiles of the group, 0, 0}

VDN_HD int64_t max_tiles(int F, int T, int C) {
  return (int64_t)F * T / TILE_M + max_groups(F, C) + 1;
}

// ---------------------------------------------------------------- workspace plan
constexpr size_t WS_ALIGN = 256;
VDN_HD size_t align_up(size_t x) { return (x + WS_ALIGN - 1) / WS_ALIGN * WS_ALIGN; }

// Scan plan (written by the tables kernel): the frames [1, F-1) that the two memories
// can hold are cut at every memory boundary (the end e_g of a forward memory and the
// start b_g of a backward one) into nseg segments; the forward memory of group g is the
// sum of segments [0, ie[g]) and its backward memory that of segments [ib[g], nseg).
// int32 layout: {nseg, G, 0, 0, bnd[F + 1], ie[gcap], ib[gcap]} with bnd[j] the first
// frame of segment j and bnd[nseg] = F - 1.
VDN_HD int64_t splan_ints(int F, int gcap) { return 4 + (int64_t)F + 1 + 2 * (int64_t)gcap; }
VDN_HD int splan_ie(int F) { return 4 + F + 1; }
VDN_HD int splan_ib(int F, int gcap) { return 4 + F + 1 + gcap; }
// Segments one block of the segmented scan keeps in shared memory (three float4 rows of
// 32 lanes per segment); layouts with more fall back to the per-frame walk.
constexpr int SCAN_SEG_MAX = 96;

// Memory boundaries of a group: forward memory [1, e), backward memory [b, F-1).
VDN_HD void memory_bounds(const FrameSets &s, int F, int *e, int *b) {
  *e = s.fwd[1] > s.fwd[0] ? s.fwd[1] : 1;
  *b = s.bwd[1] > s.bwd[0] ? s.bwd[0] : F - 1;
}

struct WsPlan {
  // step part (tables, tile list, scan plan, tables scratch, status)
  size_t status, ftab, gtab, meta, qamax, tiles, splan, tscr, step_end;
  // read staging: per-group summed memory in bf16 (tensor-core B operand), summed
  // normaliser, linear-gate weights in bf16
  size_t ssum, zsum, wl, stage_end;
  // layer part
  size_t S, z, St, zt, Sf, Sb, zf, zb, Os, Ol, A, q8, k8, v8, kt8, vt8, scales, amax, ascale, w8, wsc, total;
};

// e4m3 softmax branch (VDN_E4M3 and VDN_E4M3_PROJ); e4m3 output projection as well
inline bool dtype_e4m3_softmax(vdn_dtype dt) { return dt == VDN_E4M3 || dt == VDN_E4M3_PROJ; }
inline bool dtype_e4m3_proj(vdn_dtype dt) { return dt == VDN_E4M3_PROJ; }

// The whole layer runs on the tensor-core path (softmax and linear read write A
// directly; O_s and O_l are never stored) for bf16 activations with D = 128.
inline bool layer_fused(const vdn_shape &s, vdn_dtype dtype) {
  return (dtype == VDN_BF16 || dtype_e4m3_softmax(dtype)) && s.head_dim == 128;
}

// Number of scan segments of a layout (the same rule the tables kernel applies).
inline int host_scan_segments(int F, int T, int C, int L) {
  if (F < 3) return 0;
  int n = 0;
  bool *mark = new bool[F + 1]();
  mark[1] = mark[F - 1] = true;
  FrameSets cur;
  for (int f = 0; f < F; ++f) {
    frame_sets(f, F, T, C, L, &cur);
    int e, b;
    memory_bounds(cur, F, &e, &b);
    mark[e] = mark[b] = true;
  }
  for (int f = 1; f <= F - 1; ++f) n += mark[f] ? 1 : 0;
  delete[] mark;
  return n - 1;
}

// The ELU1 memories go through the segmented scan when the segments fit one block.
inline bool layer_seg_scan(const vdn_shape &s, vdn_lin_kind kind) {
  return kind == VDN_LIN_ELU1 &&
         host_scan_segments(s.frames, s.tokens_per_frame, s.chunk_frames, s.text_tokens) <= SCAN_SEG_MAX;
}

// meta: int32[8] = {G, n_tiles, ...}
inline WsPlan plan_workspace(const vdn_shape &s, vdn_lin_kind kind, vdn_dtype dtype) {
  WsPlan p{};
  size_t F = s.frames, T = s.tokens_per_frame, L = s.text_tokens, H = s.heads, D = s.head_dim;
  size_t G = (size_t)max_groups(s.frames, s.chunk_frames);
  size_t Nv = F * T;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
  p.status = take(256);
  p.ftab = take(F * 8 * 4);
  p.gtab = take(G * 16 * 4);
  p.meta = take(64);
  p.qamax = take(3 * H * 4);
  p.tiles = take((size_t)max_tiles(s.frames, s.tokens_per_frame, s.chunk_frames) * TILE_REC * 4);
  p.splan = take((size_t)splan_ints(s.frames, (int)G) * 4);
  p.tscr = take((4 * G + 2 * (F + 1)) * 4);  // keys, order, count, first; mark, idx
  p.step_end = off;
  // bf16 operands of the tensor-core read: per (group, 128-feature head group) a 128 x 128
  // block-diagonal S_sum and W_l (one block per head: 128 / D heads per head group), so
  // G * H * D * 128 entries (G * H * D * D when D = 128)
  p.ssum = take(G * H * D * 128 * 2);
  p.zsum = take(G * H * D * 4);
  p.wl = take(H * D * 128 * 2);
  p.stage_end = off;
  size_t act = (dtype == VDN_F32) ? 4 : 2;
  // per-frame states: ELU1 S [F][H][D][D]; DELTA kbar [F][H][D] in S, vbar in z
  p.S = take(kind == VDN_LIN_ELU1 ? F * H * D * D * 4 : F * H * D * 4);
  p.z = take(F * H * D * 4);
  p.St = take(H * D * D * 4);
  p.zt = take(H * D * 4);
  // the segmented scan of the fused layer writes the bf16 sum S_fwd + S_bwd directly
  const bool fused = layer_fused(s, dtype);
  const size_t Gm = (fused && layer_seg_scan(s, kind)) ? 0 : G;
  p.Sf = take(Gm * H * D * D * 4);
  p.Sb = take(Gm * H * D * D * 4);
  p.zf = take(Gm * H * D * 4);
  p.zb = take(Gm * H * D * 4);
  p.Os = take(fused ? 0 : Nv * H * D * act);
  p.Ol = take(fused ? 0 : Nv * H * D * act);
  // A: bf16 (or float), or e4m3 codes when the projection runs in e4m3
  p.A = take(Nv * 2 * H * D * (dtype_e4m3_proj(dtype) ? 1 : act));
  if (dtype_e4m3_softmax(dtype)) {
    p.q8 = take(Nv * H * D);
    p.k8 = take(Nv * H * D);
    p.v8 = take(Nv * H * D);
    p.kt8 = take(L * H * D + 16);
    p.vt8 = take(L * H * D + 16);
    p.scales = take(3 * H * 4);
    p.amax = take(3 * H * 4);
  }
  if (dtype_e4m3_proj(dtype)) {
    p.ascale = take(2 * H * 4);          // A's dequantisation scales per (branch half, head)
    p.w8 = take(H * D * 2 * H * D);      // e4m3 [W_os | W_ol] with A's scales folded in
    p.wsc = take(H * D * 4);             // its per-output-column scales
  }
  p.total = off;
  return p;
}

// ---------------------------------------------------------------- device status word
struct DevStatus {
  uint32_t code;    // 0 ok, VDN_ERR_TIMEOUT, VDN_ERR_DEVICE
  uint32_t where;   // kernel id
  uint32_t block;   // linear block index of the first reporter
  uint32_t detail;  // kernel-specific
};

enum KernelId : uint32_t {
  K_TABLES = 1, K_SOFTMAX_SIMT = 2, K_SOFTMAX_TC = 3, K_STATE = 4, K_SCAN = 5, K_READ = 6,
  K_FUSE = 7, K_GEMM_SIMT = 8, K_GEMM_TC = 9, K_QUANT = 10, K_DELTA = 11, K_DEBUG_WAIT = 12,
  K_STATE_TC = 13, K_READ_STAGE = 14, K_READ_TC = 15, K_LIN_BWD_ROWS = 16, K_LIN_BWD_FRAMES = 17,
  K_LIN_BWD_KEYS = 18, K_LIN_BWD_GROUPS = 19,
};

__device__ __forceinline__ void report(DevStatus *st, uint32_t code, uint32_t where, uint32_t detail) {
  if (atomicCAS(&st->code, 0u, code) == 0u) {
    st->where = where;
    st->block = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    st->detail = detail;
  }
}

// ---------------------------------------------------------------- range-check build
// Built with VDN_BOUNDS_CHECK=1 (libvdn_checked.so, a test build standing in for a memory
// checker), the tensor-core kernels check every global index they derive from the layout
// tables against its tensor's extent before use; the first violation goes to the status
// word as VDN_ERR_DEVICE with detail 0x10000 | site, and the access is skipped.  The
// normal build compiles the checks away.
#ifndef VDN_BOUNDS_CHECK
#define VDN_BOUNDS_CHECK 0
#endif
__device__ __forceinline__ bool in_range(DevStatus *st, int64_t i, int64_t n, uint32_t kid, uint32_t site) {
#if VDN_BOUNDS_CHECK
  if (i >= 0 && i < n) return true;
  report(st, VDN_ERR_DEVICE, kid, 0x10000u | site);
  return false;
#else
  (void)st; (void)i; (void)n; (void)kid; (void)site;
  return true;
#endif
}

// Bound on device polls of an mbarrier or flag before a kernel gives up (about a
// second at the polling rates involved).  Settable per call for the wait test.
constexpr uint32_t DEFAULT_MAX_POLLS = 1u << 26;

// ---------------------------------------------------------------- element access
template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// elu(x) + 1 as max(x, 0) + e^min(x, 0): no branch, the same value (e^0 = 1 exactly)
__device__ __forceinline__ float phi_elu1(float x) { return fmaxf(x, 0.f) + expf(fminf(x, 0.f)); }

// ---------------------------------------------------------------- launchers
struct Dims {
  int F, T, C, L, H, D;
  __host__ __device__ int64_t Nv() const { return (int64_t)F * T; }
};

inline Dims dims_of(const vdn_shape &s) {
  return Dims{s.frames, s.tokens_per_frame, s.chunk_frames, s.text_tokens, s.heads, s.head_dim};
}

// Group and tile counts from the same rules the device tables kernel runs.
inline int host_group_count(const Dims &d) {
  FrameSets prev, cur;
  int G = 0;
  for (int f = 0; f < d.F; ++f) {
    frame_sets(f, d.F, d.T, d.C, d.L, &cur);
    if (!(f > 0 && same_sets(cur, prev))) ++G;
    prev = cur;
  }
  return G;
}

inline int host_tile_count(const Dims &d) {
  FrameSets prev, cur;
  int64_t n = 0, lo = 0;
  for (int f = 0; f < d.F; ++f) {
    frame_sets(f, d.F, d.T, d.C, d.L, &cur);
    if (f > 0 && !same_sets(cur, prev)) {
      n += ((int64_t)f * d.T - lo + TILE_M - 1) / TILE_M;
      lo = (int64_t)f * d.T;
    }
    prev = cur;
  }
  n += (d.Nv() - lo + TILE_M - 1) / TILE_M;
  return (int)n;
}

// tables + tile list into the workspace (device kernel, one block)
cudaError_t launch_tables(const Dims &d, char *ws, const WsPlan &p, cudaStream_t st);

cudaError_t launch_softmax_simt(const Dims &d, vdn_dtype dt, const void *q, const void *k, const void *v,
                                const void *kt, const void *vt, float scale_log2, void *o, float *lse,
                                char *ws, const WsPlan &p, cudaStream_t st);
cudaError_t launch_softmax_tc(const Dims &d, vdn_dtype dt, const void *q, const void *k, const void *v,
                              const void *kt, const void *vt, const float *scales, float scale_log2, void *o,
                              float *lse, char *ws, const WsPlan &p, cudaStream_t st);
bool softmax_tc_supported(const Dims &d, vdn_dtype dt);

// amax (delta rule, bf16, D = 128 only): also the per-head max |k|, |v| of the video and text
// rows, atomicMax'ed into amax[H + h], amax[2H + h] (float bits; zeroed by the caller)
cudaError_t launch_state_build(const Dims &d, vdn_lin_kind kind, vdn_dtype dt, const void *k, const void *v,
                               const void *kt, const void *vt, float *S, float *z, float *St, float *zt,
                               cudaStream_t st, uint32_t *amax = nullptr);
cudaError_t launch_state_scan(const Dims &d, vdn_lin_kind kind, const float *S, const float *z, const float *St,
                              const float *zt, const float *beta, float *Sf, float *Sb, float *zf, float *zb,
                              char *ws, const WsPlan &p, cudaStream_t st);
// ELU1 memories of the fused layer: S_fwd + S_bwd in bf16 and z_fwd + z_bwd straight
// into the read staging buffers (segmented scan; needs at most SCAN_SEG_MAX segments)
cudaError_t launch_state_scan_sum(const Dims &d, const float *S, const float *z, const float *St, const float *zt,
                                  char *ws, const WsPlan &p, cudaStream_t st);
cudaError_t launch_linear_read(const Dims &d, vdn_lin_kind kind, vdn_dtype dt, const void *q, const float *Sf,
                               const float *Sb, const float *zf, const float *zb, void *o, char *ws,
                               const WsPlan &p, cudaStream_t st);
// tensor-core linear branch (bf16, D = 128)
bool linear_tc_supported(const Dims &d, vdn_dtype dt);
cudaError_t launch_state_build_tc(const Dims &d, const void *k, const void *v, const void *kt, const void *vt,
                                  float *S, float *z, float *St, float *zt, char *ws, const WsPlan &p,
                                  cudaStream_t st);
// sums the two memories of every group into the bf16 staging buffers (skipped when Sf is
// NULL: the segmented scan wrote them) and converts the gate weights to bf16
cudaError_t launch_read_stage(const Dims &d, vdn_lin_kind kind, const float *Sf, const float *Sb, const float *zf,
                              const float *zb, const float *wgl, int G_l, char *ws, const WsPlan &p,
                              cudaStream_t st);
// o_l (plain) or, with gate weights, A_l = g_l * gamma * RMSNorm(o_l) into the linear half of A
// a8_scale (fused only): A_l written as e4m3 codes in units of a8_scale[h]
cudaError_t launch_read_tc(const Dims &d, vdn_lin_kind kind, const void *q, void *out, const float *wgl, int G_l,
                           const float *gamma, float eps, char *ws, const WsPlan &p, cudaStream_t st,
                           const float *a8_scale = nullptr, uint32_t *amax_q = nullptr);  // amax_q: per-head max |q|
// a8: A_s written as e4m3 codes in units of the V scale (e4m3 softmax only)
cudaError_t launch_softmax_tc_gated(const Dims &d, vdn_dtype dt, const void *q, const void *k, const void *v,
                                    const void *kt, const void *vt, const float *scales, const float *w_gate_s,
                                    float sl2, void *a, char *ws, const WsPlan &p, cudaStream_t st, bool a8 = false);
// per-head e4m3 quantisation of q, k (+ text), v (+ text); scales float[3][H]
// Backward of the elu+1 linear branch (CUDA cores, fp32), launched stage by stage (the
// forward's scan runs between the state rebuild and the row stage).
enum LinBwdStage : int {
  LIN_BWD_STATE = 0,   // per-frame and text states S, z, St, zt in fp32
  LIN_BWD_ROWS = 1,    // per query row: dq, dnum, dden
  LIN_BWD_FRAMES = 2,  // per query frame: sum of phi(q)^T dnum and phi(q) dden (part, zpart)
  LIN_BWD_GROUPS = 3,  // per group: dN, dZ from the frame sums
  LIN_BWD_KEYS = 4,    // per key frame and the text: dk, dv, dkt, dvt
};
struct LinBwdArgs {
  Dims d;
  const void *q, *k, *v, *kt, *vt;  // bf16 [rows][H][D]
  const float *dO;
  float *S, *z, *St, *zt;           // [F][H][D][D], [F][H][D], [H][D][D], [H][D]
  float *Sf, *Sb, *zf, *zb;         // group memories [G][H][D][D], [G][H][D]
  const int32_t *ftab, *gtab;
  int G;
  float *dnum, *dden;               // [Nv][H][D], [Nv][H]
  float *part, *zpart;              // [F][H][D][D], [F][H][D]
  float *dN, *dZ;                   // [G][H][D][D], [G][H][D]
  float *dq, *dk, *dv, *dkt, *dvt;
};
cudaError_t launch_linear_bwd(const LinBwdArgs &a, int stage, cudaStream_t st);
// Dynamic shared memory of the backward's key kernel: the D x D gradient and its transpose,
// two 64-row tiles, and one flag per group.
size_t linear_bwd_keys_smem(int D, int G);
constexpr size_t MAX_DYN_SMEM = 232448;  // per block, sm_100 (227 KB)
cudaError_t launch_fp8_quant(const Dims &d, const void *q, const void *k, const void *v, const void *kt,
                             const void *vt, void *q8, void *k8, void *v8, void *kt8, void *vt8, float *scales,
                             uint32_t *amax_bits, cudaStream_t st);
// the cast alone, with amax_bits already holding every head's max |q|, |k|, |v|
cudaError_t launch_fp8_cast(const Dims &d, const void *q, const void *k, const void *v, const void *kt,
                            const void *vt, void *q8, void *k8, void *v8, void *kt8, void *vt8, float *scales,
                            const uint32_t *amax_bits, cudaStream_t st);
constexpr int FP8_MAX_HD = 256 * 8 * 8;  // column chunks the amax pass keeps in registers

cudaError_t launch_fuse(const Dims &d, vdn_dtype dt, const void *q, const void *os, const void *ol,
                        const float *wgs, const float *wgl, int G_l, const float *gamma, float eps, void *a,
                        cudaStream_t st);
cudaError_t launch_out_proj_simt(const Dims &d, vdn_dtype dt, const void *a, const void *wos, const void *wol,
                                 void *y, cudaStream_t st);
// n_out > 0: W_os, W_ol [n_out][H D] (this call's heads' input columns of a wider
// projection) and y [N_v][n_out]; y_f32: float output (partial sums of the head split)
cudaError_t launch_out_proj_tc(const Dims &d, const void *a, const void *wos, const void *wol, void *y,
                               char *ws, const WsPlan &p, cudaStream_t st, int n_out = 0, bool y_f32 = false);
bool out_proj_tc_supported(const Dims &d);
// e4m3 projection: A8 [N_v][2HD] codes with dequantisation scales ascale[2][H] (per branch
// half and head), bf16 W_os, W_ol; w8 (HD x 2HD bytes) and wsc (HD floats) are scratch
bool out_proj_e4m3_supported(const Dims &d);
// halves: 1 the A_s scales (= the V scales), 2 the A_l scales (from gamma), 3 both
cudaError_t launch_a8_scales(const Dims &d, const float *vscale, const float *gamma, float *ascale, cudaStream_t st,
                             int halves = 3);
cudaError_t launch_out_proj_e4m3(const Dims &d, const void *a8, const float *ascale, const void *wos, const void *wol,
                                 void *y, uint8_t *w8, float *wsc, DevStatus *status, cudaStream_t st);
cudaError_t launch_debug_wait(char *ws, uint32_t max_polls, cudaStream_t st);

}  // namespace vdn
