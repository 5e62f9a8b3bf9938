"""Python binding of libvdn, the sm_100a implementation of the VDN-H3 hybrid attention
layer (forward).  Argument marshalling only: every step runs in the library's CUDA
kernels; torch is used for device memory and streams.

The functions carry the C entry points' names without the ``vdn_`` prefix and accept
torch tensors (their ``data_ptr()`` is passed) or raw integer device pointers.  A
non-zero status raises :class:`VdnError` with the library's message.  If libvdn.so is
missing, :func:`lib` raises: there is no fallback path.  The whole-layer calls check each
torch tensor's element count, element size, contiguity and placement first and raise
ValueError on a mismatch.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = [
    "VdnError", "Shape", "lib", "F32", "BF16", "E4M3", "E4M3_PROJ", "ELU1", "DELTA",
    "mask_layout_build", "max_groups", "hybrid_attn_workspace_size", "step_workspace_size", "workspace_init",
    "softmax_branch_fwd", "linear_state_build", "linear_state_scan", "linear_read", "hybrid_fuse", "out_proj",
    "hybrid_attn_fwd", "hybrid_attn_host_workspace_size", "hybrid_attn_fwd_host", "hybrid_attn_intermediate", "check_device_status", "debug_unset_flag_wait", "version",
    "profile_begin", "profile_end", "fp8_quant_per_head", "softmax_branch_fwd_noalloc",
    "out_proj_e4m3", "out_proj_e4m3_workspace_size", "hybrid_attn_fwd_partial",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvdn.so")

F32, BF16, E4M3, E4M3_PROJ = 0, 1, 2, 3
ELU1, DELTA = 0, 1
STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA", 5: "TIMEOUT", 6: "DEVICE"}


class VdnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"vdn status {status} ({STATUS.get(status, '?')}): {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("frames", ctypes.c_int32), ("tokens_per_frame", ctypes.c_int32), ("chunk_frames", ctypes.c_int32),
                ("text_tokens", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]

    @classmethod
    def of(cls, s) -> "Shape":
        if isinstance(s, Shape):
            return s
        return cls(s.frames, s.tokens_per_frame, s.chunk_frames, s.text_tokens, s.heads, s.head_dim)


_lib = None
_vp, _sz, _i32, _f32, _u32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_float, ctypes.c_uint32
_SP = ctypes.POINTER(Shape)

_SIGS = {
    "vdn_version": (ctypes.c_int, []),
    "vdn_last_error": (ctypes.c_char_p, []),
    "vdn_mask_layout_build": (ctypes.c_int, [_SP, _vp, _vp, _vp, _sz]),
    "vdn_max_groups": (_i32, [_SP]),
    "vdn_hybrid_attn_workspace_size": (_sz, [_SP, ctypes.c_int, ctypes.c_int]),
    "vdn_step_workspace_size": (_sz, [_SP]),
    "vdn_workspace_init": (ctypes.c_int, [_vp, _sz, _vp]),
    "vdn_softmax_branch_fwd": (ctypes.c_int, [_SP, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp, _vp,
                                              _sz, _vp]),
    "vdn_linear_state_build": (ctypes.c_int, [_SP, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                              _vp, _vp, _sz, _vp]),
    "vdn_linear_state_scan": (ctypes.c_int, [_SP, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                             _sz, _vp]),
    "vdn_linear_read": (ctypes.c_int, [_SP, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                       _vp]),
    "vdn_linear_branch_bwd_workspace_size": (_sz, [_SP]),
    "vdn_linear_branch_bwd": (ctypes.c_int, [_SP, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                             _vp, _vp, _vp, _vp, _sz, _vp]),
    "vdn_hybrid_fuse": (ctypes.c_int, [_SP, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _f32, _vp, _vp]),
    "vdn_out_proj": (ctypes.c_int, [_SP, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "vdn_out_proj_e4m3_workspace_size": (_sz, [_SP]),
    "vdn_out_proj_e4m3": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "vdn_hybrid_attn_fwd": (ctypes.c_int, [_SP, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                           _i32, _vp, _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "vdn_hybrid_attn_fwd_partial": (ctypes.c_int, [_SP, _i32, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp,
                                                   _vp, _vp, _vp, _i32, _vp, _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "vdn_hybrid_attn_host_workspace_size": (_sz, [_SP, ctypes.c_int, ctypes.c_int]),
    "vdn_hybrid_attn_fwd_host": (ctypes.c_int, [_SP, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                _vp, _i32, _vp, _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "vdn_hybrid_attn_intermediate": (_vp, [_SP, ctypes.c_int, ctypes.c_int, _vp, ctypes.c_int]),
    "vdn_check_device_status": (ctypes.c_int, [_vp, _sz, _vp]),
    "vdn_debug_unset_flag_wait": (ctypes.c_int, [_vp, _sz, _u32, _vp]),
    "vdn_softmax_branch_fwd_noalloc": (ctypes.c_int, [_SP, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp,
                                                      _vp]),
    "vdn_fp8_quant_per_head": (ctypes.c_int, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                              _vp]),
    "vdn_profile_begin": (ctypes.c_int, [_i32]),
    "vdn_profile_end": (ctypes.c_int, [_vp, _vp, _i32]),
}

PROF_KERNELS = 20
KERNEL_NAMES = {1: "tables", 2: "softmax_simt", 3: "softmax_tc", 4: "state_build", 5: "scan", 6: "read", 7: "fuse",
                8: "out_proj_simt", 9: "out_proj_tc", 10: "fp8_quant", 11: "delta_stats", 13: "state_build_tc",
                14: "read_stage", 15: "read_tc", 16: "lin_bwd_rows", 17: "lin_bwd_frames", 18: "lin_bwd_keys",
                19: "lin_bwd_groups"}


def lib() -> ctypes.CDLL:
    """The loaded libvdn.so (built in-tree by ``python -m hybrid_softmax_linear_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libvdn.so not found at {LIB_PATH}; build it with "
                               "`python -m hybrid_softmax_linear_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def _p(x):
    """Device pointer of a tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _nbytes(ws):
    return ws.numel() * ws.element_size()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != 0:
        raise VdnError(status, lib().vdn_last_error().decode(errors="replace"))


def version() -> int:
    return lib().vdn_version()


def max_groups(shape) -> int:
    return lib().vdn_max_groups(ctypes.byref(Shape.of(shape)))


def mask_layout_build(shape, cap: int | None = None):
    """(frame_tab int32[F, 8], group_tab int32[G, 16]) from the host layout builder."""
    s = Shape.of(shape)
    cap = max_groups(s) if cap is None else cap
    ftab = np.zeros((s.frames, 8), np.int32)
    gtab = np.zeros((max(cap, 1), 16), np.int32)
    G = ctypes.c_int32(0)
    _check(lib().vdn_mask_layout_build(ctypes.byref(s), ftab.ctypes.data, gtab.ctypes.data, ctypes.byref(G), cap))
    return ftab, gtab[:G.value].copy()


def hybrid_attn_workspace_size(shape, kind: int, dtype: int) -> int:
    return lib().vdn_hybrid_attn_workspace_size(ctypes.byref(Shape.of(shape)), kind, dtype)


def step_workspace_size(shape) -> int:
    return lib().vdn_step_workspace_size(ctypes.byref(Shape.of(shape)))


def workspace_init(ws, stream=None):
    _check(lib().vdn_workspace_init(_p(ws), _nbytes(ws), _stream(stream)))


def softmax_branch_fwd(shape, dtype, q, k, v, kt, vt, o_s, ws, scales=None, sm_scale=0.0, lse=None, stream=None):
    _check(lib().vdn_softmax_branch_fwd(ctypes.byref(Shape.of(shape)), dtype, _p(q), _p(k), _p(v), _p(kt), _p(vt),
                                        _p(scales), sm_scale, _p(o_s), _p(lse), _p(ws), _nbytes(ws),
                                        _stream(stream)))


def softmax_branch_fwd_noalloc(shape, dtype, q, k, v, kt, vt, o_s, sm_scale=0.0, lse=None, stream=None):
    """Softmax branch without a workspace: the library's fixed device scratch array is
    used instead (for callers that cannot allocate device memory)."""
    _check(lib().vdn_softmax_branch_fwd_noalloc(ctypes.byref(Shape.of(shape)), dtype, _p(q), _p(k), _p(v), _p(kt),
                                                _p(vt), sm_scale, _p(o_s), _p(lse), _stream(stream)))


def fp8_quant_per_head(shape, q, k, v, kt, vt, q8, k8, v8, kt8, vt8, scales, ws, stream=None):
    """Per-head e4m3 copies of q, k (+ kt), v (+ vt) and their float[3][H] scales."""
    _check(lib().vdn_fp8_quant_per_head(ctypes.byref(Shape.of(shape)), _p(q), _p(k), _p(v), _p(kt), _p(vt), _p(q8),
                                        _p(k8), _p(v8), _p(kt8), _p(vt8), _p(scales), _p(ws), _nbytes(ws),
                                        _stream(stream)))


def linear_state_build(shape, kind, dtype, k, v, kt, vt, S, z, S_txt, z_txt, ws, stream=None):
    _check(lib().vdn_linear_state_build(ctypes.byref(Shape.of(shape)), kind, dtype, _p(k), _p(v), _p(kt), _p(vt),
                                        _p(S), _p(z), _p(S_txt), _p(z_txt), _p(ws), _nbytes(ws), _stream(stream)))


def linear_state_scan(shape, kind, S, z, S_txt, z_txt, beta, S_fwd, S_bwd, z_fwd, z_bwd, ws, stream=None):
    _check(lib().vdn_linear_state_scan(ctypes.byref(Shape.of(shape)), kind, _p(S), _p(z), _p(S_txt), _p(z_txt),
                                       _p(beta), _p(S_fwd), _p(S_bwd), _p(z_fwd), _p(z_bwd), _p(ws), _nbytes(ws),
                                       _stream(stream)))


def linear_read(shape, kind, dtype, q, S_fwd, S_bwd, z_fwd, z_bwd, o_l, ws, stream=None):
    _check(lib().vdn_linear_read(ctypes.byref(Shape.of(shape)), kind, dtype, _p(q), _p(S_fwd), _p(S_bwd),
                                 _p(z_fwd), _p(z_bwd), _p(o_l), _p(ws), _nbytes(ws), _stream(stream)))


def linear_branch_bwd_workspace_size(shape) -> int:
    return lib().vdn_linear_branch_bwd_workspace_size(ctypes.byref(Shape.of(shape)))


def linear_branch_bwd(shape, kind, dtype, q, k, v, kt, vt, do_l, dq, dk, dv, dkt, dvt, ws, stream=None):
    """Gradients of sum(o_l * do_l) of the elu+1 linear branch with respect to q, k, v, kt, vt
    (fp32 outputs; see vdn_linear_branch_bwd in include/vdn.h)."""
    _check(lib().vdn_linear_branch_bwd(ctypes.byref(Shape.of(shape)), kind, dtype, _p(q), _p(k), _p(v), _p(kt),
                                       _p(vt), _p(do_l), _p(dq), _p(dk), _p(dv), _p(dkt), _p(dvt), _p(ws),
                                       _nbytes(ws), _stream(stream)))


def hybrid_fuse(shape, dtype, q, o_s, o_l, w_gate_s, w_gate_l, G_l, gamma, eps, a, stream=None):
    _check(lib().vdn_hybrid_fuse(ctypes.byref(Shape.of(shape)), dtype, _p(q), _p(o_s), _p(o_l), _p(w_gate_s),
                                 _p(w_gate_l), G_l, _p(gamma), eps, _p(a), _stream(stream)))


def out_proj(shape, dtype, a, w_os, w_ol, y, ws, stream=None):
    _check(lib().vdn_out_proj(ctypes.byref(Shape.of(shape)), dtype, _p(a), _p(w_os), _p(w_ol), _p(y), _p(ws),
                              _nbytes(ws), _stream(stream)))


def out_proj_e4m3_workspace_size(shape) -> int:
    return lib().vdn_out_proj_e4m3_workspace_size(ctypes.byref(Shape.of(shape)))


def out_proj_e4m3(shape, a8, a_scales, w_os, w_ol, y, ws, stream=None):
    """y = A W_os^T + A W_ol^T from e4m3 A codes (uint8 [N_v][2HD]) with per-(branch half,
    head) scales a_scales float[2][H]; bf16 weights and y."""
    _check(lib().vdn_out_proj_e4m3(ctypes.byref(Shape.of(shape)), _p(a8), _p(a_scales), _p(w_os), _p(w_ol), _p(y),
                                   _p(ws), _nbytes(ws), _stream(stream)))


def _need(name: str, t, numel: int, esize: int, where: str | None):
    """Checks a torch tensor argument of the whole-layer calls before its pointer is passed:
    the library sees only addresses, so a short or strided buffer would be read or written
    out of bounds.  Raw integer pointers and None go through unchecked (the library checks
    for NULL).  where: "device", "host" or None (no placement check)."""
    if t is None or isinstance(t, int):
        return
    if where == "device" and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if where == "host" and t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.element_size() != esize:
        raise ValueError(f"{name}: {esize}-byte elements expected, got {t.dtype}")
    if t.numel() != numel:
        raise ValueError(f"{name}: {numel} elements expected, got {t.numel()}")


def _check_layer_args(shape, dtype, q, k, v, kt, vt, beta, w_gate_s, w_gate_l, G_l, gamma, w_os, w_ol, y,
                      io: str | None, weights: str | None):
    """Element counts and sizes of the layer's tensors (vdn.h, whole layer): q, k, v, y
    [N_v][H][D], kt, vt [L][H][D] and w_os, w_ol [HD][HD] in float (VDN_F32) or bf16; beta
    float[F][H]; w_gate_s, gamma float[H][D]; w_gate_l float[H][D][G_l].  io places the
    per-call tensors, weights the weights."""
    s = Shape.of(shape)
    nv, hd = s.frames * s.tokens_per_frame, s.heads * s.head_dim
    act = 4 if dtype == F32 else 2
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(name, t, nv * hd, act, io)
    for name, t in (("kt", kt), ("vt", vt)):
        _need(name, t, s.text_tokens * hd, act, io)
    _need("beta", beta, s.frames * s.heads, 4, io)
    _need("y", y, nv * hd, act, io)
    _need("w_gate_s", w_gate_s, hd, 4, weights)
    if isinstance(G_l, int) and G_l > 0:
        _need("w_gate_l", w_gate_l, hd * G_l, 4, weights)
    _need("gamma", gamma, hd, 4, weights)
    _need("w_os", w_os, hd * hd, act, weights)
    _need("w_ol", w_ol, hd * hd, act, weights)


def hybrid_attn_fwd(shape, kind, dtype, q, k, v, kt, vt, beta, w_gate_s, w_gate_l, G_l, gamma, eps, w_os, w_ol, y,
                    ws, stream=None):
    _check_layer_args(shape, dtype, q, k, v, kt, vt, beta, w_gate_s, w_gate_l, G_l, gamma, w_os, w_ol, y,
                      "device", "device")
    _check(lib().vdn_hybrid_attn_fwd(ctypes.byref(Shape.of(shape)), kind, dtype, _p(q), _p(k), _p(v), _p(kt),
                                     _p(vt), _p(beta), _p(w_gate_s), _p(w_gate_l), G_l, _p(gamma), eps, _p(w_os),
                                     _p(w_ol), _p(y), _p(ws), _nbytes(ws), _stream(stream)))


def hybrid_attn_fwd_partial(shape, out_features, kind, dtype, q, k, v, kt, vt, beta, w_gate_s, w_gate_l, G_l, gamma,
                            eps, w_os, w_ol, y_partial, ws, stream=None):
    """One rank's share of the head-split layer: shape.heads = this rank's heads, inputs are
    their slices, w_os/w_ol [out_features][H_r D] bf16, y_partial float [N_v][out_features]."""
    s = Shape.of(shape)
    nv, hd = s.frames * s.tokens_per_frame, s.heads * s.head_dim
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(name, t, nv * hd, 2, "device")
    for name, t in (("kt", kt), ("vt", vt)):
        _need(name, t, s.text_tokens * hd, 2, "device")
    _need("beta", beta, s.frames * s.heads, 4, "device")
    _need("w_gate_s", w_gate_s, hd, 4, "device")
    if isinstance(G_l, int) and G_l > 0:
        _need("w_gate_l", w_gate_l, hd * G_l, 4, "device")
    _need("gamma", gamma, hd, 4, "device")
    _need("w_os", w_os, out_features * hd, 2, "device")
    _need("w_ol", w_ol, out_features * hd, 2, "device")
    _need("y_partial", y_partial, nv * out_features, 4, "device")
    _check(lib().vdn_hybrid_attn_fwd_partial(ctypes.byref(s), out_features, kind, dtype, _p(q), _p(k), _p(v), _p(kt),
                                             _p(vt), _p(beta), _p(w_gate_s), _p(w_gate_l), G_l, _p(gamma), eps,
                                             _p(w_os), _p(w_ol), _p(y_partial), _p(ws), _nbytes(ws),
                                             _stream(stream)))


def hybrid_attn_host_workspace_size(shape, kind: int, dtype: int) -> int:
    return lib().vdn_hybrid_attn_host_workspace_size(ctypes.byref(Shape.of(shape)), kind, dtype)


def hybrid_attn_fwd_host(shape, kind, dtype, q, k, v, kt, vt, beta, w_gate_s, w_gate_l, G_l, gamma, eps, w_os,
                         w_ol, y, ws, stream=None):
    """The layer with q, k, v, kt, vt, beta and y in (page-locked) host memory; weights on
    the device.  Asynchronous on `stream`: y is complete when the stream is."""
    _check_layer_args(shape, dtype, q, k, v, kt, vt, beta, w_gate_s, w_gate_l, G_l, gamma, w_os, w_ol, y,
                      "host", "device")
    _check(lib().vdn_hybrid_attn_fwd_host(ctypes.byref(Shape.of(shape)), kind, dtype, _p(q), _p(k), _p(v), _p(kt),
                                          _p(vt), _p(beta), _p(w_gate_s), _p(w_gate_l), G_l, _p(gamma), eps,
                                          _p(w_os), _p(w_ol), _p(y), _p(ws), _nbytes(ws), _stream(stream)))


def hybrid_attn_intermediate(shape, kind, dtype, ws, which: int) -> int:
    """Device address of an intermediate inside ws (0 O_s, 1 O_l, 2 A, 3 S_fwd, 4 S_bwd)."""
    return lib().vdn_hybrid_attn_intermediate(ctypes.byref(Shape.of(shape)), kind, dtype, _p(ws), which) or 0


def check_device_status(ws, stream=None):
    _check(lib().vdn_check_device_status(_p(ws), _nbytes(ws), _stream(stream)))


def profile_begin(max_launches: int = 4096):
    """Start per-kernel CUDA-event timing of the entry points' launches."""
    _check(lib().vdn_profile_begin(max_launches))


def profile_end() -> dict:
    """{kernel name: (total ms, launches)} of the launches recorded since profile_begin."""
    ms = (ctypes.c_float * PROF_KERNELS)()
    n = (ctypes.c_int32 * PROF_KERNELS)()
    _check(lib().vdn_profile_end(ms, n, PROF_KERNELS))
    return {KERNEL_NAMES.get(k, str(k)): (float(ms[k]), int(n[k])) for k in range(PROF_KERNELS) if n[k] > 0}


def debug_unset_flag_wait(ws, max_polls: int, stream=None):
    _check(lib().vdn_debug_unset_flag_wait(_p(ws), _nbytes(ws), max_polls, _stream(stream)))
