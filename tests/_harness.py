"""Shared helpers of the GPU parity tests: run the layer's entry points through the C
ABI on seeded inputs and compare with the float64 oracle."""
from __future__ import annotations

import functools

import numpy as np
import torch

import hybrid_softmax_linear_b200 as vdn
from hybrid_softmax_linear_b200 import synth
from hybrid_softmax_linear_b200.tensors import to_device, to_numpy, empty, workspace
from oracle import vdn_oracle as vo

# Tolerances fixed for this layer: fp32 rel-L2 <= 1e-5; bf16 rel-L2 <= 5e-3 and
# max-abs <= 3e-2; fp8 softmax rel-L2 <= 3e-2; layout bit-exact.
TOL = {"f32": (1e-5, None), "bf16": (5e-3, 3e-2), "e4m3": (3e-2, None)}


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    den = np.sqrt((b * b).sum())
    return float(np.sqrt(((a - b) ** 2).sum()) / (den if den > 0 else 1.0))


def max_abs(a, b) -> float:
    return float(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)).max())


def assert_close(name, got, ref, kind):
    rel, mab = TOL[kind]
    r = rel_l2(got, ref)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    assert r <= rel, f"{name}: rel-L2 {r:.3e} > {rel:.1e}"
    if mab is not None:
        m = max_abs(got, ref)
        assert m <= mab, f"{name}: max-abs {m:.3e} > {mab:.1e}"
    return r


def f64(x):
    return synth.to_f64(x) if x.dtype == np.uint16 else np.asarray(x, np.float64)


def f32view(x):
    """Exact float32 values of a stored input (bf16 bits widen exactly)."""
    return synth.bf16_bits_to_f32(x) if x.dtype == np.uint16 else np.asarray(x, np.float32)


class Run:
    """Device copies of one input set plus a workspace for the layer."""

    def __init__(self, shape: synth.Shape, inp: dict, dtype: str, kind: int = vdn.ELU1, G_l: int | None = None,
                 layer_dtype: int | None = None):
        self.shape, self.inp, self.dtype, self.kind = shape, inp, dtype, kind
        # dtype of the layer call (VDN_E4M3 runs the softmax branch in e4m3 on bf16 inputs)
        self.cdt = layer_dtype if layer_dtype is not None else (vdn.F32 if dtype == "f32" else vdn.BF16)
        self.dev = {n: to_device(a) for n, a in inp.items()}
        self.G_l = inp["w_gate_l"].shape[2] if G_l is None else G_l
        s = shape
        self.ws = workspace(vdn.hybrid_attn_workspace_size(s, kind, self.cdt))
        vdn.workspace_init(self.ws)
        self.Nv, self.H, self.D = s.n_video, s.heads, s.head_dim

    def layer(self):
        d = self.dev
        y = empty((self.Nv, self.H * self.D), self.dtype)
        vdn.hybrid_attn_fwd(self.shape, self.kind, self.cdt, d["q"], d["k"], d["v"], d["kt"], d["vt"],
                            d.get("beta") if self.kind == vdn.DELTA else None, d["w_gate_s"], d["w_gate_l"],
                            self.G_l, d["gamma"], 1e-6, d["w_os"], d["w_ol"], y, self.ws)
        vdn.check_device_status(self.ws)
        return y

    def materialises_branches(self) -> bool:
        """False on the fused tensor-core path, where O_s and O_l never reach memory."""
        return vdn.hybrid_attn_intermediate(self.shape, self.kind, self.cdt, self.ws, 0) != 0

    def intermediate(self, which, shape, tdtype):
        ptr = vdn.hybrid_attn_intermediate(self.shape, self.kind, self.cdt, self.ws, which)
        n = int(np.prod(shape))
        esz = torch.tensor([], dtype=tdtype).element_size()
        off = ptr - self.ws.data_ptr()   # view of the workspace slice at ptr
        assert 0 <= off and off + n * esz <= self.ws.numel()
        return self.ws[off:off + n * esz].view(tdtype).view(*shape)


@functools.lru_cache(maxsize=2)
def cfg_inputs(cfg: int):
    return synth.workload_inputs(cfg)


def oracle_inputs(inp: dict) -> dict:
    """float32 views (exact) of every stored input; the oracle widens to float64 itself."""
    return {n: f32view(a) for n, a in inp.items()}
