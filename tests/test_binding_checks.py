"""CPU tests of the Python binding's tensor checks on the whole-layer calls.

The library sees only addresses, so the binding checks each torch tensor's element count,
element size, contiguity and placement before passing its pointer.  The argument sets
below are built the way the GPU tests, the smoke run and the bench build theirs (the same
generators and conversions, on the host), so these checks cannot reject a call that the
GPU side makes."""
import numpy as np
import pytest
import torch

import hybrid_softmax_linear_b200 as vdn
from hybrid_softmax_linear_b200 import synth
from hybrid_softmax_linear_b200.tensors import to_torch


def _args(shape, dtype="bf16", kind=vdn.ELU1, gate_l_cols=None, host_bits=False):
    """The layer's tensors as the device call sites build them (to_torch of the generated
    arrays, y from torch.empty); host_bits: bf16 activations as int16 bit patterns, as the
    host-entry-point test passes them."""
    inp = synth.make_inputs(shape, dtype, seed=3, with_beta=kind == vdn.DELTA, gate_l_cols=gate_l_cols)
    t = {n: to_torch(a) for n, a in inp.items()}
    if host_bits:
        for n in ("q", "k", "v", "kt", "vt"):
            t[n] = torch.from_numpy(inp[n].view(np.int16))
    tdt = torch.float32 if dtype == "f32" else (torch.int16 if host_bits else torch.bfloat16)
    y = torch.empty((shape.n_video, shape.hidden), dtype=tdt)
    return dict(q=t["q"], k=t["k"], v=t["v"], kt=t["kt"], vt=t["vt"], beta=t.get("beta"), w_gate_s=t["w_gate_s"],
                w_gate_l=t["w_gate_l"], G_l=inp["w_gate_l"].shape[2], gamma=t["gamma"], w_os=t["w_os"],
                w_ol=t["w_ol"], y=y)


def _run(shape, cdt, a, io=None, weights=None):
    vdn._check_layer_args(shape, cdt, a["q"], a["k"], a["v"], a["kt"], a["vt"], a["beta"], a["w_gate_s"],
                          a["w_gate_l"], a["G_l"], a["gamma"], a["w_os"], a["w_ol"], a["y"], io, weights)


CASES = [
    # shape, input dtype, layer dtype, kind, gate columns
    (synth.Shape(12, 64, 5, 16, 2, 128), "bf16", vdn.BF16, vdn.ELU1, None),    # smoke
    (synth.Shape(12, 300, 5, 40, 2, 128), "bf16", vdn.E4M3, vdn.DELTA, None),
    (synth.Shape(12, 300, 5, 40, 2, 128), "bf16", vdn.BF16, vdn.DELTA, 1),     # scalar gate
    (synth.Shape(20, 100, 5, 0, 2, 128), "bf16", vdn.BF16, vdn.ELU1, None),    # no text
    (synth.Shape(2, 70, 5, 0, 1, 64), "f32", vdn.F32, vdn.ELU1, None),
    (synth.Shape(9, 17, 1, 2, 2, 32), "f32", vdn.F32, vdn.ELU1, None),
]


@pytest.mark.parametrize("shape,dtype,cdt,kind,cols", CASES)
def test_call_site_arguments_pass(shape, dtype, cdt, kind, cols):
    _run(shape, cdt, _args(shape, dtype, kind, cols))
    if dtype == "bf16":
        _run(shape, cdt, _args(shape, dtype, kind, cols, host_bits=True))


def test_placement_is_checked_before_any_library_call():
    s = synth.Shape(12, 64, 5, 16, 2, 128)
    a = _args(s)
    call = [s, vdn.ELU1, vdn.BF16, a["q"], a["k"], a["v"], a["kt"], a["vt"], None, a["w_gate_s"], a["w_gate_l"],
            a["G_l"], a["gamma"], 1e-6, a["w_os"], a["w_ol"], a["y"], 0]
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        vdn.hybrid_attn_fwd(*call)
    # host entry point: the per-call tensors may sit in host memory, the weights may not
    with pytest.raises(ValueError, match="w_gate_s must be a CUDA tensor"):
        vdn.hybrid_attn_fwd_host(*call)


@pytest.mark.parametrize("fault", ["short", "long", "strided", "esize", "beta", "gate_cols", "y"])
def test_bad_tensors_are_rejected(fault):
    s = synth.Shape(12, 300, 5, 40, 2, 128)
    a = _args(s, kind=vdn.DELTA)
    if fault == "short":
        a["k"] = a["k"].reshape(-1)[:-1]
    elif fault == "long":
        a["vt"] = torch.cat([a["vt"].reshape(-1), a["vt"].reshape(-1)[:8]])
    elif fault == "strided":
        a["q"] = torch.empty((a["q"].shape[0], a["q"].shape[1], 2 * a["q"].shape[2]), dtype=a["q"].dtype)[..., ::2]
    elif fault == "esize":
        a["v"] = a["v"].float()
    elif fault == "beta":
        a["beta"] = a["beta"].double()
    elif fault == "gate_cols":
        a["G_l"] = 1          # w_gate_l still holds D columns
    elif fault == "y":
        a["y"] = a["y"][:-1]
    with pytest.raises(ValueError):
        _run(s, vdn.BF16, a)


def test_raw_pointers_and_none_pass_through():
    s = synth.Shape(12, 64, 5, 16, 2, 128)
    a = {n: 1 << 20 for n in ("q", "k", "v", "kt", "vt", "w_gate_s", "w_gate_l", "gamma", "w_os", "w_ol", "y")}
    a.update(beta=None, G_l=128)
    _run(s, vdn.BF16, a, "device", "device")
