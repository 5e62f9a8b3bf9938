"""Stand-in for a device memory checker (compute-sanitizer is closed on this machine): reads
of scratch memory that no kernel wrote first.

Every byte of the workspace (and, for the host entry point, of its staging area) is
filled with 0xFF before the call: a NaN bit pattern in float32, bfloat16 and e4m3 alike.
Only the 256-byte status word is then cleared, as vdn_workspace_init documents.  The
library reduces in a fixed order, so the call on the poisoned workspace must give
exactly the bits of the same call on a zero-filled one: a kernel that read a scratch
byte before writing it would turn part of y into NaN or change its bits (a zero-filled
workspace, which a fresh torch allocation often is, hides such a read)."""
import numpy as np
import pytest
import torch

import hybrid_softmax_linear_b200 as vdn
from hybrid_softmax_linear_b200 import synth
from hybrid_softmax_linear_b200.tensors import to_device, empty, workspace

pytestmark = pytest.mark.gpu

CASES = [
    # name, shape (F, T, C, L, H, D), storage dtype, linear kind, layer dtype
    ("small D64 (CUDA-core linear branch)", (30, 256, 5, 64, 8, 64), "bf16", vdn.ELU1, vdn.BF16),
    ("D128 tensor-core path, ragged frames", (13, 200, 5, 40, 3, 128), "bf16", vdn.ELU1, vdn.BF16),
    ("no text, short last chunk", (7, 130, 3, 0, 2, 128), "bf16", vdn.ELU1, vdn.BF16),
    ("e4m3 softmax, delta rule", (12, 96, 5, 24, 2, 128), "bf16", vdn.DELTA, vdn.E4M3),
    ("fp32 CUDA cores", (15, 16, 1, 4, 2, 32), "f32", vdn.ELU1, vdn.F32),
    ("medium 60x1008, 24 heads", (60, 1008, 5, 256, 24, 128), "bf16", vdn.ELU1, vdn.BF16),
]


def _inputs(shape, dt, kind, seed):
    inp = synth.make_inputs(synth.Shape(*shape), dt, seed=seed, with_beta=(kind == vdn.DELTA))
    return {n: to_device(a) for n, a in inp.items()}


def _layer(s, kind, cdt, dt, d, ws, host=False):
    args = (d["q"], d["k"], d["v"], d["kt"], d["vt"], d.get("beta") if kind == vdn.DELTA else None)
    if host:
        args = tuple(None if a is None else a.cpu().pin_memory() for a in args)
        y = empty((s.n_video, s.heads * s.head_dim), dt, device="cpu").pin_memory()
        vdn.hybrid_attn_fwd_host(s, kind, cdt, *args, d["w_gate_s"], d["w_gate_l"], s.head_dim, d["gamma"], 1e-6,
                                 d["w_os"], d["w_ol"], y, ws)
    else:
        y = empty((s.n_video, s.heads * s.head_dim), dt)
        vdn.hybrid_attn_fwd(s, kind, cdt, *args, d["w_gate_s"], d["w_gate_l"], s.head_dim, d["gamma"], 1e-6,
                            d["w_os"], d["w_ol"], y, ws)
    torch.cuda.synchronize()
    vdn.check_device_status(ws)
    return y.cpu()


def _fresh(nbytes, fill):
    ws = workspace(nbytes)
    ws.fill_(fill)
    vdn.workspace_init(ws)      # clears the status word only
    return ws


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_layer_reads_no_unwritten_scratch(case):
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    _, shape, dt, kind, cdt = case
    s = synth.Shape(*shape)
    d = _inputs(shape, dt, kind, seed=99)
    n = vdn.hybrid_attn_workspace_size(s, kind, cdt)
    y0 = _layer(s, kind, cdt, dt, d, _fresh(n, 0))
    assert torch.isfinite(y0.float()).all()
    y1 = _layer(s, kind, cdt, dt, d, _fresh(n, 0xFF))
    assert torch.equal(y0.view(torch.int16 if dt == "bf16" else torch.int32),
                       y1.view(torch.int16 if dt == "bf16" else torch.int32)), \
        f"poisoned workspace changed {int((y0 != y1).sum())} of {y0.numel()} outputs"


@pytest.mark.parametrize("case", CASES[1:4], ids=[c[0] for c in CASES[1:4]])
def test_host_entry_point_reads_no_unwritten_staging(case):
    _, shape, dt, kind, cdt = case
    s = synth.Shape(*shape)
    d = _inputs(shape, dt, kind, seed=98)
    y0 = _layer(s, kind, cdt, dt, d, _fresh(vdn.hybrid_attn_workspace_size(s, kind, cdt), 0))
    y1 = _layer(s, kind, cdt, dt, d, _fresh(vdn.hybrid_attn_host_workspace_size(s, kind, cdt), 0xFF), host=True)
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


@pytest.mark.parametrize("shape", [(30, 256, 5, 64, 8, 64), (13, 200, 5, 40, 3, 128)])
def test_softmax_entry_point_reads_no_unwritten_scratch(shape):
    s = synth.Shape(*shape)
    d = _inputs(shape, "bf16", vdn.ELU1, seed=97)
    outs = []
    for fill in (0, 0xFF):
        ws = _fresh(vdn.step_workspace_size(s), fill)
        o = empty((s.n_video, s.heads, s.head_dim), "bf16")
        lse = torch.empty((s.n_video, s.heads), dtype=torch.float32, device="cuda")
        vdn.softmax_branch_fwd(s, vdn.BF16, d["q"], d["k"], d["v"], d["kt"], d["vt"], o, ws, lse=lse)
        vdn.check_device_status(ws)
        outs.append((o.cpu().view(torch.int16), lse.cpu()))
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])
