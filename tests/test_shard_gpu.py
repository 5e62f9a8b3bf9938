"""GPU check of vdn_hybrid_attn_fwd_partial, the per-rank share of the layer split by heads:
on one GPU, the partial outputs of every rank's head slice (computed one after another,
with no rank waiting on another) summed on the device equal the whole layer's output and
the float64 oracle within the bf16 tolerance."""
import numpy as np
import pytest
import torch

import hybrid_softmax_linear_b200 as vdn
from hybrid_softmax_linear_b200 import shard, synth
from hybrid_softmax_linear_b200.tensors import to_device, to_numpy, workspace
from oracle import vdn_oracle as vo
from _harness import Run, assert_close, oracle_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,world,kind", [((13, 200, 5, 40, 4, 128), 2, vdn.ELU1),
                                              ((12, 96, 5, 24, 6, 128), 4, vdn.DELTA)])
def test_head_partials_sum_to_the_layer(shape, world, kind):
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    s = synth.Shape(*shape)
    inp = synth.make_inputs(s, "bf16", seed=23, with_beta=(kind == vdn.DELTA))
    full = to_numpy(Run(s, inp, "bf16", kind=kind).layer())
    HD = s.heads * s.head_dim
    y = torch.zeros((s.n_video, HD), dtype=torch.float32, device="cuda")
    for rank in range(world):
        h0, h1 = shard.head_range(s.heads, world, rank)
        part = {n: to_device(a) for n, a in shard.slice_inputs(inp, s.heads, s.head_dim, h0, h1).items()}
        sr = synth.Shape(s.frames, s.tokens_per_frame, s.chunk_frames, s.text_tokens, h1 - h0, s.head_dim)
        ws = workspace(vdn.hybrid_attn_workspace_size(sr, kind, vdn.BF16))
        vdn.workspace_init(ws)
        yp = torch.full((s.n_video, HD), float("nan"), dtype=torch.float32, device="cuda")
        vdn.hybrid_attn_fwd_partial(sr, HD, kind, vdn.BF16, part["q"], part["k"], part["v"], part["kt"], part["vt"],
                                    part.get("beta") if kind == vdn.DELTA else None, part["w_gate_s"],
                                    part["w_gate_l"], s.head_dim, part["gamma"], 1e-6, part["w_os"], part["w_ol"],
                                    yp, ws)
        vdn.check_device_status(ws)
        y += yp
    got = y.double().cpu().numpy()
    assert_close("sum of head partials vs whole layer", got, full, "bf16")
    ref = vo.layer(oracle_inputs(inp), s.frames, s.tokens_per_frame, s.chunk_frames,
                   linear="delta" if kind == vdn.DELTA else "elu1")["y"]
    assert_close("sum of head partials vs oracle", got, ref, "bf16")
