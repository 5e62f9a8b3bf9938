"""GPU checks of the e4m3 output projection (vdn_out_proj_e4m3 and the whole layer with
VDN_E4M3_PROJ); the model card's "Inference with Diffusers" runs every wide Linear in fp8
e4m3.

1. The projection alone against the same arithmetic written out on the host: A as e4m3
   codes with per-(branch half, head) scales, [W_os | W_ol] scaled by them in float32 and
   rounded to e4m3 with one scale per output column (amax / 448, round to nearest even,
   saturating), products summed in float64.  Only the summation order and y's bf16
   rounding differ, so the bf16 tolerance applies.  Against the exact float64 product of
   the unrounded operands the error is e4m3's own, held to the bound the CPU error model
   derives (tests/test_fp8_error_model.py).
2. The whole layer with the e4m3 softmax and e4m3 projection against the float64 oracle on
   the bf16 inputs, at the bound derived the same way for the layer."""
import numpy as np
import pytest
import torch

import hybrid_softmax_linear_b200 as vdn
from hybrid_softmax_linear_b200 import synth
from hybrid_softmax_linear_b200.tensors import to_device, to_numpy, workspace
from oracle import vdn_oracle as vo
from _harness import assert_close, rel_l2, oracle_inputs, cfg_inputs, Run
from test_fp8_error_model import PROJ_GPU_BOUND, LAYER_E4M3_BOUND

pytestmark = pytest.mark.gpu


def _e4m3_codes(x: torch.Tensor) -> torch.Tensor:
    """float32 -> e4m3 codes (uint8), round to nearest even, saturating at 448."""
    return x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def _e4m3_values(codes: torch.Tensor) -> torch.Tensor:
    return codes.view(torch.float8_e4m3fn).to(torch.float64)


def _host_weights(w_os, w_ol, ascale, D):
    """The weight copy as the library defines it: w' = W_cat * ascale[c / D] (float32), the
    column scale amax(w') / 448, codes e4m3(w' * (ascale / scale))."""
    wcat = torch.cat([w_os, w_ol], 1).float()                       # [HD, 2HD]
    sc = ascale.reshape(-1).repeat_interleave(D)                      # [2HD], per column of A
    wp = wcat * sc
    amax = wp.abs().amax(1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    inv = 1.0 / scale
    codes = _e4m3_codes(wcat * (sc[None, :] * inv[:, None]))
    return codes, scale


@pytest.mark.parametrize("shape", [(4, 500, 5, 0, 8, 128), (3, 700, 5, 0, 2, 128)])
def test_out_proj_e4m3_matches_host_arithmetic(shape):
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    s = synth.Shape(*shape)
    H, D, Nv = s.heads, s.head_dim, s.n_video
    HD = H * D
    g = torch.Generator().manual_seed(5)
    a = torch.randn(Nv, 2 * HD, generator=g)
    a[:, :HD] *= 0.3                                   # the softmax half is smaller
    ascale = torch.stack([a[:, :HD].reshape(Nv, H, D).abs().amax((0, 2)),
                          a[:, HD:].reshape(Nv, H, D).abs().amax((0, 2))]) / 448.0   # [2, H]
    a8 = _e4m3_codes(a / ascale.reshape(-1).repeat_interleave(D)[None, :])
    w_os = (torch.randn(HD, HD, generator=g) * 0.02).bfloat16()
    w_ol = (torch.randn(HD, HD, generator=g) * 0.02).bfloat16()
    y = torch.empty(Nv, HD, dtype=torch.bfloat16, device="cuda")
    ws = workspace(vdn.out_proj_e4m3_workspace_size(s))
    vdn.workspace_init(ws)
    vdn.out_proj_e4m3(s, a8.cuda(), ascale.float().contiguous().cuda(), w_os.cuda(), w_ol.cuda(), y, ws)
    vdn.check_device_status(ws)
    got = y.float().cpu().double().numpy()
    # the same arithmetic on the host
    w8, wsc = _host_weights(w_os, w_ol, ascale.float(), D)
    ref = (_e4m3_values(a8) @ _e4m3_values(w8).T) * wsc.double()[None, :]
    assert_close("e4m3 projection vs host arithmetic", got, ref.numpy(), "bf16")
    # and the exact product of the unrounded operands, within the e4m3 model bound
    exact = a.double() @ torch.cat([w_os, w_ol], 1).double().T
    err = rel_l2(got, exact.numpy())
    assert err < PROJ_GPU_BOUND, err


def test_out_proj_e4m3_rejects_unsupported_width():
    s = synth.Shape(2, 64, 5, 0, 1, 64)   # H*D = 64, not a multiple of 256
    ws = workspace(vdn.out_proj_e4m3_workspace_size(s))
    with pytest.raises(vdn.VdnError) as e:
        vdn.out_proj_e4m3(s, ws, ws, ws, ws, ws, ws)
    assert e.value.status == 2


def _layer_e4m3_proj(shape, inp, kind):
    s = shape
    run = Run(s, inp, "bf16", kind=kind, layer_dtype=vdn.E4M3_PROJ)
    return to_numpy(run.layer())


@pytest.mark.parametrize("kind", [vdn.ELU1, vdn.DELTA])
def test_layer_e4m3_projection_small(kind):
    s = synth.Shape(12, 96, 5, 24, 2, 128)
    inp = synth.make_inputs(s, "bf16", seed=41, with_beta=(kind == vdn.DELTA))
    got = _layer_e4m3_proj(s, inp, kind)
    ref = vo.layer(oracle_inputs(inp), s.frames, s.tokens_per_frame, s.chunk_frames,
                   linear="delta" if kind == vdn.DELTA else "elu1")["y"]
    err = rel_l2(got, ref)
    assert np.all(np.isfinite(got)) and err < LAYER_E4M3_BOUND, err


def test_config5_full_size_e4m3_projection_sampled():
    """Config 5 (e4m3 softmax, delta rule) with the e4m3 projection as well, on sampled rows."""
    w = synth.CONFIGS[5]
    s = w.shape
    inp = cfg_inputs(5)
    got = _layer_e4m3_proj(s, inp, vdn.DELTA)
    rows = synth.sample_rows(s)
    ref = vo.layer(oracle_inputs(inp), s.frames, s.tokens_per_frame, s.chunk_frames, rows=rows, linear="delta")["y"]
    err = rel_l2(got[rows], ref)
    assert np.all(np.isfinite(got)) and err < LAYER_E4M3_BOUND, err
