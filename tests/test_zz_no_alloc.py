"""GPU check of vdn_softmax_branch_fwd_noalloc, the softmax-branch entry point for
callers that cannot allocate device memory (for example a plug-in that only receives
tensors from a host framework that owns all device memory): it keeps its scratch in the
library's fixed device array instead of a caller workspace.

Its output must match vdn_softmax_branch_fwd (the workspace entry point) within the
tolerances used throughout the tests, on two calls in a row, so the second call is
not disturbed by what the first left in the shared array.  This file is collected last
and passes both alone in a fresh process and after the other tests."""
import numpy as np
import pytest
import torch

import hybrid_softmax_linear_b200 as vdn
from hybrid_softmax_linear_b200 import synth
from hybrid_softmax_linear_b200.tensors import to_device, to_numpy, empty, workspace
from _harness import assert_close

pytestmark = pytest.mark.gpu

CASES = [
    # F, T, C, L, H, D, dtype: tensor-core path (bf16, D = 64 and 128) and CUDA-core path (f32)
    (30, 256, 5, 64, 8, 64, "bf16"),
    (20, 100, 5, 130, 3, 128, "bf16"),
    (15, 16, 1, 4, 2, 32, "f32"),
]


def _setup(case, seed):
    F, T, C, L, H, D, dt = case
    s = synth.Shape(F, T, C, L, H, D)
    inp = synth.make_inputs(s, dt, seed=seed)
    return s, {n: to_device(a) for n, a in inp.items()}


def _workspace_reference(s, dt, d):
    cdt = vdn.F32 if dt == "f32" else vdn.BF16
    ws = workspace(vdn.step_workspace_size(s))
    vdn.workspace_init(ws)
    ref = empty((s.n_video, s.heads, s.head_dim), dt)
    ref_lse = torch.empty((s.n_video, s.heads), dtype=torch.float32, device="cuda")
    vdn.softmax_branch_fwd(s, cdt, d["q"], d["k"], d["v"], d["kt"], d["vt"], ref, ws, lse=ref_lse)
    vdn.check_device_status(ws)
    return to_numpy(ref), ref_lse.cpu().numpy(), ref.dtype


def _noalloc_call(s, dt, d, out_dtype):
    cdt = vdn.F32 if dt == "f32" else vdn.BF16
    out = torch.full((s.n_video, s.heads, s.head_dim), float("nan"), dtype=out_dtype, device="cuda")
    lse = torch.full((s.n_video, s.heads), float("nan"), dtype=torch.float32, device="cuda")
    vdn.softmax_branch_fwd_noalloc(s, cdt, d["q"], d["k"], d["v"], d["kt"], d["vt"], out, lse=lse)
    torch.cuda.synchronize()
    return to_numpy(out), lse.cpu().numpy()


@pytest.mark.parametrize("case", CASES)
def test_noalloc_matches_workspace_entry_point_twice(case):
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    dt = case[-1]
    s, d = _setup(case, 77 + case[0])
    ref_np, ref_lse_np, odt = _workspace_reference(s, dt, d)
    for call in range(2):
        out, lse = _noalloc_call(s, dt, d, odt)
        assert_close(f"no-alloc output, call {call + 1}", out, ref_np, "f32" if dt == "f32" else "bf16")
        np.testing.assert_allclose(lse, ref_lse_np, rtol=1e-5, atol=1e-5)


def test_noalloc_after_a_larger_call_with_other_tables():
    # the shared array keeps the previous call's tables and tile list: a smaller shape with
    # another frame count, chunk size and text length must not read any of them
    big = (40, 300, 4, 70, 4, 128, "bf16")
    small = (11, 130, 3, 9, 3, 128, "bf16")
    s_big, d_big = _setup(big, 5)
    s_small, d_small = _setup(small, 6)
    ref_np, ref_lse_np, odt = _workspace_reference(s_small, "bf16", d_small)
    _noalloc_call(s_big, "bf16", d_big, odt)
    out, lse = _noalloc_call(s_small, "bf16", d_small, odt)
    assert_close("no-alloc output after a larger call", out, ref_np, "bf16")
    np.testing.assert_allclose(lse, ref_lse_np, rtol=1e-5, atol=1e-5)


def test_noalloc_at_the_size_limit():
    # 2604 frames of 256 tokens in 5-frame chunks is the largest frame count whose tables and
    # query-tile list fit the 256 KiB array (2605 is rejected, see tests/test_abi_cpu.py)
    case = (2604, 256, 5, 16, 1, 64, "bf16")
    s, d = _setup(case, 8)
    ref_np, ref_lse_np, odt = _workspace_reference(s, "bf16", d)
    out, lse = _noalloc_call(s, "bf16", d, odt)
    assert_close("no-alloc output at the size limit", out, ref_np, "bf16")
    np.testing.assert_allclose(lse, ref_lse_np, rtol=1e-5, atol=1e-5)


def test_noalloc_rejects_shapes_beyond_the_fixed_scratch():
    # 2^26 video tokens need about 262k query tiles: far more than the 256 KiB array holds
    s = synth.Shape(4096, 16384, 5, 0, 1, 64)
    with pytest.raises(vdn.VdnError) as e:
        vdn.softmax_branch_fwd_noalloc(s, vdn.BF16, 16, 16, 16, None, None, 16)
    assert e.value.status == 3
    assert "256 KiB" in str(e.value)
