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


@pytest.mark.parametrize("case", CASES)
def test_noalloc_matches_workspace_entry_point_twice(case):
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    F, T, C, L, H, D, dt = case
    s = synth.Shape(F, T, C, L, H, D)
    cdt = vdn.F32 if dt == "f32" else vdn.BF16
    tol = "f32" if dt == "f32" else "bf16"
    inp = synth.make_inputs(s, dt, seed=77 + F)
    d = {n: to_device(a) for n, a in inp.items()}
    Nv = s.n_video

    ws = workspace(vdn.step_workspace_size(s))
    vdn.workspace_init(ws)
    ref = empty((Nv, H, D), dt)
    ref_lse = torch.empty((Nv, H), dtype=torch.float32, device="cuda")
    vdn.softmax_branch_fwd(s, cdt, d["q"], d["k"], d["v"], d["kt"], d["vt"], ref, ws, lse=ref_lse)
    vdn.check_device_status(ws)
    ref_np, ref_lse_np = to_numpy(ref), ref_lse.cpu().numpy()

    for call in range(2):
        out = torch.full((Nv, H, D), float("nan"), dtype=ref.dtype, device="cuda")
        lse = torch.full((Nv, H), float("nan"), dtype=torch.float32, device="cuda")
        vdn.softmax_branch_fwd_noalloc(s, cdt, d["q"], d["k"], d["v"], d["kt"], d["vt"], out, lse=lse)
        torch.cuda.synchronize()
        assert_close(f"no-alloc output, call {call + 1}", to_numpy(out), ref_np, tol)
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse_np, rtol=1e-5, atol=1e-5)


def test_noalloc_rejects_shapes_beyond_the_fixed_scratch():
    # 2^26 video tokens need about 262k query tiles: far more than the 256 KiB array holds
    s = synth.Shape(4096, 16384, 5, 0, 1, 64)
    with pytest.raises(vdn.VdnError) as e:
        vdn.softmax_branch_fwd_noalloc(s, vdn.BF16, 16, 16, 16, None, None, 16)
    assert e.value.status == 3
    assert "256 KiB" in str(e.value)
