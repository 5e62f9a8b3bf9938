"""CPU checks of the C ABI: the library loads without a GPU, exports every entry point
that include/vdn.h declares, builds layout tables identical to the oracle's, and rejects
bad arguments before touching CUDA."""
import ctypes
import os
import re

import numpy as np
import pytest

import hybrid_softmax_linear_b200 as vdn
from hybrid_softmax_linear_b200 import synth
from oracle import vdn_oracle as vo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "vdn.h"), encoding="utf-8").read()
    return sorted(set(re.findall(r"VDN_API[^;(]*?\b(vdn_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 17
    L = ctypes.CDLL(vdn.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(vdn._SIGS), "binding and header disagree"


def test_version():
    assert vdn.version() >= 100


SHAPES = [(15, 16, 1, 4, 2, 32), (30, 256, 5, 64, 8, 64), (60, 1008, 5, 256, 24, 128), (90, 1008, 5, 512, 40, 128),
          (87, 1008, 5, 512, 40, 128), (1, 4, 5, 3, 1, 32), (2, 5, 5, 0, 1, 32), (3, 7, 1, 0, 1, 64),
          (16, 1, 2, 1, 1, 32), (11, 100, 2, 0, 2, 64), (40, 3, 6, 9, 1, 32), (13, 5, 13, 2, 1, 32)]


@pytest.mark.parametrize("sh", SHAPES)
def test_layout_bit_exact_vs_oracle(sh):
    F, T, C, L, H, D = sh
    ftab, gtab = vdn.mask_layout_build(synth.Shape(F, T, C, L, H, D))
    oft, ogt = vo.layout_tables(F, T, C, L)
    np.testing.assert_array_equal(ftab, oft)
    np.testing.assert_array_equal(gtab, ogt)
    assert len(gtab) <= vdn.max_groups(synth.Shape(F, T, C, L, H, D))


def test_layout_all_small_shapes_vs_oracle():
    for F in range(1, 41):
        for C in range(1, 7):
            for T, L in ((1, 0), (3, 2)):
                ftab, gtab = vdn.mask_layout_build(synth.Shape(F, T, C, L, 1, 32))
                oft, ogt = vo.layout_tables(F, T, C, L)
                assert np.array_equal(ftab, oft) and np.array_equal(gtab, ogt), (F, C, T, L)


def test_layout_capacity_error():
    s = synth.Shape(90, 1008, 5, 512, 40, 128)
    with pytest.raises(vdn.VdnError) as e:
        vdn.mask_layout_build(s, cap=3)
    assert e.value.status == 1


@pytest.mark.parametrize("bad", [(0, 16, 1, 4, 2, 32), (15, 0, 1, 4, 2, 32), (15, 16, 0, 4, 2, 32),
                                 (15, 16, 1, -1, 2, 32), (15, 16, 1, 4, 0, 32)])
def test_bad_shape_rejected(bad):
    with pytest.raises(vdn.VdnError) as e:
        vdn.mask_layout_build(vdn.Shape(*bad), cap=64)
    assert e.value.status == 1


def test_unsupported_head_dim():
    with pytest.raises(vdn.VdnError) as e:
        vdn.mask_layout_build(vdn.Shape(15, 16, 1, 4, 2, 48), cap=64)
    assert e.value.status == 2


def test_workspace_sizes():
    s = synth.Shape(90, 1008, 5, 512, 40, 128)
    step = vdn.step_workspace_size(s)
    full = vdn.hybrid_attn_workspace_size(s, vdn.ELU1, vdn.BF16)
    assert 0 < step < full
    # the fused bf16 layer keeps A = [A_s | A_l] (bf16) plus per-frame and per-group fp32
    # states; O_s and O_l never reach memory, so the workspace stays below A + O_s + O_l
    nv, hd = 90 * 1008, 40 * 128
    assert nv * hd * 2 * 2 <= full < nv * hd * 2 * 4
    # the CUDA-core f32 path also stores O_s and O_l
    assert vdn.hybrid_attn_workspace_size(s, vdn.ELU1, vdn.F32) >= nv * hd * 4 * 4
    assert vdn.hybrid_attn_workspace_size(s, vdn.DELTA, vdn.E4M3) > 0


def test_argument_checks_precede_cuda():
    """Null pointers and small workspaces are reported without a device."""
    s = vdn.Shape(15, 16, 1, 4, 2, 32)
    L = vdn.lib()
    st = L.vdn_softmax_branch_fwd(ctypes.byref(s), vdn.F32, None, 16, 16, 16, 16, None, 0.0, 16, None, 256, 1 << 20,
                                  None)
    assert st == 1 and b"q" in L.vdn_last_error()
    st = L.vdn_softmax_branch_fwd(ctypes.byref(s), vdn.F32, 16, 16, 16, 16, 16, None, 0.0, 16, None, 256, 16, None)
    assert st == 3
    st = L.vdn_softmax_branch_fwd(ctypes.byref(s), vdn.F32, 16, 16, 16, 16, 16, None, 0.0, 16, None, 100, 1 << 20,
                                  None)
    assert st == 3  # misaligned workspace
    st = L.vdn_softmax_branch_fwd(ctypes.byref(s), vdn.F32, 24, 16, 16, 16, 16, None, 0.0, 16, None, 256, 1 << 20,
                                  None)
    assert st == 1  # misaligned q
    st = L.vdn_softmax_branch_fwd(ctypes.byref(s), vdn.F32, 16, 16, 16, 16, 16, 16, 0.0, 16, None, 256, 1 << 20, None)
    assert st == 1  # scales with a non-fp8 dtype
    st = L.vdn_hybrid_fuse(ctypes.byref(s), vdn.BF16, 16, 16, 16, 16, 16, 7, 16, 1e-6, 16, None)
    assert st == 1  # G_l not in {1, D}
    st = L.vdn_hybrid_attn_fwd(ctypes.byref(s), vdn.ELU1, vdn.F32, 16, 16, 16, 16, 16, 16, 16, 16, 32, 16, 1e-6, 16,
                               16, 16, 256, 1 << 30, None)
    assert st == 1  # beta given for ELU1
    st = L.vdn_hybrid_attn_fwd(ctypes.byref(s), 7, vdn.F32, 16, 16, 16, 16, 16, None, 16, 16, 32, 16, 1e-6, 16, 16,
                               16, 256, 1 << 30, None)
    assert st == 1  # unknown kind
    for polls in (0, 1000001, 0xFFFFFFFF):
        assert L.vdn_debug_unset_flag_wait(256, 1 << 20, polls, None) == 1  # the test wait stays short


def test_linear_branch_bwd_checks():
    """The backward of the linear branch: ELU1 and bf16 only, text pointers required when
    L > 0, workspace size reported without a device and checked before any launch."""
    s = vdn.Shape(12, 40, 5, 6, 2, 64)
    L = vdn.lib()
    need = L.vdn_linear_branch_bwd_workspace_size(ctypes.byref(s))
    assert need > 0 and need % 256 == 0
    assert L.vdn_linear_branch_bwd_workspace_size(ctypes.byref(vdn.Shape(0, 40, 5, 6, 2, 64))) == 0
    args = [16] * 11
    st = L.vdn_linear_branch_bwd(ctypes.byref(s), vdn.DELTA, vdn.BF16, *args, 256, need, None)
    assert st == 2  # delta rule: not built
    st = L.vdn_linear_branch_bwd(ctypes.byref(s), vdn.ELU1, vdn.F32, *args, 256, need, None)
    assert st == 2  # f32 inputs: not built
    st = L.vdn_linear_branch_bwd(ctypes.byref(s), vdn.ELU1, vdn.BF16, 16, 16, 16, None, 16, 16, 16, 16, 16, 16, 16,
                                 256, need, None)
    assert st == 1 and b"kt" in L.vdn_last_error()
    st = L.vdn_linear_branch_bwd(ctypes.byref(s), vdn.ELU1, vdn.BF16, *args, 256, need - 256, None)
    assert st == 3  # workspace too small
    # one-frame chunks give one group per frame; the key kernel's per-group flags overflow
    # its shared memory past 29184 groups at D = 128, refused before any device work
    big = vdn.Shape(30000, 1, 1, 0, 1, 128)
    st = L.vdn_linear_branch_bwd(ctypes.byref(big), vdn.ELU1, vdn.BF16, *args, 256, 1 << 40, None)
    assert st == 2 and b"groups" in L.vdn_last_error()


def test_noalloc_checks_match_the_workspace_entry_point():
    """The no-allocation softmax entry point rejects exactly what vdn_softmax_branch_fwd
    rejects, before any device work, and refuses shapes whose scratch exceeds its fixed
    256 KiB array (2604 frames of 256 tokens in 5-frame chunks fit, 2605 do not)."""
    L = vdn.lib()
    ok = vdn.Shape(15, 16, 1, 4, 2, 32)
    cases = [
        (ok, 0.0, (None, 16, 16, 16, 16), 1),                      # q NULL
        (ok, 0.0, (24, 16, 16, 16, 16), 1),                        # q misaligned
        (ok, float("inf"), (16, 16, 16, 16, 16), 1),               # non-finite scale
        (ok, float("nan"), (16, 16, 16, 16, 16), 1),
        (vdn.Shape(4, 4, 1, 0, 1025, 64), 0.0, (16, 16, 16, 16, 16), 1),   # H*D > 65536
        (vdn.Shape(4, 4, 1, 0, 1, 48), 0.0, (16, 16, 16, 16, 16), 2),      # head_dim 48
        (vdn.Shape(0, 4, 1, 0, 1, 32), 0.0, (16, 16, 16, 16, 16), 1),      # no frames
    ]
    for sh, scale, (q, k, v, kt, vt), want in cases:
        a = L.vdn_softmax_branch_fwd(ctypes.byref(sh), vdn.BF16, q, k, v, kt, vt, None, scale, 16, None, 256, 1 << 30,
                                     None)
        b = L.vdn_softmax_branch_fwd_noalloc(ctypes.byref(sh), vdn.BF16, q, k, v, kt, vt, scale, 16, None, None)
        assert a == b == want, (sh.frames, sh.heads, sh.head_dim, scale, a, b)
    st = L.vdn_softmax_branch_fwd_noalloc(ctypes.byref(ok), vdn.E4M3, 16, 16, 16, 16, 16, 0.0, 16, None, None)
    assert st == 2  # e4m3 needs scales, which this entry point does not take
    fits, over = vdn.Shape(2604, 256, 5, 16, 1, 64), vdn.Shape(2605, 256, 5, 16, 1, 64)
    st = L.vdn_softmax_branch_fwd_noalloc(ctypes.byref(fits), vdn.BF16, 16, 16, 16, 16, 16, 0.0, 16, None, None)
    assert st not in (0, 1, 3)  # passes every argument check; fails only for want of a GPU here
    st = L.vdn_softmax_branch_fwd_noalloc(ctypes.byref(over), vdn.BF16, 16, 16, 16, 16, 16, 0.0, 16, None, None)
    assert st == 3 and b"256 KiB" in L.vdn_last_error()


def test_partial_layer_checks():
    """vdn_hybrid_attn_fwd_partial (one rank's share of the head split) rejects what it
    cannot run before touching the device: head_dim other than 128, an out_features that
    is not a multiple of 32, and the e4m3 projection."""
    L = vdn.lib()
    p = [16] * 5

    def call(shape, n_out, dtype):
        s = vdn.Shape(*shape)
        return L.vdn_hybrid_attn_fwd_partial(ctypes.byref(s), n_out, vdn.ELU1, dtype, *p, None, 16, 16, shape[5], 16,
                                             1e-6, 16, 16, 16, 256, 1 << 40, None)
    assert call((4, 64, 5, 0, 2, 64), 128, vdn.BF16) == 2
    assert call((4, 64, 5, 0, 2, 128), 100, vdn.BF16) == 1
    assert call((4, 64, 5, 0, 2, 128), 0, vdn.BF16) == 1
    assert call((4, 64, 5, 0, 2, 128), 256, vdn.E4M3_PROJ) == 2
    assert call((4, 64, 5, 0, 2, 128), 256, vdn.BF16) not in (1, 2)   # valid; fails only for want of a GPU


def test_host_entry_point_checks_and_sizes():
    """The host-buffer layer: its workspace adds the staging area; missing host tensors and a
    short workspace are reported before any device work."""
    s = synth.Shape(90, 1008, 5, 512, 40, 128)
    nv, hd = 90 * 1008, 40 * 128
    full = vdn.hybrid_attn_workspace_size(s, vdn.ELU1, vdn.BF16)
    host = vdn.hybrid_attn_host_workspace_size(s, vdn.ELU1, vdn.BF16)
    # q, k, v, y (bf16) plus text k/v staged behind the layer's workspace
    assert host >= full + 4 * nv * hd * 2 + 2 * 512 * hd * 2
    assert vdn.hybrid_attn_host_workspace_size(s, vdn.DELTA, vdn.BF16) >= \
        vdn.hybrid_attn_workspace_size(s, vdn.DELTA, vdn.BF16) + 4 * nv * hd * 2 + 90 * 40 * 4
    t = vdn.Shape(15, 16, 1, 4, 2, 32)
    L = vdn.lib()
    args = [ctypes.byref(t), vdn.ELU1, vdn.F32, 16, 16, 16, 16, 16, None, 16, 16, 32, 16, 1e-6, 16, 16, 16, 256]
    big = vdn.hybrid_attn_host_workspace_size(t, vdn.ELU1, vdn.F32)
    a = list(args); a[3] = None
    assert L.vdn_hybrid_attn_fwd_host(*a, big, None) == 1 and b"host" in L.vdn_last_error()
    a = list(args); a[6] = None                                    # text k with L > 0
    assert L.vdn_hybrid_attn_fwd_host(*a, big, None) == 1
    assert L.vdn_hybrid_attn_fwd_host(*args, big - 256, None) == 3   # workspace too small
    a = list(args); a[1] = vdn.DELTA                               # the delta rule needs beta
    assert L.vdn_hybrid_attn_fwd_host(*a, vdn.hybrid_attn_host_workspace_size(t, vdn.DELTA, vdn.F32), None) == 1


@pytest.mark.parametrize("shape,kind,cdt,states", [
    ((90, 1008, 5, 512, 40, 128), vdn.ELU1, vdn.BF16, False),   # segmented scan: bf16 sum only
    ((90, 1008, 5, 512, 40, 128), vdn.DELTA, vdn.E4M3, True),
    ((12, 300, 5, 40, 2, 128), vdn.ELU1, vdn.F32, True),         # CUDA-core path: O_s, O_l too
    ((130, 4, 1, 3, 1, 128), vdn.ELU1, vdn.BF16, True),          # 127 segments: per-group states
    ((15, 16, 1, 4, 2, 64), vdn.DELTA, vdn.BF16, True),
])
def test_workspace_regions_disjoint_aligned_in_bounds(shape, kind, cdt, states):
    """The intermediates the layer exposes sit inside its workspace, 256-byte aligned, and
    do not overlap (pointer arithmetic only: a fake base address, no device)."""
    s = synth.Shape(*shape)
    F, T, C, L, H, D = shape
    base = 1 << 40
    total = vdn.hybrid_attn_workspace_size(s, kind, cdt)
    G = vdn.max_groups(s)
    act = 4 if cdt == vdn.F32 else 2
    nv = F * T
    sizes = {0: nv * H * D * act, 1: nv * H * D * act, 2: nv * 2 * H * D * act, 3: G * H * D * D * 4,
             4: G * H * D * D * 4, 5: F * 8 * 4, 6: G * 16 * 4, 7: 8 * 4, 8: 2 * 4, 9: (4 + F + 1 + 2 * G) * 4}
    regions = []
    for which, n in sizes.items():
        p = vdn.hybrid_attn_intermediate(s, kind, cdt, base, which)
        if p == 0:
            continue
        assert (p - base) % 256 == 0, which
        assert base <= p and p + n <= base + total, which
        regions.append((p, p + n, which))
    regions.sort()
    for (_, a1, wa), (b0, _, wb) in zip(regions, regions[1:]):
        assert a1 <= b0, (wa, wb)
    fused = cdt in (vdn.BF16, vdn.E4M3) and D == 128
    assert (vdn.hybrid_attn_intermediate(s, kind, cdt, base, 0) == 0) == fused
    assert (vdn.hybrid_attn_intermediate(s, kind, cdt, base, 3) != 0) == states
    assert vdn.hybrid_attn_intermediate(s, kind, cdt, base, 10) == 0
    assert vdn.hybrid_attn_intermediate(s, kind, cdt, None, 2) == 0
