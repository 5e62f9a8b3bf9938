"""The range-checked test build, libvdn_checked.so (VDN_BOUNDS_CHECK=1): a stand-in for a
device memory checker, which is closed on this machine.  In that build the tensor-core
kernels and the segmented scan check every global index they derive from the layout
tables (tile, group, rows, head, key parts, segment bounds) against its tensor's extent;
a violation is reported through the status word and the access skipped.

On the GPU, layer calls through the checked build must report no violation and give
exactly the bits of the normal build (the checks change no arithmetic)."""
import contextlib
import ctypes
import os

import numpy as np
import pytest
import torch

import hybrid_softmax_linear_b200 as vdn
from hybrid_softmax_linear_b200 import synth
from _harness import Run

CHECKED = os.path.join(os.path.dirname(vdn.LIB_PATH), "libvdn_checked.so")


def _load_checked():
    L = ctypes.CDLL(CHECKED)
    for name, (res, args) in vdn._SIGS.items():
        fn = getattr(L, name)
        fn.restype, fn.argtypes = res, args
    return L


@contextlib.contextmanager
def _using(lib):
    saved = vdn._lib
    vdn._lib = lib
    try:
        yield
    finally:
        vdn._lib = saved


def test_checked_build_exports_the_same_entry_points():
    assert os.path.exists(CHECKED), "build libvdn_checked.so with python -m hybrid_softmax_linear_b200.build --checked"
    L = _load_checked()
    assert all(hasattr(L, n) for n in vdn._SIGS)


CASES = [
    ((13, 200, 5, 40, 3, 128), vdn.ELU1, vdn.BF16),        # fused tensor-core path, ragged frames
    ((7, 130, 3, 0, 2, 128), vdn.ELU1, vdn.BF16),          # no text, short last chunk
    ((12, 96, 5, 24, 2, 128), vdn.DELTA, vdn.E4M3_PROJ),   # e4m3 softmax and projection, delta rule
    ((60, 1008, 5, 256, 24, 128), vdn.ELU1, vdn.BF16),     # medium: many groups and segments
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=["ragged", "no-text", "e4m3-delta", "medium"])
def test_checked_build_finds_nothing_and_matches(case):
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    shape, kind, cdt = case
    s = synth.Shape(*shape)
    inp = synth.make_inputs(s, "bf16", seed=61, with_beta=(kind == vdn.DELTA))
    y0 = Run(s, inp, "bf16", kind=kind, layer_dtype=cdt).layer().cpu()
    with _using(_load_checked()):
        y1 = Run(s, inp, "bf16", kind=kind, layer_dtype=cdt).layer().cpu()   # raises on a reported violation
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
