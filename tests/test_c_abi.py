"""The C ABI from C: a program that includes only include/vdn.h and links libvdn.so builds
with gcc and reproduces, on the host, the frame-7 layout printed on the pages and the
oracle's tables for a larger shape (no device needed)."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import hybrid_softmax_linear_b200 as vdn
from hybrid_softmax_linear_b200 import synth
from oracle import vdn_oracle as vo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include <stdlib.h>
#include "vdn.h"

int main(int argc, char **argv) {
  vdn_shape s;
  s.frames = atoi(argv[1]); s.tokens_per_frame = atoi(argv[2]); s.chunk_frames = atoi(argv[3]);
  s.text_tokens = atoi(argv[4]); s.heads = 1; s.head_dim = 32;
  int cap = vdn_max_groups(&s);
  int32_t *ft = (int32_t *)malloc(sizeof(int32_t) * 8 * s.frames);
  int32_t *gt = (int32_t *)malloc(sizeof(int32_t) * 16 * cap);
  int32_t G = 0;
  vdn_status st = vdn_mask_layout_build(&s, ft, gt, &G, (size_t)cap);
  if (st != VDN_OK) { printf("error %d %s\n", st, vdn_last_error()); return 1; }
  printf("version %d groups %d\n", vdn_version(), G);
  for (int f = 0; f < s.frames; ++f) {
    for (int i = 0; i < 8; ++i) printf("%d ", ft[f * 8 + i]);
    printf("\n");
  }
  /* a shape with too few group rows is refused without writing past them */
  int32_t G2 = 0;
  st = vdn_mask_layout_build(&s, ft, gt, &G2, 1);
  printf("cap1 %d\n", st);
  free(ft); free(gt);
  return 0;
}
"""


@pytest.fixture(scope="module")
def c_program(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    d = tmp_path_factory.mktemp("cabi")
    src = d / "layout.c"
    src.write_text(C_SOURCE)
    exe = d / "layout"
    libdir = os.path.dirname(vdn.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-O1", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    f"-L{libdir}", "-l:libvdn.so", f"-Wl,-rpath,{libdir}"], check=True)
    return str(exe)


def _run(exe, F, T, C, L):
    out = subprocess.run([exe, str(F), str(T), str(C), str(L)], check=True, capture_output=True, text=True).stdout
    lines = out.strip().splitlines()
    head = lines[0].split()
    ftab = np.array([[int(x) for x in ln.split()] for ln in lines[1:1 + F]], dtype=np.int32)
    return int(head[1]), int(head[3]), ftab, int(lines[-1].split()[1])


def test_c_program_reproduces_the_frame7_layout(c_program):
    """[ART] 局部精确计算 para. 2: 15 frames in 1-frame chunks; frame 7 attends exactly to
    frames {0, 6, 7, 8, 14}, its forward memory holds 1..5 and its backward memory 9..13."""
    version, G, ftab, cap1 = _run(c_program, 15, 16, 1, 4)
    assert version == vdn.version()
    g, win_lo, win_hi, anchor, fwd_lo, fwd_hi, bwd_lo, bwd_hi = ftab[7]
    assert (win_lo, win_hi, anchor) == (6, 9, 0)
    assert (fwd_lo, fwd_hi, bwd_lo, bwd_hi) == (1, 6, 9, 14)
    assert cap1 == 1  # VDN_ERR_INVALID_ARG


def test_c_program_matches_the_oracle_tables(c_program):
    F, T, C, L = 87, 40, 5, 16
    _, G, ftab, _ = _run(c_program, F, T, C, L)
    ref_ftab, ref_gtab = vo.layout_tables(F, T, C, L)
    assert G == len(ref_gtab)
    np.testing.assert_array_equal(ftab, ref_ftab)
