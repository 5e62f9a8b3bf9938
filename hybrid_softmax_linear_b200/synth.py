"""Seeded synthetic inputs for the hybrid attention layer.

This module only draws random numbers and stores them in the layer's input formats
(float32, or bfloat16 held as raw uint16 bit patterns).  It holds none of the layer's
arithmetic, so both the float64 oracle and the CUDA library can be fed from it.

Workload shapes follow the pages' 768p, ~14.4 s generation workload ("VDN-MiniMax-H3
开源" article, 性能表现; model card "Results" and "Inference with SGLang", warm-up
resolution 1344x768 with 345 frames).  The latent frame count (90), tokens per frame
(24x42 = 1008), head count and head size are not printed on the pages; they are the
workload definitions used throughout this library and are listed in ``CONFIGS``.

Generation is deterministic: one ``numpy.random.SeedSequence`` per tensor, split into
fixed chunks, each chunk filled by its own PCG64 generator.  Results do not depend on
the number of worker threads.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

BASE_SEED = 20261202
_CHUNK = 1 << 22  # elements per independently seeded chunk


@dataclasses.dataclass(frozen=True)
class Shape:
    frames: int           # F, latent frames
    tokens_per_frame: int  # T
    chunk_frames: int     # C, frames per local chunk
    text_tokens: int      # L
    heads: int            # H
    head_dim: int         # D

    @property
    def n_video(self) -> int:
        return self.frames * self.tokens_per_frame

    @property
    def hidden(self) -> int:
        return self.heads * self.head_dim


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: Shape
    dtype: str            # "f32" or "bf16": storage type of activations and out-proj weights
    keys: str = "normal"  # "normal" or "t3-10pct" (10% of key rows from Student-t, nu=3)
    softmax_fp8: bool = False   # softmax branch computed with e4m3 Q/K/V
    linear: str = "elu1"        # "elu1" (phi = elu+1 linear attention) or "delta"


CONFIGS = {
    1: Workload("tiny-15x16-c1-h2d32-f32", Shape(15, 16, 1, 4, 2, 32), "f32"),
    2: Workload("small-30x256-c5-h8d64-bf16", Shape(30, 256, 5, 64, 8, 64), "bf16"),
    3: Workload("medium-60x1008-c5-h24d128-bf16-tkeys", Shape(60, 1008, 5, 256, 24, 128), "bf16",
                keys="t3-10pct"),
    4: Workload("full-90x1008-c5-l512-h40d128-bf16", Shape(90, 1008, 5, 512, 40, 128), "bf16"),
    5: Workload("full-90x1008-c5-l512-h40d128-e4m3-delta", Shape(90, 1008, 5, 512, 40, 128), "bf16",
                softmax_fp8=True, linear="delta"),
}


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even.  Inputs are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f64(x: np.ndarray) -> np.ndarray:
    """Widen a stored input (float32, or bf16 bits as uint16) to float64, exactly."""
    if x.dtype == np.uint16:
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _fill(seed_seq: np.random.SeedSequence, n: int, draw, store_bf16: bool) -> np.ndarray:
    """Fill n values chunk by chunk; chunk i uses child seed i of seed_seq."""
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)
    kids = seed_seq.spawn(nchunks)
    out = np.empty(n, dtype=np.uint16 if store_bf16 else np.float32)

    def work(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        vals = draw(np.random.default_rng(kids[i]), hi - lo)
        out[lo:hi] = round_to_bf16_bits(vals) if store_bf16 else vals

    if nchunks == 1:
        work(0)
    else:
        with ThreadPoolExecutor(min(_threads(), nchunks)) as ex:
            list(ex.map(work, range(nchunks)))
    return out


def _normal(scale=1.0):
    def draw(g, n):
        x = g.standard_normal(n, dtype=np.float32)
        if scale != 1.0:
            x *= np.float32(scale)
        return x
    return draw


def _heavy_tail_rows(D, p=0.1, nu=3.0):
    """Rows (one (token, head) key vector of D values) drawn from Student-t(nu) with
    probability p, else N(0,1).  Chunks hold whole rows (the chunk size is a multiple of D)."""
    def draw(g, n):
        assert n % D == 0
        rows = n // D
        x = g.standard_normal(n, dtype=np.float32).reshape(rows, D)
        pick = g.random(rows) < p
        k = int(pick.sum())
        if k:
            x[pick] = g.standard_t(nu, size=(k, D)).astype(np.float32)
        return x.reshape(-1)
    return draw


def make_inputs(shape: Shape, dtype: str = "bf16", seed: int = BASE_SEED, keys: str = "normal",
                with_beta: bool = False, gate_l_cols: int | None = None) -> dict:
    """All inputs of one layer call, in generation order
    q, k, v, kt, vt, w_gate_s, w_gate_l, w_os, w_ol, (beta); gamma = 1.

    Activations and out-projection weights are stored as ``dtype`` ("bf16" -> uint16 bit
    patterns, "f32" -> float32).  Gate weights, gamma and beta are float32.
    Layouts: q/k/v [F*T, H, D] frame-major; kt/vt [L, H, D]; w_gate_s [H, D];
    w_gate_l [H, D, G_l]; w_os/w_ol [H*D (out), H*D (in)]; gamma [H, D]; beta [F, H]."""
    assert dtype in ("bf16", "f32")
    F, T, L, H, D = shape.frames, shape.tokens_per_frame, shape.text_tokens, shape.heads, shape.head_dim
    assert _CHUNK % D == 0
    G_l = D if gate_l_cols is None else gate_l_cols
    bf = dtype == "bf16"
    root = np.random.SeedSequence(seed)
    s = root.spawn(10)
    Nv, HD = F * T, H * D
    kdraw = _heavy_tail_rows(D) if keys == "t3-10pct" else _normal()
    assert keys in ("normal", "t3-10pct")
    out = {
        "q": _fill(s[0], Nv * HD, _normal(), bf).reshape(Nv, H, D),
        "k": _fill(s[1], Nv * HD, kdraw, bf).reshape(Nv, H, D),
        "v": _fill(s[2], Nv * HD, _normal(), bf).reshape(Nv, H, D),
        "kt": _fill(s[3], L * HD, kdraw, bf).reshape(L, H, D),
        "vt": _fill(s[4], L * HD, _normal(), bf).reshape(L, H, D),
        "w_gate_s": _fill(s[5], HD, _normal(0.02), False).reshape(H, D),
        "w_gate_l": _fill(s[6], HD * G_l, _normal(0.02), False).reshape(H, D, G_l),
        "w_os": _fill(s[7], HD * HD, _normal(0.02), bf).reshape(HD, HD),
        "w_ol": _fill(s[8], HD * HD, _normal(0.02), bf).reshape(HD, HD),
        "gamma": np.ones((H, D), dtype=np.float32),
    }
    if with_beta:
        z = np.random.default_rng(s[9]).standard_normal((F, H))
        out["beta"] = (1.0 / (1.0 + np.exp(-z))).astype(np.float32)
    return out


def workload_inputs(cfg: int, rank: int = 0) -> dict:
    """Inputs of configuration ``cfg`` (1..5); replica ``rank`` draws its own batch."""
    w = CONFIGS[cfg]
    return make_inputs(w.shape, w.dtype, BASE_SEED + cfg + 1000 * rank, w.keys,
                       with_beta=(w.linear == "delta"))


def sample_rows(shape: Shape, per_frame: int = 8, seed: int = 7) -> np.ndarray:
    """Video query rows checked at full size: first and last token of every frame plus
    (per_frame - 2) distinct random tokens in between, sorted."""
    F, T = shape.frames, shape.tokens_per_frame
    g = np.random.default_rng(seed)
    rows = []
    for f in range(F):
        pick = {0, T - 1}
        inner = np.arange(1, T - 1)
        k = min(per_frame - 2, inner.size)
        if k > 0:
            pick.update(g.choice(inner, size=k, replace=False).tolist())
        rows.extend(f * T + t for t in sorted(pick))
    return np.asarray(rows, dtype=np.int64)
