"""Pins of the float64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: the printed frame-7
illustration, a layout derived by hand from the simplified figure, brute-force set
enumeration, closed forms, and library routines (torch CPU float64) on cases that reduce
to them.  The planted-mistake tests at the end show that plausible slips in the oracle
(a dropped text half, swapped memories, a lost anchor, a wrong sign in the delta rule)
each make at least one pin fail.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import vdn_oracle as vo
from hybrid_softmax_linear_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as fh:
        return json.load(fh)


def _sets_from_mask(M, fq):
    return ([int(x) for x in np.nonzero(M[fq] == vo.SOFT)[0]],
            [int(x) for x in np.nonzero(M[fq] == vo.FWD)[0]],
            [int(x) for x in np.nonzero(M[fq] == vo.BWD)[0]])


def _brute_sets(F, C, fq):
    """The rule of the article, written with Python sets and chunk ids."""
    chunk = [f // C for f in range(F)]
    anchors = {0, F - 1}
    if fq in anchors:
        return sorted(range(F)), [], []
    window = {fk for fk in range(F) if abs(chunk[fk] - chunk[fq]) <= 1}
    soft = window | anchors
    rest = set(range(F)) - soft
    return sorted(soft), sorted(f for f in rest if f < min(window)), sorted(f for f in rest if f > max(window))


def _inputs(F, T, L, H, D, seed=1, keys="normal"):
    x = synth.make_inputs(synth.Shape(F, T, 1, L, H, D), "f32", seed=seed, keys=keys)
    return {n: a.astype(np.float64) for n, a in x.items()}


# ----------------------------------------------------------------------------- layout pins
@pytest.mark.parametrize("name", ["frame7_F15_C1.json", "frame7_F16_C2_derived.json"])
def test_worked_example(name):
    g = _golden(name)
    M = vo.frame_mask(g["frames"], g["chunk_frames"])
    soft, fwd, bwd = _sets_from_mask(M, g["query_frame"])
    assert soft == g["softmax_frames"]
    assert fwd == g["forward_frames"]
    assert bwd == g["backward_frames"]


@pytest.mark.parametrize("F", list(range(1, 41)))
def test_mask_brute_force_and_partition(F):
    for C in range(1, 7):
        M = vo.frame_mask(F, C)
        for fq in range(F):
            soft, fwd, bwd = _sets_from_mask(M, fq)
            assert (soft, fwd, bwd) == _brute_sets(F, C, fq)
            # every key frame in exactly one branch
            assert sorted(soft + fwd + bwd) == list(range(F))
            # anchors: read everything by softmax, and are read by everyone
            if fq in (0, F - 1):
                assert soft == list(range(F))
            assert 0 in soft and (F - 1) in soft
            # forward memory precedes the query, backward follows it
            assert all(f < fq for f in fwd) and all(f > fq for f in bwd)


def _expand(segs):
    out = set()
    for lo, hi in segs:
        out.update(range(lo, hi))
    return out


@pytest.mark.parametrize("F,T,C,L", [(15, 16, 1, 4), (30, 256, 5, 64), (87, 3, 5, 2), (16, 1, 2, 1),
                                     (2, 5, 5, 0), (1, 4, 5, 3), (11, 7, 5, 0), (90, 1008, 5, 512)])
def test_layout_tables_cover_the_explicit_sets(F, T, C, L):
    ftab, gtab = vo.layout_tables(F, T, C, L)
    covered = np.zeros(F, int)
    for g, row in enumerate(gtab):
        flo, fhi, nseg = row[0], row[1], row[2]
        segs = [(row[4 + 2 * s], row[5 + 2 * s]) for s in range(nseg)]
        assert all(row[4 + 2 * s] == 0 and row[5 + 2 * s] == 0 for s in range(nseg, 4))
        # segments sorted, disjoint and not adjacent (maximally merged)
        assert all(segs[i][1] < segs[i + 1][0] for i in range(len(segs) - 1))
        for fq in range(flo, fhi):
            covered[fq] += 1
            soft, fwd, bwd = _brute_sets(F, C, fq)
            tokens = set(range(L)) | {L + f * T + t for f in soft for t in range(T)}
            assert _expand(segs) == tokens
            assert (row[12], row[13]) == ((fwd[0], fwd[-1] + 1) if fwd else (0, 0))
            assert (row[14], row[15]) == ((bwd[0], bwd[-1] + 1) if bwd else (0, 0))
            assert ftab[fq, 0] == g
        if g > 0:  # runs are maximal: neighbours differ somewhere
            assert not np.array_equal(gtab[g - 1][2:], row[2:])
    assert (covered == 1).all()
    assert len(gtab) <= -(-F // C) + 2


# ----------------------------------------------------------------------------- softmax pins
def _token_mask(F, T, C, L):
    """Boolean [N, L+N] visibility of the softmax branch from the brute-force sets."""
    N = F * T
    m = np.zeros((N, L + N), bool)
    m[:, :L] = True  # text is visible to every frame
    for fq in range(F):
        soft, _, _ = _brute_sets(F, C, fq)
        for fk in soft:
            m[fq * T:(fq + 1) * T, L + fk * T:L + (fk + 1) * T] = True
    return m


def _sdpa(q, K, V, mask=None):
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(K).permute(1, 0, 2)[None]
    vt = torch.from_numpy(V).permute(1, 0, 2)[None]
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m)
    return o[0].permute(1, 0, 2).numpy()


def test_softmax_all_window_equals_dense_sdpa():
    F, T, C, L, H, D = 8, 5, 4, 3, 2, 16   # 2 chunks: every frame sees everything
    x = _inputs(F, T, L, H, D, seed=3)
    o = vo.softmax_branch(x["q"], x["k"], x["v"], x["kt"], x["vt"], F, T, C)
    ref = _sdpa(x["q"], np.concatenate([x["kt"], x["k"]]), np.concatenate([x["vt"], x["v"]]))
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("F,T,C,L", [(15, 4, 1, 4), (23, 3, 5, 2), (16, 2, 2, 1), (11, 3, 2, 0)])
def test_softmax_matches_masked_sdpa(F, T, C, L):
    H, D = 2, 8
    x = _inputs(F, T, L, H, D, seed=F + C)
    o = vo.softmax_branch(x["q"], x["k"], x["v"], x["kt"], x["vt"], F, T, C)
    ref = _sdpa(x["q"], np.concatenate([x["kt"], x["k"]]), np.concatenate([x["vt"], x["v"]]),
                _token_mask(F, T, C, L))
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def test_softmax_hand_case():
    # F=3, T=1, no text, D=1: every frame sees frames 0..2; scores q*k*1
    q = np.array([[[1.0]], [[0.0]], [[-2.0]]])
    k = np.array([[[0.5]], [[1.0]], [[2.0]]])
    v = np.array([[[1.0]], [[10.0]], [[100.0]]])
    e = np.zeros((0, 1, 1))
    o = vo.softmax_branch(q, k, v, e, e, 3, 1, 1)
    for i, qi in enumerate([1.0, 0.0, -2.0]):
        w = np.exp(qi * np.array([0.5, 1.0, 2.0]))
        assert abs(o[i, 0, 0] - (w @ np.array([1.0, 10.0, 100.0])) / w.sum()) < 1e-12


def test_softmax_rows_sampling_matches_full():
    F, T, C, L, H, D = 20, 6, 2, 3, 2, 8
    x = _inputs(F, T, L, H, D, seed=5)
    full = vo.softmax_branch(x["q"], x["k"], x["v"], x["kt"], x["vt"], F, T, C)
    rows = synth.sample_rows(synth.Shape(F, T, C, L, H, D), per_frame=3)
    part = vo.softmax_branch(x["q"], x["k"], x["v"], x["kt"], x["vt"], F, T, C, rows=rows)
    np.testing.assert_allclose(part, full[rows], rtol=1e-13, atol=1e-15)


# ----------------------------------------------------------------------------- linear pins
def test_phi_is_elu_plus_one():
    x = np.linspace(-30, 30, 2001)
    # torch computes elu(x) + 1 as (exp(x) - 1) + 1, exact to one ulp of 1
    np.testing.assert_allclose(vo.phi(x), torch.nn.functional.elu(torch.from_numpy(x)).numpy() + 1,
                               rtol=1e-15, atol=2.3e-16)
    np.testing.assert_array_equal(vo.phi(np.array([-1.0, 0.0, 2.5])), [np.exp(-1.0), 1.0, 3.5])


@pytest.mark.parametrize("F,T,C,L", [(15, 4, 1, 4), (23, 3, 5, 2), (16, 2, 2, 1), (30, 2, 5, 0), (11, 3, 2, 6)])
def test_linear_state_form_equals_masked_form(F, T, C, L):
    H, D = 2, 8
    x = _inputs(F, T, L, H, D, seed=2 * F + C)
    a = vo.linear_branch(x["q"], x["k"], x["v"], x["kt"], x["vt"], F, T, C)
    b = vo.linear_branch_masked(x["q"], x["k"], x["v"], x["kt"], x["vt"], F, T, C)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_linear_text_counted_once():
    # C >= F: no memory frames; the read is plain linear attention over the text alone
    F, T, C, L, H, D = 6, 3, 6, 5, 2, 8
    x = _inputs(F, T, L, H, D, seed=9)
    o = vo.linear_branch(x["q"], x["k"], x["v"], x["kt"], x["vt"], F, T, C)
    fk = torch.nn.functional.elu(torch.from_numpy(x["kt"])).numpy() + 1
    fq = torch.nn.functional.elu(torch.from_numpy(x["q"])).numpy() + 1
    for h in range(H):
        num = fq[:, h] @ (fk[:, h].T @ x["vt"][:, h])
        den = fq[:, h] @ fk[:, h].sum(0)
        np.testing.assert_allclose(o[:, h], num / den[:, None], rtol=1e-12)


def test_linear_prefix_identity():
    F, T, C, L, H, D = 27, 2, 5, 3, 2, 4
    x = _inputs(F, T, L, H, D, seed=11)
    num_f, num_b, den_f, den_b = vo.linear_memory(x["k"], x["v"], x["kt"], x["vt"], F, T, C)
    S, z = vo.frame_states(x["k"], x["v"], F, T)
    St, zt = vo.text_state(x["kt"], x["vt"])
    pref = np.concatenate([np.zeros((1,) + S.shape[1:]), np.cumsum(S, axis=0)])    # pref[a] = sum_{f<a}
    for fq in range(1, F - 1):
        a, b = vo.chunk_window(fq, F, C)
        a, b = max(a, 1), min(b, F - 1)
        np.testing.assert_allclose(num_f[fq] - 0.5 * St, pref[a] - pref[1], atol=1e-10)
        np.testing.assert_allclose(num_b[fq] - 0.5 * St, pref[F - 1] - pref[b], atol=1e-10)
    for fq in (0, F - 1):
        np.testing.assert_allclose(num_f[fq], 0.5 * St)
        np.testing.assert_allclose(den_b[fq], 0.5 * zt)


def test_linear_frame_state_closed_form():
    # one token per frame: S_f = phi(k)^T v exactly
    k = np.array([[[0.5, -1.0]]]); v = np.array([[[2.0, 3.0]]])
    S, z = vo.frame_states(k, v, 1, 1)
    pk = np.array([1.5, np.exp(-1.0)])
    np.testing.assert_allclose(S[0, 0], np.outer(pk, [2.0, 3.0]), rtol=1e-15)
    np.testing.assert_allclose(z[0, 0], pk, rtol=1e-15)


def test_branches_invariant_to_token_order_within_frames():
    F, T, C, L, H, D = 12, 5, 2, 3, 2, 8
    x = _inputs(F, T, L, H, D, seed=13)
    perm = np.concatenate([f * T + np.random.default_rng(f).permutation(T) for f in range(F)])
    y = dict(x); y["k"] = x["k"][perm]; y["v"] = x["v"][perm]
    for fn in (vo.linear_branch, vo.softmax_branch):
        np.testing.assert_allclose(fn(x["q"], x["k"], x["v"], x["kt"], x["vt"], F, T, C),
                                   fn(y["q"], y["k"], y["v"], y["kt"], y["vt"], F, T, C), rtol=1e-11, atol=1e-13)


def test_linear_empty_set_reads_zero():
    # no text and every frame inside the softmax set: the normaliser is 0 -> output 0
    F, T, C, L, H, D = 3, 2, 1, 0, 1, 4
    x = _inputs(F, T, L, H, D, seed=1)
    o = vo.linear_branch(x["q"], x["k"], x["v"], x["kt"], x["vt"], F, T, C)
    assert np.all(o == 0)


# ----------------------------------------------------------------------------- delta pins
def test_delta_beta_zero_keeps_text_init():
    F, T, C, L, H, D = 20, 3, 2, 4, 2, 8
    x = _inputs(F, T, L, H, D, seed=17)
    Sf, Sb = vo.delta_memory(x["k"], x["v"], x["kt"], x["vt"], np.zeros((F, H)), F, T, C)
    kh = x["kt"] / np.linalg.norm(x["kt"], axis=-1, keepdims=True)
    S0 = 0.5 * np.einsum("thd,the->hde", kh, x["vt"])
    for fq in range(F):
        np.testing.assert_allclose(Sf[fq], S0, rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(Sb[fq], S0, rtol=1e-13, atol=1e-15)


def test_delta_single_update_from_zero():
    rng = np.random.default_rng(0)
    kb = vo.l2_normalize(rng.standard_normal((3, 6)))
    vb = rng.standard_normal((3, 6))
    beta = np.array([0.2, 0.5, 0.9])
    S = vo.delta_update(np.zeros((3, 6, 6)), kb, vb, beta)
    for h in range(3):
        np.testing.assert_allclose(S[h], beta[h] * np.outer(kb[h], vb[h]), rtol=1e-14, atol=1e-16)


def test_delta_exact_write_at_beta_one():
    rng = np.random.default_rng(1)
    S = rng.standard_normal((2, 8, 8))
    kb = vo.l2_normalize(rng.standard_normal((2, 8)))
    vb = rng.standard_normal((2, 8))
    S1 = vo.delta_update(S, kb, vb, np.ones(2))
    for h in range(2):
        np.testing.assert_allclose(kb[h] @ S1[h], vb[h], rtol=1e-12, atol=1e-12)   # k^T S_new = v^T


def test_delta_frame_stats_single_token_frames():
    # T = 1: the frame mean is the token itself, so kb = k / ||k|| and vb = v exactly
    rng = np.random.default_rng(31)
    F, H, D = 5, 3, 7
    k, v = rng.standard_normal((F, H, D)) * 3, rng.standard_normal((F, H, D))
    kb, vb = vo.delta_frame_stats(k, v, F, 1)
    np.testing.assert_allclose(kb, k / np.linalg.norm(k, axis=-1, keepdims=True), rtol=1e-15)
    np.testing.assert_array_equal(vb, v)


def test_delta_frame_stats_closed_forms():
    F, T, H, D = 3, 2, 1, 2
    k = np.zeros((F * T, H, D)); v = np.zeros((F * T, H, D))
    # frame 0: keys (3, 0) and (0, 1): mean (1.5, 0.5), normalised (3, 1) / sqrt(10); taking
    # each key's direction first would give (1, 1) / sqrt(2)
    k[0, 0] = [3.0, 0.0]; k[1, 0] = [0.0, 1.0]
    v[0, 0] = [2.0, -4.0]; v[1, 0] = [4.0, 8.0]
    # frame 1: two identical tokens: kb = k / ||k||, vb = v
    k[2, 0] = k[3, 0] = [-6.0, 8.0]
    v[2, 0] = v[3, 0] = [0.5, 0.25]
    # frame 2: keys k and -k: zero mean, which normalises to zero (R13)
    k[4, 0] = [1.0, 2.0]; k[5, 0] = [-1.0, -2.0]
    kb, vb = vo.delta_frame_stats(k, v, F, T)
    np.testing.assert_allclose(kb[0, 0], np.array([3.0, 1.0]) / np.sqrt(10.0), rtol=1e-15)
    np.testing.assert_allclose(vb[0, 0], [3.0, 2.0], rtol=1e-15)
    np.testing.assert_allclose(kb[1, 0], [-0.6, 0.8], rtol=1e-15)
    np.testing.assert_allclose(vb[1, 0], [0.5, 0.25], rtol=1e-15)
    np.testing.assert_array_equal(kb[2, 0], [0.0, 0.0])


def test_delta_frame_stats_matches_torch_composition():
    # frame-major rows [F*T, H, D]: frame f is rows f*T .. f*T+T-1; the mean runs over the
    # tokens of a frame, separately for every head and feature
    F, T, H, D = 6, 5, 3, 4
    rng = np.random.default_rng(32)
    k = rng.standard_normal((F * T, H, D)) * rng.uniform(0.1, 5.0, (F * T, H, 1))
    v = rng.standard_normal((F * T, H, D))
    kb, vb = vo.delta_frame_stats(k, v, F, T)
    tk, tv = torch.from_numpy(k).view(F, T, H, D), torch.from_numpy(v).view(F, T, H, D)
    ref_kb = torch.nn.functional.normalize(tk.mean(dim=1), dim=-1)
    np.testing.assert_allclose(kb, ref_kb.numpy(), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(vb, tv.mean(dim=1).numpy(), rtol=1e-13, atol=1e-15)


def test_delta_per_group_rerun_equals_single_pass_snapshots():
    F, T, C, L, H, D = 33, 2, 5, 3, 2, 8
    x = _inputs(F, T, L, H, D, seed=19)
    beta = 1 / (1 + np.exp(-np.random.default_rng(3).standard_normal((F, H))))
    Sf, Sb = vo.delta_memory(x["k"], x["v"], x["kt"], x["vt"], beta, F, T, C)
    kb, vb = vo.delta_frame_stats(x["k"], x["v"], F, T)
    S0 = vo.delta_text_init(x["kt"], x["vt"])
    # forward pass once over frames 1..F-2 with the rank-one form of the update, snapshots
    fwd = [S0]
    S = S0.copy()
    for f in range(1, F - 1):
        u = np.einsum("hd,hde->he", kb[f], S)
        S = S + beta[f][:, None, None] * kb[f][:, :, None] * (vb[f] - u)[:, None, :]
        fwd.append(S)          # fwd[j] = state after frames 1..j
    bwd = {F - 1: S0}
    S = S0.copy()
    for f in range(F - 2, 0, -1):
        u = np.einsum("hd,hde->he", kb[f], S)
        S = S + beta[f][:, None, None] * kb[f][:, :, None] * (vb[f] - u)[:, None, :]
        bwd[f] = S             # state after frames F-2 .. f
    for fq in range(1, F - 1):
        a, b = vo.chunk_window(fq, F, C)
        a, b = max(a, 1), min(b, F - 1)
        np.testing.assert_allclose(Sf[fq], fwd[a - 1], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(Sb[fq], bwd[b], rtol=1e-10, atol=1e-12)


def test_delta_read_is_normalised_query():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((4, 1, 5)) * 7
    Sf = rng.standard_normal((1, 1, 5, 5)); Sb = rng.standard_normal((1, 1, 5, 5))
    o = vo.delta_read(q, Sf, Sb, 4)
    for n in range(4):
        qh = q[n, 0] / np.linalg.norm(q[n, 0])
        np.testing.assert_allclose(o[n, 0], (Sf[0, 0] + Sb[0, 0]).T @ qh, rtol=1e-13)


# ----------------------------------------------------------------------------- fuse + projection pins
def test_fuse_matches_torch_routines():
    n, H, D = 7, 3, 8
    rng = np.random.default_rng(4)
    q, o_s, o_l = (rng.standard_normal((n, H, D)) for _ in range(3))
    ws = rng.standard_normal((H, D)) * 0.3
    wl = rng.standard_normal((H, D, D)) * 0.3
    gamma = rng.standard_normal((H, D))
    a = vo.hybrid_fuse(q, o_s, o_l, ws, wl, gamma, 1e-6)
    tq = torch.from_numpy(q)
    gs = torch.sigmoid((tq * torch.from_numpy(ws)).sum(-1, keepdim=True))
    gl = torch.sigmoid(torch.einsum("nhd,hde->nhe", tq, torch.from_numpy(wl)))
    nrm = torch.nn.functional.rms_norm(torch.from_numpy(o_l), (D,), eps=1e-6) * torch.from_numpy(gamma)
    ref = torch.cat([(gs * torch.from_numpy(o_s)).reshape(n, -1), (gl * nrm).reshape(n, -1)], 1)
    np.testing.assert_allclose(a, ref.numpy(), rtol=1e-13, atol=1e-15)


def test_fuse_closed_forms():
    n, H, D = 2, 2, 4
    q = np.ones((n, H, D)); o_s = np.full((n, H, D), 3.0); o_l = np.full((n, H, D), 2.0)
    a = vo.hybrid_fuse(q, o_s, o_l, np.zeros((H, D)), np.zeros((H, D, 1)), np.ones((H, D)), 0.0)
    np.testing.assert_allclose(a[:, :H * D], 1.5)   # sigmoid(0) * 3
    np.testing.assert_allclose(a[:, H * D:], 0.5)   # sigmoid(0) * (2 / 2)


def test_out_proj_identity_and_torch():
    rng = np.random.default_rng(5)
    a = rng.standard_normal((5, 12))
    y = vo.out_proj(a, np.eye(6), np.eye(6))
    np.testing.assert_allclose(y, a[:, :6] + a[:, 6:], rtol=1e-15)
    w1, w2 = rng.standard_normal((6, 6)), rng.standard_normal((6, 6))
    ref = torch.nn.functional.linear(torch.from_numpy(a[:, :6]), torch.from_numpy(w1)) + \
        torch.nn.functional.linear(torch.from_numpy(a[:, 6:]), torch.from_numpy(w2))
    np.testing.assert_allclose(vo.out_proj(a, w1, w2), ref.numpy(), rtol=1e-13)


def _torch_layer(x, F, T, C, L):
    """The layer composed from torch float64 routines on the token-level masks."""
    N, H, D = x["q"].shape
    q, k, v = (torch.from_numpy(x[n]) for n in ("q", "k", "v"))
    kt, vt = torch.from_numpy(x["kt"]), torch.from_numpy(x["vt"])
    K, V = torch.cat([kt, k]), torch.cat([vt, v])
    soft = torch.from_numpy(_token_mask(F, T, C, L))
    o_s = torch.nn.functional.scaled_dot_product_attention(
        q.permute(1, 0, 2), K.permute(1, 0, 2), V.permute(1, 0, 2), attn_mask=soft).permute(1, 0, 2)
    w = (~soft).double(); w[:, :L] = 1.0
    fq, fk = torch.nn.functional.elu(q) + 1, torch.nn.functional.elu(K) + 1
    A = torch.einsum("nhd,mhd->hnm", fq, fk) * w
    o_l = (torch.einsum("hnm,mhd->nhd", A, V) / A.sum(-1).T[..., None])
    gs = torch.sigmoid((q * torch.from_numpy(x["w_gate_s"])).sum(-1, keepdim=True))
    gl = torch.sigmoid(torch.einsum("nhd,hde->nhe", q, torch.from_numpy(x["w_gate_l"])))
    nrm = torch.nn.functional.rms_norm(o_l, (D,), eps=1e-6) * torch.from_numpy(x["gamma"])
    y = torch.nn.functional.linear((gs * o_s).reshape(N, -1), torch.from_numpy(x["w_os"])) + \
        torch.nn.functional.linear((gl * nrm).reshape(N, -1), torch.from_numpy(x["w_ol"]))
    return y.numpy()


@pytest.mark.parametrize("cfg_shape", [(15, 16, 1, 4, 2, 32), (20, 3, 2, 5, 3, 8)])
def test_layer_matches_torch_composition(cfg_shape):
    F, T, C, L, H, D = cfg_shape
    x = synth.make_inputs(synth.Shape(F, T, C, L, H, D), "f32", seed=21)
    x = {n: a.astype(np.float64) for n, a in x.items()}
    out = vo.layer(x, F, T, C)
    np.testing.assert_allclose(out["y"], _torch_layer(x, F, T, C, L), rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------- planted mistakes
def _pins_hold():
    """Run a bundle of pins; True when all pass."""
    checks = [
        lambda: test_worked_example("frame7_F15_C1.json"),
        lambda: test_mask_brute_force_and_partition(17),
        lambda: test_linear_text_counted_once(),
        lambda: test_linear_state_form_equals_masked_form(23, 3, 5, 2),
        lambda: test_layer_matches_torch_composition((20, 3, 2, 5, 3, 8)),
        lambda: test_delta_single_update_from_zero(),
        lambda: test_delta_exact_write_at_beta_one(),
        lambda: test_delta_per_group_rerun_equals_single_pass_snapshots(),
        lambda: test_delta_frame_stats_single_token_frames(),
        lambda: test_delta_frame_stats_closed_forms(),
        lambda: test_delta_frame_stats_matches_torch_composition(),
        lambda: test_softmax_matches_masked_sdpa(23, 3, 5, 2),
    ]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def test_pins_hold_on_the_unmodified_oracle():
    assert _pins_hold()


def _mask_without_anchor_reads(F, C):
    M = np.full((F, F), -1, dtype=np.int8)
    for fq in range(F):
        lo, hi = vo.chunk_window(fq, F, C)
        for fk in range(F):
            if vo.is_anchor(fk, F) or lo <= fk < hi:      # anchors no longer read every frame
                M[fq, fk] = vo.SOFT
            else:
                M[fq, fk] = vo.FWD if fk < lo else vo.BWD
    return M


def _mask_swapped(F, C):
    M = vo.__dict__["_orig_frame_mask"](F, C)
    out = M.copy()
    out[M == vo.FWD] = vo.BWD
    out[M == vo.BWD] = vo.FWD
    return out


def _text_state_full(kt, vt):
    S, z = vo.__dict__["_orig_text_state"](kt, vt)
    return 2 * S, 2 * z                                   # text written fully into each state


def _delta_update_wrong_sign(S, kb, vb, beta):
    H, D = kb.shape
    b = np.asarray(beta, np.float64)[:, None, None]
    return np.matmul(np.eye(D)[None] + b * kb[:, :, None] * kb[:, None, :], S) + b * kb[:, :, None] * vb[:, None, :]


def _softmax_without_text(q, k, v, kt, vt, F, T, C, scale=None, rows=None):
    return vo.__dict__["_orig_softmax_branch"](q, k, v, kt[:0], vt[:0], F, T, C, scale, rows)


def _delta_stats_tokens_normalised_first(k, v, F, T):
    kb, vb = vo.__dict__["_orig_delta_frame_stats"](vo.l2_normalize(k), v, F, T)
    return kb, vb                                         # each key's direction averaged


def _delta_stats_unnormalised(k, v, F, T):
    N, H, D = k.shape
    kb = np.asarray(k, np.float64).reshape(F, T, H, D).mean(axis=1)   # mean key, left unnormalised
    return kb, np.asarray(v, np.float64).reshape(F, T, H, D).mean(axis=1)


def _delta_stats_strided_frames(k, v, F, T):
    # frame f taken as rows f, f+F, f+2F, ... (token-major reading of frame-major rows)
    N, H, D = k.shape
    kb = vo.l2_normalize(np.asarray(k, np.float64).reshape(T, F, H, D).mean(axis=0))
    return kb, np.asarray(v, np.float64).reshape(T, F, H, D).mean(axis=0)


@pytest.mark.parametrize("attr,bad", [
    ("frame_mask", _mask_without_anchor_reads),
    ("frame_mask", _mask_swapped),
    ("text_state", _text_state_full),
    ("delta_update", _delta_update_wrong_sign),
    ("softmax_branch", _softmax_without_text),
    ("delta_frame_stats", _delta_stats_tokens_normalised_first),
    ("delta_frame_stats", _delta_stats_unnormalised),
    ("delta_frame_stats", _delta_stats_strided_frames),
])
def test_planted_mistake_is_caught(monkeypatch, attr, bad):
    monkeypatch.setattr(vo, "_orig_" + attr, getattr(vo, attr), raising=False)
    monkeypatch.setattr(vo, attr, bad)
    assert not _pins_hold()
