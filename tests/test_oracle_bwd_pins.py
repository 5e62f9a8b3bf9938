"""Pins of the backward oracle (oracle/vdn_oracle_bwd.py), CPU only.

Every gradient is checked against central finite differences of the forward oracle, which
is pinned on its own (tests/test_oracle_pins.py).  The checks use a random direction per
input tensor (all of its entries at once) plus a few single entries, in float64.  The
softmax branch with every key visible is also checked against torch's autograd of dense
attention, a library routine.  The shapes cover chunk windows, both anchors, forward and
backward memories, text and no text, one-frame chunks, the scalar linear gate, and both
linear branches (elu+1 and the delta rule)."""
import numpy as np
import pytest
import torch

from oracle import vdn_oracle as vo
from oracle import vdn_oracle_bwd as vb

NAMES = ("q", "k", "v", "kt", "vt", "w_gate_s", "w_gate_l", "gamma", "w_os", "w_ol")


def _inputs(F, T, L, H, D, G_l=None, seed=0):
    rng = np.random.default_rng(seed)
    N, HD = F * T, H * D
    G_l = D if G_l is None else G_l
    return {"q": rng.standard_normal((N, H, D)), "k": rng.standard_normal((N, H, D)),
            "v": rng.standard_normal((N, H, D)), "kt": rng.standard_normal((L, H, D)),
            "vt": rng.standard_normal((L, H, D)), "w_gate_s": 0.5 * rng.standard_normal((H, D)),
            "w_gate_l": 0.5 * rng.standard_normal((H, D, G_l)), "gamma": 1.0 + 0.1 * rng.standard_normal((H, D)),
            "w_os": 0.3 * rng.standard_normal((HD, HD)), "w_ol": 0.3 * rng.standard_normal((HD, HD))}


def _check_fd(loss, inp, grads, names, seed=1, eps=1e-6, entries=3, rtol=1e-6):
    """grads[n] against central differences of loss() along a random direction and at a
    few single entries of inp[n]."""
    rng = np.random.default_rng(seed)
    for n in names:
        x = inp[n]
        if x.size == 0:
            assert grads[n].size == 0
            continue
        dirs = [rng.standard_normal(x.shape)]
        for _ in range(entries):
            e = np.zeros(x.size)
            e[rng.integers(x.size)] = 1.0
            dirs.append(e.reshape(x.shape))
        for u in dirs:
            inp[n] = x + eps * u
            lp = loss()
            inp[n] = x - eps * u
            lm = loss()
            inp[n] = x
            fd = (lp - lm) / (2 * eps)
            an = float((grads[n] * u).sum())
            assert abs(fd - an) <= rtol * max(1.0, abs(fd)) + 1e-8, (n, fd, an)


SHAPES = [
    # F, T, C, L, H, D, G_l
    (7, 2, 2, 3, 2, 4, None),    # windows, anchors, both memories, text
    (6, 3, 1, 0, 1, 4, None),    # one-frame chunks, no text (anchors read nothing linear)
    (9, 2, 2, 2, 1, 4, 1),       # scalar linear gate
]


@pytest.mark.parametrize("F,T,C,L,H,D,G_l", SHAPES)
def test_layer_gradients_match_finite_differences(F, T, C, L, H, D, G_l):
    inp = _inputs(F, T, L, H, D, G_l)
    dy = np.random.default_rng(7).standard_normal((F * T, H * D))
    grads = vb.layer_bwd(inp, dy, F, T, C)
    _check_fd(lambda: float((vo.layer(inp, F, T, C)["y"] * dy).sum()), inp, grads, NAMES)


@pytest.mark.parametrize("F,T,C,L,H,D,G_l", SHAPES[:2])
def test_delta_layer_gradients_match_finite_differences(F, T, C, L, H, D, G_l):
    """The layer with the delta-rule linear branch: beta is an input too."""
    inp = _inputs(F, T, L, H, D, G_l, seed=13)
    inp["beta"] = 1.0 / (1.0 + np.exp(-np.random.default_rng(14).standard_normal((F, H))))
    dy = np.random.default_rng(15).standard_normal((F * T, H * D))
    grads = vb.layer_bwd(inp, dy, F, T, C, linear="delta")
    _check_fd(lambda: float((vo.layer(inp, F, T, C, linear="delta")["y"] * dy).sum()), inp, grads,
              NAMES + ("beta",))


@pytest.mark.parametrize("F,T,C,L,H,D,G_l", SHAPES[:2])
def test_branch_gradients_match_finite_differences(F, T, C, L, H, D, G_l):
    """Each branch alone, so a mistake is located at its branch."""
    inp = _inputs(F, T, L, H, D, G_l, seed=3)
    do = np.random.default_rng(8).standard_normal((F * T, H, D))
    names = ("q", "k", "v", "kt", "vt")

    def soft():
        return float((vo.softmax_branch(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"], F, T, C) * do).sum())

    def lin():
        return float((vo.linear_branch(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"], F, T, C) * do).sum())

    g = vb.softmax_branch_bwd(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"], F, T, C, do)
    _check_fd(soft, inp, dict(zip(names, g)), names)
    g = vb.linear_branch_bwd(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"], F, T, C, do)
    _check_fd(lin, inp, dict(zip(names, g)), names)
    inp["beta"] = np.random.default_rng(9).uniform(0.05, 0.95, (F, H))

    def delta():
        return float((vo.delta_branch(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"], inp["beta"], F, T, C)
                      * do).sum())

    g = vb.delta_branch_bwd(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"], inp["beta"], F, T, C, do)
    _check_fd(delta, inp, dict(zip(names + ("beta",), g)), names + ("beta",))


def test_linear_branch_gradients_are_per_head():
    """The linear branch mixes no heads, so its gradients for all heads at once equal those of
    each one-head slice of the inputs (what the full-size GPU check relies on); a head or
    feature axis mixed up anywhere in the backward breaks this."""
    F, T, C, L, H, D = 9, 6, 2, 4, 3, 8
    inp = _inputs(F, T, L, H, D, None, seed=12)
    do = np.random.default_rng(13).standard_normal((F * T, H, D))
    names = ("q", "k", "v", "kt", "vt")
    whole = vb.linear_branch_bwd(*(inp[n] for n in names), F, T, C, do)
    for h in range(H):
        one = vb.linear_branch_bwd(*(inp[n][:, h:h + 1] for n in names), F, T, C, do[:, h:h + 1])
        for a, b in zip(whole, one):
            np.testing.assert_allclose(a[:, h:h + 1], b, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("G_l", [None, 1])
def test_fuse_gradients_match_finite_differences(G_l):
    H, D, n = 2, 4, 5
    rng = np.random.default_rng(4)
    inp = _inputs(1, n, 0, H, D, G_l, seed=5)
    inp["o_s"] = rng.standard_normal((n, H, D))
    inp["o_l"] = rng.standard_normal((n, H, D))
    da = rng.standard_normal((n, 2 * H * D))

    def loss():
        return float((vo.hybrid_fuse(inp["q"], inp["o_s"], inp["o_l"], inp["w_gate_s"], inp["w_gate_l"],
                                     inp["gamma"]) * da).sum())

    dq, do_s, do_l, dws, dwl, dg = vb.hybrid_fuse_bwd(inp["q"], inp["o_s"], inp["o_l"], inp["w_gate_s"],
                                                      inp["w_gate_l"], inp["gamma"], da)
    grads = {"q": dq, "o_s": do_s, "o_l": do_l, "w_gate_s": dws, "w_gate_l": dwl, "gamma": dg}
    _check_fd(loss, inp, grads, tuple(grads))


def test_softmax_gradients_with_every_key_visible_match_torch_autograd():
    """F = 3 frames in one-frame chunks: every query's window spans all frames, so the branch
    is dense attention over [text | video], whose gradient torch's autograd gives."""
    F, T, C, L, H, D = 3, 4, 1, 3, 2, 8
    inp = _inputs(F, T, L, H, D, seed=11)
    do = np.random.default_rng(12).standard_normal((F * T, H, D))
    g = vb.softmax_branch_bwd(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"], F, T, C, do)
    t = {n: torch.tensor(inp[n], dtype=torch.float64, requires_grad=True) for n in ("q", "k", "v", "kt", "vt")}
    K = torch.cat([t["kt"], t["k"]]).transpose(0, 1)          # [H, L + N, D]
    V = torch.cat([t["vt"], t["v"]]).transpose(0, 1)
    o = torch.nn.functional.scaled_dot_product_attention(t["q"].transpose(0, 1), K, V)
    (o.transpose(0, 1) * torch.tensor(do)).sum().backward()
    for n, got in zip(("q", "k", "v", "kt", "vt"), g):
        np.testing.assert_allclose(got, t[n].grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=n)


def test_out_proj_gradients_are_the_transposed_products():
    rng = np.random.default_rng(2)
    n, HD = 6, 8
    a = rng.standard_normal((n, 2 * HD))
    w_os, w_ol = rng.standard_normal((HD, HD)), rng.standard_normal((HD, HD))
    dy = rng.standard_normal((n, HD))
    da, dwos, dwol = vb.out_proj_bwd(a, w_os, w_ol, dy)
    ta = torch.tensor(a, requires_grad=True)
    tws, twl = torch.tensor(w_os, requires_grad=True), torch.tensor(w_ol, requires_grad=True)
    (torch.nn.functional.linear(ta[:, :HD], tws) + torch.nn.functional.linear(ta[:, HD:], twl)).mul(
        torch.tensor(dy)).sum().backward()
    np.testing.assert_allclose(da, ta.grad.numpy(), rtol=1e-12)
    np.testing.assert_allclose(dwos, tws.grad.numpy(), rtol=1e-12)
    np.testing.assert_allclose(dwol, twl.grad.numpy(), rtol=1e-12)


@pytest.mark.parametrize("slip", ["text_once", "rms_sign", "phi_prime", "gate_prime", "no_center",
                                  "delta_transpose"])
def test_planted_backward_mistakes_are_caught(monkeypatch, slip):
    """Plausible slips in the backward oracle fail the finite-difference pin."""
    F, T, C, L, H, D = 7, 2, 2, 3, 1, 4
    inp = _inputs(F, T, L, H, D, seed=21)
    dy = np.random.default_rng(22).standard_normal((F * T, H * D))
    if slip == "text_once":      # text counted in both memories (weight 2 instead of 1)
        orig = vo.text_state
        monkeypatch.setattr(vb.vo, "text_state", lambda kt, vt: tuple(2 * x for x in orig(kt, vt)))
    elif slip == "rms_sign":     # the RMSNorm correction term added instead of subtracted
        orig_fuse = vb.hybrid_fuse_bwd

        def bad(q, o_s, o_l, ws, wl, gamma, da, eps=1e-6):
            out = list(orig_fuse(q, o_s, o_l, ws, wl, gamma, da, eps))
            r = np.sqrt((o_l * o_l).mean(axis=-1, keepdims=True) + eps)
            dn = vo.sigmoid(np.einsum("nhd,hdg->nhg", q, wl)) * da[:, H * D:].reshape(o_l.shape)
            out[2] = out[2] + 2 * o_l * (gamma[None] * o_l * dn).sum(axis=-1, keepdims=True) / (D * r ** 3)
            return tuple(out)
        monkeypatch.setattr(vb, "hybrid_fuse_bwd", bad)
    elif slip == "phi_prime":    # phi' taken as 1 everywhere
        monkeypatch.setattr(vb, "dphi", lambda x: np.ones_like(np.asarray(x, np.float64)))
    elif slip == "gate_prime":   # sigmoid' dropped from the softmax gate's chain rule
        orig_fuse = vb.hybrid_fuse_bwd

        def bad(q, o_s, o_l, ws, wl, gamma, da, eps=1e-6):
            dq, do_s, do_l, dws, dwl, dg = orig_fuse(q, o_s, o_l, ws, wl, gamma, da, eps)
            g_s = vo.sigmoid(np.einsum("nhd,hd->nh", q, ws))
            t = (da[:, :H * D].reshape(o_s.shape) * o_s).sum(axis=-1) * (1.0 - g_s * (1.0 - g_s))
            return dq + t[..., None] * ws[None], do_s, do_l, dws + np.einsum("nh,nhd->hd", t, q), dwl, dg
        monkeypatch.setattr(vb, "hybrid_fuse_bwd", bad)
    elif slip == "no_center":    # the softmax Jacobian without its -dO.o term
        monkeypatch.setattr(vb, "attention_ds", lambda p, dO, o, V: p * (dO @ V.T))
    elif slip == "delta_transpose":  # only one of the two S terms of dkb in the delta step
        orig_step = vb.delta_update_bwd

        def bad(S, kb, vb_, beta, dS1):
            dS, dkb, dvb, dbeta = orig_step(S, kb, vb_, beta, dS1)
            return dS, dkb + np.asarray(beta)[:, None] * np.einsum("hde,hfe,hf->hd", S, dS1, kb), dvb, dbeta
        monkeypatch.setattr(vb, "delta_update_bwd", bad)
    linear = "delta" if slip == "delta_transpose" else "elu1"
    names = NAMES
    if linear == "delta":
        inp["beta"] = np.random.default_rng(23).uniform(0.05, 0.95, (F, H))
        names = NAMES + ("beta",)
    grads = vb.layer_bwd(inp, dy, F, T, C, linear=linear)
    monkeypatch.undo()
    with pytest.raises(AssertionError):
        _check_fd(lambda: float((vo.layer(inp, F, T, C, linear=linear)["y"] * dy).sum()), inp, grads, names)
