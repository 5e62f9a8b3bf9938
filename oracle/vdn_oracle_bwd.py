"""Float64 CPU oracle of the VDN-H3 hybrid attention layer, backward pass (elu+1 and
delta-rule linear branches): the gradients of a loss L(y) with respect to every input of
the forward oracle.

TEST INFRASTRUCTURE, like the forward oracle in vdn_oracle.py: only the test suite may
import it; the CUDA library shares no code with it.

The forward it differentiates is vdn_oracle.layer (linear="elu1") term by term, in the
same notation; the pages define only the forward ([ART] 技术解读: 局部精确计算 and
独立门控), so each step below is the chain rule applied to one forward step:

  y     = A_s W_os^T + A_l W_ol^T                            (out_proj)
  A_s   = g_s O_s,  g_s = sigmoid(q . w_s[h])                (hybrid_fuse)
  A_l   = g_l N,    g_l = sigmoid(q W_l[h]),  N = gamma O_l / r,  r = sqrt(mean_D O_l^2 + eps)
  O_s   = sum_j p_j V_j,  p = softmax(scale q K_J^T) over the query's key set J
  O_l   = phi(q) Num / (phi(q) . Den)   (0 where the normaliser is 0, R7; no gradient there)
  Num_f = S_txt + sum_{fk in FWD(f) u BWD(f)} S_fk,  Den_f likewise with z
          (the two text halves of the forward and backward memories add up to one, R5)
  S_fk  = sum_{t in fk} phi(k_t) v_t^T,  z_fk = sum_{t in fk} phi(k_t)
  delta rule ([BLOG] III; R12, R13): O_l = (S_f + S_b)^T q_hat, each memory the recurrence
          S <- S - beta kb (kb^T S) + beta kb vb^T over its frames from
          S_0 = 1/2 sum_text k_hat v^T, with kb = normalised frame-mean key, vb = frame-mean value

phi = elu + 1 has the continuous derivative phi'(x) = 1 for x > 0, e^x otherwise.
The gradients are pinned against central finite differences of the forward oracle and,
for the softmax branch with every key visible, against torch's autograd of dense
attention (tests/test_oracle_bwd_pins.py).
"""
from __future__ import annotations

import numpy as np

from oracle import vdn_oracle as vo


def dphi(x):
    """phi'(x) for phi = elu + 1: 1 for x > 0, e^x otherwise."""
    x = np.asarray(x, np.float64)
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


def out_proj_bwd(a, w_os, w_ol, dy):
    """y = A_s W_os^T + A_l W_ol^T  ->  (dA [n, 2HD], dW_os, dW_ol)."""
    HD = np.asarray(w_os).shape[1]
    a = np.asarray(a, np.float64)
    dy = np.asarray(dy, np.float64)
    da = np.concatenate([dy @ np.asarray(w_os, np.float64), dy @ np.asarray(w_ol, np.float64)], axis=1)
    return da, dy.T @ a[:, :HD], dy.T @ a[:, HD:]


def hybrid_fuse_bwd(q, o_s, o_l, w_gate_s, w_gate_l, gamma, da, eps=1e-6):
    """Backward of A = [g_s O_s | g_l gamma O_l / r] for rows q [n, H, D].
    Returns dq, do_s, do_l [n, H, D], dw_gate_s [H, D], dw_gate_l [H, D, G_l], dgamma [H, D]."""
    q = np.asarray(q, np.float64)
    n, H, D = q.shape
    o_s = np.asarray(o_s, np.float64)
    o_l = np.asarray(o_l, np.float64)
    ws = np.asarray(w_gate_s, np.float64)
    wl = np.asarray(w_gate_l, np.float64)
    gamma = np.asarray(gamma, np.float64)
    da_s = np.asarray(da, np.float64)[:, :H * D].reshape(n, H, D)
    da_l = np.asarray(da, np.float64)[:, H * D:].reshape(n, H, D)
    # softmax half: A_s = g_s O_s with a scalar gate per token and head
    g_s = vo.sigmoid(np.einsum("nhd,hd->nh", q, ws))
    do_s = g_s[..., None] * da_s
    t_s = (da_s * o_s).sum(axis=-1) * g_s * (1.0 - g_s)              # d(q . w_s) [n, H]
    dq = t_s[..., None] * ws[None]
    dws = np.einsum("nh,nhd->hd", t_s, q)
    # linear half: A_l = g_l N, g_l with G_l columns (D: element-wise, 1: broadcast)
    g_l = vo.sigmoid(np.einsum("nhd,hdg->nhg", q, wl))
    r = np.sqrt((o_l * o_l).mean(axis=-1, keepdims=True) + eps)       # [n, H, 1]
    nrm = gamma[None] * o_l / r
    dn = g_l * da_l                                                    # dN
    dg = da_l * nrm if wl.shape[2] == D else (da_l * nrm).sum(axis=-1, keepdims=True)
    t_l = dg * g_l * (1.0 - g_l)                                       # d(q W_l) [n, H, G_l]
    dq = dq + np.einsum("nhg,hdg->nhd", t_l, wl)
    dwl = np.einsum("nhd,nhg->hdg", q, t_l)
    # RMSNorm: N_d = gamma_d x_d / r, dr/dx_e = x_e / (D r)
    dgamma = np.einsum("nhd,nhd->hd", dn, o_l / r)
    do_l = gamma[None] * dn / r - o_l * (gamma[None] * o_l * dn).sum(axis=-1, keepdims=True) / (D * r ** 3)
    return dq, do_s, do_l, dws, dwl, dgamma


def attention_ds(p, dO, o, V):
    """Gradient of the scores of o = p V, p = softmax(s): ds_j = p_j (dO . V_j - dO . o)."""
    return p * (dO @ V.T - (dO * o).sum(axis=1, keepdims=True))


def softmax_branch_bwd(q, k, v, kt, vt, F, T, C, do_s, scale=None):
    """Backward of the local softmax branch for all video query rows: with p = softmax(s)
    over the key set, ds_j = p_j (dO . V_j - dO . O).  Returns dq [N, H, D], dk, dv
    [N, H, D], dkt, dvt [L, H, D]."""
    N, H, D = q.shape
    L = kt.shape[0]
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    M = vo.frame_mask(F, C)
    dq = np.zeros((N, H, D)); dk = np.zeros((N, H, D)); dv = np.zeros((N, H, D))
    dkt = np.zeros((L, H, D)); dvt = np.zeros((L, H, D))
    for h in range(H):
        kh, vh = np.asarray(k[:, h], np.float64), np.asarray(v[:, h], np.float64)
        kth, vth = np.asarray(kt[:, h], np.float64), np.asarray(vt[:, h], np.float64)
        for fq in range(F):
            rows = np.arange(fq * T, (fq + 1) * T)
            tok = np.concatenate([np.arange(f * T, (f + 1) * T) for f in np.nonzero(M[fq] == vo.SOFT)[0]])
            K = np.concatenate([kth, kh[tok]])
            V = np.concatenate([vth, vh[tok]])
            qr = np.asarray(q[rows, h], np.float64)
            s = qr @ K.T * scale
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            o = p @ V
            dO = np.asarray(do_s[rows, h], np.float64)
            ds = attention_ds(p, dO, o, V)
            dq[rows, h] += scale * ds @ K
            dK = scale * ds.T @ qr
            dV = p.T @ dO
            dkt[:, h] += dK[:L]; dvt[:, h] += dV[:L]
            np.add.at(dk[:, h], tok, dK[L:])
            np.add.at(dv[:, h], tok, dV[L:])
    return dq, dk, dv, dkt, dvt


def linear_branch_bwd(q, k, v, kt, vt, F, T, C, do_l):
    """Backward of the elu+1 linear branch for all video query rows.
    Per row: o = num / den, num = phi(q) Num_f, den = phi(q) . Den_f; dnum = dO / den,
    dden = -(dO . o) / den; d phi(q) = Num_f dnum + Den_f dden; dNum_f = phi(q)^T dnum,
    dDen_f = phi(q) dden; then through the frame sums and S_fk = sum phi(k) v^T.
    Returns dq, dk, dv [N, H, D], dkt, dvt [L, H, D]."""
    N, H, D = q.shape
    L = kt.shape[0]
    M = vo.frame_mask(F, C)
    S, z = vo.frame_states(k, v, F, T)
    St, zt = vo.text_state(kt, vt)
    mem = ((M == vo.FWD) | (M == vo.BWD)).astype(np.float64)           # mem[fq, fk]
    Num = St[None] + (mem @ S.reshape(F, -1)).reshape(F, H, D, D)
    Den = zt[None] + (mem @ z.reshape(F, -1)).reshape(F, H, D)
    dq = np.zeros((N, H, D))
    dNum = np.zeros((F, H, D, D)); dDen = np.zeros((F, H, D))
    for f in range(F):
        rows = np.arange(f * T, (f + 1) * T)
        qr = np.asarray(q[rows], np.float64)
        pq = vo.phi(qr)                                                  # [T, H, D]
        num = np.einsum("nhd,hde->nhe", pq, Num[f])
        den = np.einsum("nhd,hd->nh", pq, Den[f])[..., None]
        live = den > 0
        o = np.where(live, num / np.where(live, den, 1.0), 0.0)
        dO = np.asarray(do_l[rows], np.float64)
        dnum = np.where(live, dO / np.where(live, den, 1.0), 0.0)
        dden = np.where(live, -(dO * o).sum(axis=-1, keepdims=True) / np.where(live, den, 1.0), 0.0)
        dpq = np.einsum("hde,nhe->nhd", Num[f], dnum) + Den[f][None] * dden
        dq[rows] = dpq * dphi(qr)
        dNum[f] = np.einsum("nhd,nhe->hde", pq, dnum)
        dDen[f] = (pq * dden).sum(axis=0)
    # Num_f = S_txt + sum_{fk in mem(f)} S_fk
    dSt = dNum.sum(axis=0); dzt = dDen.sum(axis=0)
    dS = (mem.T @ dNum.reshape(F, -1)).reshape(F, H, D, D)
    dz = (mem.T @ dDen.reshape(F, -1)).reshape(F, H, D)
    dk = np.zeros((N, H, D)); dv = np.zeros((N, H, D))
    for f in range(F):
        rows = np.arange(f * T, (f + 1) * T)
        kr = np.asarray(k[rows], np.float64)
        pk = vo.phi(kr)
        vr = np.asarray(v[rows], np.float64)
        dpk = np.einsum("hde,nhe->nhd", dS[f], vr) + dz[f][None]
        dk[rows] = dpk * dphi(kr)
        dv[rows] = np.einsum("hde,nhd->nhe", dS[f], pk)
    ktr, vtr = np.asarray(kt, np.float64), np.asarray(vt, np.float64)
    dkt = (np.einsum("hde,nhe->nhd", dSt, vtr) + dzt[None]) * dphi(ktr)
    dvt = np.einsum("hde,nhd->nhe", dSt, vo.phi(ktr))
    return dq, dk, dv, dkt, dvt


def l2_normalize_bwd(x, dy, axis=-1):
    """y = x / ||x||  ->  dx = (dy - y (y . dy)) / ||x||; zero where x is zero (R13)."""
    x = np.asarray(x, np.float64)
    n = np.sqrt((x * x).sum(axis=axis, keepdims=True))
    y = np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)
    g = dy - y * (y * dy).sum(axis=axis, keepdims=True)
    return np.where(n > 0, g / np.where(n > 0, n, 1.0), 0.0)


def delta_update_bwd(S, kb, vb, beta, dS1):
    """Backward of one delta step S1 = S - beta kb (kb^T S) + beta kb vb^T (all heads):
    dS = (I - beta kb kb^T) dS1 (the factor is symmetric);
    dkb = -beta (dS1 S^T + S dS1^T) kb + beta dS1 vb;  dvb = beta dS1^T kb;
    dbeta = kb^T dS1 (vb - S^T kb).  Shapes S, dS1 [H, D, D]; kb, vb [H, D]; beta [H]."""
    H, D = kb.shape
    b = np.asarray(beta, np.float64)
    A = np.eye(D)[None] - b[:, None, None] * kb[:, :, None] * kb[:, None, :]
    dS = np.matmul(A, dS1)
    Stk = np.einsum("hde,hd->he", S, kb)                                  # S^T kb
    dkb = (-b[:, None] * (np.einsum("hde,hfe,hf->hd", dS1, S, kb) + np.einsum("hde,hfe,hf->hd", S, dS1, kb))
           + b[:, None] * np.einsum("hde,he->hd", dS1, vb))
    dvb = b[:, None] * np.einsum("hde,hd->he", dS1, kb)
    dbeta = np.einsum("hd,hde,he->h", kb, dS1, vb - Stk)
    return dS, dkb, dvb, dbeta


def delta_branch_bwd(q, k, v, kt, vt, beta, F, T, C, do_l):
    """Backward of the delta-rule linear branch for all video query rows
    (o = (S_f + S_b)^T q_hat, [BLOG] III; R12, R13).  The memory gradient of every distinct
    frame sequence is summed over the query frames that read it and taken back through
    its recurrence once, to the text init, the frame statistics and beta.
    Returns dq, dk, dv [N, H, D], dkt, dvt [L, H, D], dbeta [F, H]."""
    N, H, D = q.shape
    L = kt.shape[0]
    M = vo.frame_mask(F, C)
    kb_raw = np.stack([np.asarray(k[f * T:(f + 1) * T], np.float64).mean(axis=0) for f in range(F)])
    kb, vb = vo.delta_frame_stats(k, v, F, T)
    S0 = vo.delta_text_init(kt, vt)
    beta = np.asarray(beta, np.float64)
    Sf, Sb = vo.delta_memory(k, v, kt, vt, beta, F, T, C)
    dq = np.zeros((N, H, D))
    dmem = {}                                                            # frame sequence -> dS
    for f in range(F):
        rows = np.arange(f * T, (f + 1) * T)
        qr = np.asarray(q[rows], np.float64)
        qh = vo.l2_normalize(qr)
        dO = np.asarray(do_l[rows], np.float64)
        dq[rows] = l2_normalize_bwd(qr, np.einsum("hde,nhe->nhd", Sf[f] + Sb[f], dO))
        dS = np.einsum("nhd,nhe->hde", qh, dO)
        for frames in (np.nonzero(M[f] == vo.FWD)[0], np.nonzero(M[f] == vo.BWD)[0][::-1]):
            key = tuple(frames.tolist())
            dmem[key] = dmem.get(key, 0.0) + dS
    dS0 = np.zeros((H, D, D)); dkb = np.zeros((F, H, D)); dvb = np.zeros((F, H, D)); dbeta = np.zeros((F, H))
    for key, dS in dmem.items():
        states = [S0]
        for f in key:
            states.append(vo.delta_update(states[-1], kb[f], vb[f], beta[f]))
        for i in range(len(key) - 1, -1, -1):
            f = key[i]
            dS, gk, gv, gb = delta_update_bwd(states[i], kb[f], vb[f], beta[f], dS)
            dkb[f] += gk; dvb[f] += gv; dbeta[f] += gb
        dS0 += dS
    # frame statistics: kb = normalise(mean k), vb = mean v
    dkraw = l2_normalize_bwd(kb_raw, dkb)
    dk = np.repeat(dkraw / T, T, axis=0)
    dv = np.repeat(dvb / T, T, axis=0)
    # text init S0 = 1/2 sum k_hat v^T
    ktr, vtr = np.asarray(kt, np.float64), np.asarray(vt, np.float64)
    kth = vo.l2_normalize(ktr)
    dkt = l2_normalize_bwd(ktr, 0.5 * np.einsum("hde,nhe->nhd", dS0, vtr))
    dvt = 0.5 * np.einsum("hde,nhd->nhe", dS0, kth)
    return dq, dk, dv, dkt, dvt, dbeta


def layer_bwd(inp: dict, dy, F, T, C, eps=1e-6, scale=None, linear="elu1") -> dict:
    """Gradients of sum(y * dy) for the whole layer over all video rows, with respect to
    q, k, v, kt, vt, w_gate_s, w_gate_l, gamma, w_os, w_ol (and beta for the delta rule)."""
    q, k, v, kt, vt = (np.asarray(inp[n], np.float64) for n in ("q", "k", "v", "kt", "vt"))
    fwd = vo.layer(inp, F, T, C, linear=linear, eps=eps, scale=scale)
    da, dwos, dwol = out_proj_bwd(fwd["a"], inp["w_os"], inp["w_ol"], dy)
    dq, do_s, do_l, dws, dwl, dgamma = hybrid_fuse_bwd(q, fwd["o_s"], fwd["o_l"], inp["w_gate_s"], inp["w_gate_l"],
                                                       inp["gamma"], da, eps)
    sq, sk, sv, skt, svt = softmax_branch_bwd(q, k, v, kt, vt, F, T, C, do_s, scale)
    out = {"w_gate_s": dws, "w_gate_l": dwl, "gamma": dgamma, "w_os": dwos, "w_ol": dwol}
    if linear == "delta":
        lq, lk, lv, lkt, lvt, out["beta"] = delta_branch_bwd(q, k, v, kt, vt, inp["beta"], F, T, C, do_l)
    else:
        lq, lk, lv, lkt, lvt = linear_branch_bwd(q, k, v, kt, vt, F, T, C, do_l)
    out.update(q=dq + sq + lq, k=sk + lk, v=sv + lv, kt=skt + lkt, vt=svt + lvt)
    return out
