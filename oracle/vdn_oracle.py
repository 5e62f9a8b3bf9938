"""Float64 CPU oracle of the VDN-H3 hybrid attention layer, forward pass.

TEST INFRASTRUCTURE.  Only the test suite, the package's smoke check and the benchmark's
CPU-baseline / reference leg may import or run this module.  The CUDA library never calls
it and shares no code with it; it is slow and plain on purpose, so that each function can
be checked against the pages by eye.

Sources (page titles with the section each function follows):
  [ART]  "VDN-MiniMax-H3 开源：全新混合注意力加速视频生成，8步生成，近乎无损画质"
         (ModelScope community article), section 技术解读:
           - "局部精确计算，远程线性记忆" paragraph 1: chunks of 5 latent frames, each chunk
             attends to itself and its two neighbour chunks; first and last frame are
             boundary anchors that every frame reads and that read every frame; the
             linear branch summarises the frames before and after the local window and
             leaves out window and anchor frames so that nothing is counted twice.
           - same section, paragraph 2: the frame-7 illustration (softmax keeps 6, 7, 8
             and anchors 0, 14; forward state holds 1-5, backward state 9-13; both states
             are read at the query position).
           - same section, paragraph 3: text is visible to every frame in the softmax
             branch, and is written half into each linear state so that the merged read
             counts it once.
           - same section, paragraph 4: the simplified figure (16 frames, 2 frames per
             chunk).
           - "独立门控，融合两条注意力分支": a sigmoid gate per branch that depends on the
             input, separate output projections summed into the residual stream; the
             linear output goes through RMSNorm and then an element-wise gate.
  [BLOG] "MiniMax H3 加速五件套" / "H3, accelerated", section "III. VDN: Splitting
         Attention by Distance": the long-range branch is delta-rule linear attention,
         a state matrix updated over time.
  [CARD] "Video DeltaNet: Hybrid Attention to Speed Up Video Models with Near-Lossless
         Quality" (vdn-minimax-h3 model card), "Set up": the local softmax is a window
         softmax.

Readings taken where the pages are silent (the same list is kept with the design notes):
  R1  windows are chunk-granular: chunks c-1, c, c+1 of the query's chunk c;
  R2  chunks start at frame 0 and the last chunk may be short;
  R3  anchor query frames take a softmax over all frames plus text; their linear read
      sees text only;
  R4  an anchor inside the window is one key set member (set union, no duplicates);
  R5  text goes half into each state; one normaliser over the summed numerators and
      denominators, so text weighs exactly 1;
  R6  feature map phi = elu + 1;
  R7  no epsilon in the linear normaliser; an empty key set (no text, no memory) reads 0;
  R8  softmax scale 1/sqrt(D);
  R9  gates are computed from the query of each head: g_s = sigmoid(q . w_s[h]) (scalar
      per token and head), g_l = sigmoid(q W_l[h]) (G_l = D columns: element-wise; G_l = 1:
      scalar); no biases;
  R10 RMSNorm over the D values of one head, learnable gamma, eps = 1e-6;
  R11 only video tokens are queries; text contributes keys and values;
  R12 delta rule with S in R^{Dk x Dv}: S <- (I - beta kb kb^T) S + beta kb vb^T; read S^T q_hat;
  R13 delta inputs: kb = L2-normalised mean key of a frame, vb = mean value of the frame,
      beta per (frame, head) given; text init = 1/2 sum_text k_hat v^T with per-token
      L2-normalised text keys; q_hat = q / ||q||; no read normaliser; a zero vector
      normalises to zero;
  R14 FP8 is not modelled here (the tolerance of the FP8 comparison absorbs it).

Array conventions: video q/k/v [F*T, H, D] frame-major (token t of frame f is row f*T+t);
text kt/vt [L, H, D]; every function works in float64 on whatever it is given.
"""
from __future__ import annotations

import numpy as np

SOFT, FWD, BWD = 0, 1, 2


# ----------------------------------------------------------------------------- layout
def chunk_window(f: int, F: int, C: int) -> tuple[int, int]:
    """Half-open frame range of the local window of query frame f: the chunk holding f and
    the chunks on either side, clipped to [0, F).  [ART] 局部精确计算 para. 1 (R1, R2)."""
    c = f // C
    return max(0, (c - 1) * C), min(F, (c + 2) * C)


def is_anchor(f: int, F: int) -> bool:
    """First and last frame are boundary anchors.  [ART] 局部精确计算 para. 1."""
    return f == 0 or f == F - 1


def frame_mask(F: int, C: int) -> np.ndarray:
    """M[fq, fk]: the branch through which query frame fq reads key frame fk.

    SOFT: fk is in the local window of fq, or either frame is an anchor ([ART] para. 1:
    every frame reads the anchors, the anchors read every frame).  Otherwise fk lies
    before the window (FWD, forward state) or after it (BWD, backward state)."""
    M = np.full((F, F), -1, dtype=np.int8)
    for fq in range(F):
        lo, hi = chunk_window(fq, F, C)
        for fk in range(F):
            if is_anchor(fq, F) or is_anchor(fk, F) or lo <= fk < hi:
                M[fq, fk] = SOFT
            elif fk < lo:
                M[fq, fk] = FWD
            else:
                M[fq, fk] = BWD
    return M


def _range_of(frames: np.ndarray) -> tuple[int, int]:
    """A contiguous run of frames as a half-open range; empty -> (0, 0)."""
    if frames.size == 0:
        return 0, 0
    lo, hi = int(frames[0]), int(frames[-1]) + 1
    assert hi - lo == frames.size, "memory frames must be contiguous"
    return lo, hi


def _soft_segments(soft_frames: np.ndarray, T: int, L: int) -> list[tuple[int, int]]:
    """Softmax key set as sorted, merged, half-open ranges of the concatenated key index
    space [text | video]: text is [0, L), frame f is [L + f*T, L + (f+1)*T)."""
    ranges = ([(0, L)] if L > 0 else []) + [(L + f * T, L + (f + 1) * T) for f in soft_frames]
    ranges.sort()
    merged: list[list[int]] = []
    for lo, hi in ranges:
        if merged and lo <= merged[-1][1]:
            merged[-1][1] = max(merged[-1][1], hi)
        else:
            merged.append([lo, hi])
    return [(a, b) for a, b in merged]


def frame_sets(F: int, T: int, C: int, L: int):
    """Per query frame: (softmax key segments, forward frame range, backward frame range),
    all read off the explicit mask."""
    M = frame_mask(F, C)
    out = []
    for f in range(F):
        segs = _soft_segments(np.nonzero(M[f] == SOFT)[0], T, L)
        out.append((tuple(segs), _range_of(np.nonzero(M[f] == FWD)[0]),
                    _range_of(np.nonzero(M[f] == BWD)[0])))
    return out


MAX_SEGMENTS = 4


def layout_tables(F: int, T: int, C: int, L: int):
    """The canonical layout tables that the library's mask-layout builder must reproduce
    bit for bit.

    frame table int32 [F, 8]: group, win_lo, win_hi, is_anchor, fwd_lo, fwd_hi, bwd_lo,
        bwd_hi.  win is the chunk window (all frames for an anchor); an empty memory range
        is (0, 0).
    group table int32 [G, 16]: frame_lo, frame_hi, n_seg, 0, then 4 (lo, hi) softmax key
        segments in [text | video] index space (unused ones (0, 0)), fwd_lo, fwd_hi,
        bwd_lo, bwd_hi.  A group is a maximal run of consecutive query frames whose three
        sets are identical."""
    sets = frame_sets(F, T, C, L)
    groups: list[list[int]] = []
    gid = np.zeros(F, dtype=np.int32)
    for f in range(F):
        if f > 0 and sets[f] == sets[f - 1]:
            groups[-1][1] = f + 1
        else:
            groups.append([f, f + 1])
        gid[f] = len(groups) - 1
    ftab = np.zeros((F, 8), dtype=np.int32)
    for f in range(F):
        lo, hi = (0, F) if is_anchor(f, F) else chunk_window(f, F, C)
        _, fw, bw = sets[f]
        ftab[f] = [gid[f], lo, hi, int(is_anchor(f, F)), fw[0], fw[1], bw[0], bw[1]]
    gtab = np.zeros((len(groups), 16), dtype=np.int32)
    for g, (flo, fhi) in enumerate(groups):
        segs, fw, bw = sets[flo]
        assert len(segs) <= MAX_SEGMENTS
        row = [flo, fhi, len(segs), 0]
        for s in range(MAX_SEGMENTS):
            row += list(segs[s]) if s < len(segs) else [0, 0]
        row += [fw[0], fw[1], bw[0], bw[1]]
        gtab[g] = row
    return ftab, gtab


# ----------------------------------------------------------------------------- softmax branch
def softmax_branch(q, k, v, kt, vt, F, T, C, scale=None, rows=None):
    """Local softmax branch O_s for the video query rows `rows` (default: all).

    For a query in frame fq the key set is the text plus every token of the frames with
    M[fq, fk] == SOFT ([ART] para. 1 and 3); O_s = softmax(q K^T * scale) V over that set,
    with the row maximum subtracted before exp.  Returns [len(rows), H, D] float64."""
    N, H, D = q.shape
    L = kt.shape[0]
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    M = frame_mask(F, C)
    out = np.zeros((rows.size, H, D))
    for h in range(H):
        kh, vh = np.asarray(k[:, h, :], np.float64), np.asarray(v[:, h, :], np.float64)
        kth, vth = np.asarray(kt[:, h, :], np.float64), np.asarray(vt[:, h, :], np.float64)
        cache = {}
        for fq in range(F):
            sel = np.nonzero(rows // T == fq)[0]
            if sel.size == 0:
                continue
            key_frames = tuple(np.nonzero(M[fq] == SOFT)[0].tolist())
            if key_frames not in cache:
                tok = np.concatenate([np.arange(f * T, (f + 1) * T) for f in key_frames])
                cache[key_frames] = (np.concatenate([kth, kh[tok]]), np.concatenate([vth, vh[tok]]))
            K, V = cache[key_frames]
            s = np.asarray(q[rows[sel], h, :], np.float64) @ K.T * scale
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            out[sel, h, :] = (p @ V) / p.sum(axis=1, keepdims=True)
        del cache
    return out


# ----------------------------------------------------------------------------- linear branch
def phi(x):
    """Feature map elu(x) + 1 (R6): x + 1 for x > 0, exp(x) otherwise."""
    x = np.asarray(x, np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def frame_states(k, v, F, T):
    """Per-frame states S_f = sum_{t in f} phi(k_t)^T v_t  [F, H, D, D] and
    z_f = sum_{t in f} phi(k_t)  [F, H, D] ([ART] para. 1: the linear branch is frame-wise)."""
    N, H, D = k.shape
    S = np.zeros((F, H, D, D))
    z = np.zeros((F, H, D))
    for f in range(F):
        kf = phi(k[f * T:(f + 1) * T])                       # [T, H, D]
        vf = np.asarray(v[f * T:(f + 1) * T], np.float64)    # [T, H, D]
        S[f] = np.matmul(kf.transpose(1, 2, 0), vf.transpose(1, 0, 2))
        z[f] = kf.sum(axis=0)
    return S, z


def text_state(kt, vt):
    """S_txt = sum_text phi(k)^T v  [H, D, D] and z_txt = sum_text phi(k)  [H, D]."""
    kf = phi(kt)
    vf = np.asarray(vt, np.float64)
    return np.matmul(kf.transpose(1, 2, 0), vf.transpose(1, 0, 2)), kf.sum(axis=0)


def linear_memory(k, v, kt, vt, F, T, C):
    """Forward and backward memories of every query frame, each re-summed over its own
    explicit frame set: num_f = 1/2 S_txt + sum_{fk: M=FWD} S_fk, num_b likewise with BWD,
    and the same for the normalisers ([ART] para. 1-3, R5).
    Returns (num_f, num_b, den_f, den_b) with shapes [F, H, D, D] and [F, H, D]."""
    M = frame_mask(F, C)
    S, z = frame_states(k, v, F, T)
    St, zt = text_state(kt, vt)
    H, D = St.shape[0], St.shape[1]
    # sum over the explicit frame set of every query frame: indicator rows times the
    # stacked per-frame states (one matrix product per memory)
    w_f = (M == FWD).astype(np.float64)   # w_f[fq, fk] = 1 if fk is in fq's forward set
    w_b = (M == BWD).astype(np.float64)
    num_f = 0.5 * St[None] + (w_f @ S.reshape(F, -1)).reshape(F, H, D, D)
    num_b = 0.5 * St[None] + (w_b @ S.reshape(F, -1)).reshape(F, H, D, D)
    den_f = 0.5 * zt[None] + (w_f @ z.reshape(F, -1)).reshape(F, H, D)
    den_b = 0.5 * zt[None] + (w_b @ z.reshape(F, -1)).reshape(F, H, D)
    return num_f, num_b, den_f, den_b


def linear_read(q, num_f, num_b, den_f, den_b, T, rows=None):
    """o = phi(q)(num_f + num_b) / (phi(q) . (den_f + den_b)) for the query rows; the two
    memories are read at the query position and merged under one normaliser, so the text
    halves add up to one ([ART] para. 2-3, R5); 0 where the normaliser is 0 (R7)."""
    N, H, D = q.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = np.zeros((rows.size, H, D))
    for f in np.unique(rows // T):
        sel = np.nonzero(rows // T == f)[0]
        pq = phi(q[rows[sel]])                                              # [n, H, D]
        num = np.einsum("nhd,hde->nhe", pq, num_f[f] + num_b[f])
        den = np.einsum("nhd,hd->nh", pq, den_f[f] + den_b[f])[..., None]
        out[sel] = np.where(den > 0, num / np.where(den > 0, den, 1.0), 0.0)
    return out


def linear_branch(q, k, v, kt, vt, F, T, C, rows=None):
    """Linear branch O_l (elu+1 feature map) for the query rows, [n, H, D] float64."""
    return linear_read(q, *linear_memory(k, v, kt, vt, F, T, C), T, rows)


def linear_branch_masked(q, k, v, kt, vt, F, T, C):
    """The same branch written token by token, O(N^2): weights w = 1 for key tokens in
    FWD or BWD frames of the query, 1/2 + 1/2 for text, 0 for softmax frames;
    o = (phi(Q) phi(K)^T * w) V / rowsum(phi(Q) phi(K)^T * w).  Small inputs only."""
    N, H, D = q.shape
    L = kt.shape[0]
    M = frame_mask(F, C)
    fr = np.arange(N) // T
    W = np.zeros((N, L + N))
    W[:, :L] = 0.5 + 0.5
    W[:, L:] = (M[fr][:, fr] != SOFT).astype(np.float64)
    out = np.zeros((N, H, D))
    for h in range(H):
        Kall = np.concatenate([np.asarray(kt[:, h], np.float64), np.asarray(k[:, h], np.float64)])
        Vall = np.concatenate([np.asarray(vt[:, h], np.float64), np.asarray(v[:, h], np.float64)])
        A = (phi(q[:, h]) @ phi(Kall).T) * W
        den = A.sum(axis=1, keepdims=True)
        out[:, h] = np.where(den > 0, (A @ Vall) / np.where(den > 0, den, 1.0), 0.0)
    return out


# ----------------------------------------------------------------------------- delta variant
def l2_normalize(x, axis=-1):
    """x / ||x||_2 along axis; a zero vector stays zero (R13)."""
    x = np.asarray(x, np.float64)
    n = np.sqrt((x * x).sum(axis=axis, keepdims=True))
    return np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)


def delta_frame_stats(k, v, F, T):
    """kb_f = L2-normalised mean key of frame f, vb_f = mean value of frame f; [F, H, D]."""
    N, H, D = k.shape
    kb = np.stack([np.asarray(k[f * T:(f + 1) * T], np.float64).mean(axis=0) for f in range(F)])
    vb = np.stack([np.asarray(v[f * T:(f + 1) * T], np.float64).mean(axis=0) for f in range(F)])
    return l2_normalize(kb), vb


def delta_text_init(kt, vt):
    """S_0 = 1/2 sum_text k_hat v^T, [H, D, D] (R13: text written half into each state)."""
    kh = l2_normalize(kt)
    return 0.5 * np.matmul(kh.transpose(1, 2, 0), np.asarray(vt, np.float64).transpose(1, 0, 2))


def delta_update(S, kb, vb, beta):
    """One delta-rule step on the states of all heads ([BLOG] III; R12):
    S <- (I - beta kb kb^T) S + beta kb vb^T, with S [H, Dk, Dv], kb/vb [H, D], beta [H]."""
    H, D = kb.shape
    b = np.asarray(beta, np.float64)[:, None, None]
    outer_kk = kb[:, :, None] * kb[:, None, :]
    outer_kv = kb[:, :, None] * vb[:, None, :]
    return np.matmul(np.eye(D)[None] - b * outer_kk, S) + b * outer_kv


def delta_memory(k, v, kt, vt, beta, F, T, C):
    """Per query frame, the forward state (recurrence over its FWD frames in ascending
    order) and backward state (its BWD frames in descending order), each started from the
    text init; states are re-run from scratch for every distinct frame set.
    Returns (S_f, S_b) [F, H, D, D]."""
    M = frame_mask(F, C)
    kb, vb = delta_frame_stats(k, v, F, T)
    S0 = delta_text_init(kt, vt)
    beta = np.asarray(beta, np.float64)
    H, D = S0.shape[0], S0.shape[1]
    Sf = np.zeros((F, H, D, D)); Sb = np.zeros((F, H, D, D))
    cache = {}
    for fq in range(F):
        for tgt, frames in ((Sf, np.nonzero(M[fq] == FWD)[0]), (Sb, np.nonzero(M[fq] == BWD)[0][::-1])):
            key = tuple(frames.tolist())
            if key not in cache:
                S = S0.copy()
                for f in frames:
                    S = delta_update(S, kb[f], vb[f], beta[f])
                cache[key] = S
            tgt[fq] = cache[key]
    return Sf, Sb


def delta_read(q, Sf, Sb, T, rows=None):
    """o = (S_f + S_b)^T q_hat with q_hat = q / ||q|| (R12, R13)."""
    N, H, D = q.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = np.zeros((rows.size, H, D))
    for f in np.unique(rows // T):
        sel = np.nonzero(rows // T == f)[0]
        out[sel] = np.einsum("hde,nhd->nhe", Sf[f] + Sb[f], l2_normalize(q[rows[sel]]))
    return out


def delta_branch(q, k, v, kt, vt, beta, F, T, C, rows=None):
    return delta_read(q, *delta_memory(k, v, kt, vt, beta, F, T, C), T, rows)


# ----------------------------------------------------------------------------- fuse + projections
def sigmoid(x):
    x = np.asarray(x, np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def hybrid_fuse(q, o_s, o_l, w_gate_s, w_gate_l, gamma, eps=1e-6):
    """A = [g_s * O_s | g_l * RMSNorm(O_l)]  ([ART] 独立门控; R9, R10).

    g_s = sigmoid(q . w_s[h]) per token and head; g_l = sigmoid(q W_l[h]) with G_l columns
    (D: element-wise, 1: scalar); RMSNorm(x) = gamma * x / sqrt(mean_D(x^2) + eps).
    Shapes: q/o_s/o_l [n, H, D]; w_gate_s [H, D]; w_gate_l [H, D, G_l]; gamma [H, D].
    Returns [n, 2*H*D]: softmax half first, both halves head-major (h*D + d)."""
    q = np.asarray(q, np.float64)
    n, H, D = q.shape
    g_s = sigmoid(np.einsum("nhd,hd->nh", q, np.asarray(w_gate_s, np.float64)))[..., None]
    g_l = sigmoid(np.einsum("nhd,hdg->nhg", q, np.asarray(w_gate_l, np.float64)))
    o_l = np.asarray(o_l, np.float64)
    rms = np.sqrt((o_l * o_l).mean(axis=-1, keepdims=True) + eps)
    nrm = np.asarray(gamma, np.float64)[None] * o_l / rms
    a_s = g_s * np.asarray(o_s, np.float64)
    a_l = g_l * nrm
    return np.concatenate([a_s.reshape(n, H * D), a_l.reshape(n, H * D)], axis=1)


def out_proj(a, w_os, w_ol):
    """y = A_s W_os^T + A_l W_ol^T: separate output projections of the two branches,
    summed ([ART] 独立门控 para. 1).  W [out, in]; no bias; the residual add is the
    caller's."""
    HD = np.asarray(w_os).shape[1]
    a = np.asarray(a, np.float64)
    return a[:, :HD] @ np.asarray(w_os, np.float64).T + a[:, HD:] @ np.asarray(w_ol, np.float64).T


def layer(inp: dict, F, T, C, rows=None, linear="elu1", eps=1e-6, scale=None):
    """The whole layer for the query rows: both branches, fuse, projections.  `inp` holds
    float64-convertible arrays q, k, v, kt, vt, w_gate_s, w_gate_l, gamma, w_os, w_ol
    (and beta for the delta variant).  Returns dict(o_s, o_l, a, y)."""
    q, k, v, kt, vt = (inp[n] for n in ("q", "k", "v", "kt", "vt"))
    N = q.shape[0]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    o_s = softmax_branch(q, k, v, kt, vt, F, T, C, scale, rows)
    if linear == "delta":
        o_l = delta_branch(q, k, v, kt, vt, inp["beta"], F, T, C, rows)
    else:
        o_l = linear_branch(q, k, v, kt, vt, F, T, C, rows)
    a = hybrid_fuse(q[rows], o_s, o_l, inp["w_gate_s"], inp["w_gate_l"], inp["gamma"], eps)
    y = out_proj(a, inp["w_os"], inp["w_ol"])
    return {"o_s": o_s, "o_l": o_l, "a": a, "y": y}
