"""GPU parity of every C-ABI entry point against the float64 oracle, on seeded inputs.

Configurations 1 and 2 are compared on every output element; 3 and 4 (full size) on
sampled query rows (first, last and six random tokens of every frame, all heads, all
output columns) plus every per-group memory state.  Edge shapes cover a ragged last
chunk, no text, frame sizes that are not a multiple of the 128-row tile, everything
inside one window, single frames and the scalar linear gate."""
import numpy as np
import pytest
import torch

import hybrid_softmax_linear_b200 as vdn
from hybrid_softmax_linear_b200 import synth
from hybrid_softmax_linear_b200.tensors import to_device, to_numpy, empty, workspace
from oracle import vdn_oracle as vo
from _harness import Run, assert_close, cfg_inputs, oracle_inputs, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    vdn.lib()


def _group_rows(gtab, T):
    return [(int(r[0]) * T, int(r[1]) * T) for r in gtab]


def _check_tables(run: Run):
    s = run.shape
    ftab, gtab = vdn.mask_layout_build(s)
    meta = run.intermediate(8, (2,), torch.int32).cpu().numpy()
    G, n = int(meta[0]), int(meta[1])
    assert G == len(gtab)
    np.testing.assert_array_equal(run.intermediate(5, (s.frames, 8), torch.int32).cpu().numpy(), ftab)
    np.testing.assert_array_equal(run.intermediate(6, (G, 16), torch.int32).cpu().numpy(), gtab)
    tiles = run.intermediate(7, (n, 8), torch.int32).cpu().numpy()
    covered = np.zeros(s.n_video, np.int32)
    for i, (g, lo, hi, keys, first, count, _, _) in enumerate(tiles):
        assert first <= i < first + count and all(tiles[first:first + count, 0] == g)
        assert 0 < hi - lo <= 256
        flo, fhi = gtab[g][0] * s.tokens_per_frame, gtab[g][1] * s.tokens_per_frame
        assert flo <= lo < hi <= fhi
        assert keys == sum(gtab[g][5 + 2 * i] - gtab[g][4 + 2 * i] for i in range(gtab[g][2]))
        covered[lo:hi] += 1
    assert (covered == 1).all()
    assert all(tiles[i][3] >= tiles[i + 1][3] for i in range(n - 1)), "tiles not longest-first"
    _check_scan_plan(run, gtab)


def _check_scan_plan(run: Run, gtab):
    """Segments of the frames [1, F-1) cut at every memory boundary; each group's
    forward memory [1, e) and backward memory [b, F-1) are unions of whole segments."""
    s = run.shape
    F, G = s.frames, len(gtab)
    gcap = vdn.max_groups(s)
    plan = run.intermediate(9, (4 + F + 1 + 2 * gcap,), torch.int32).cpu().numpy()
    nseg = int(plan[0])
    assert int(plan[1]) == G
    ends = [int(r[13]) if r[13] > r[12] else 1 for r in gtab]
    starts = [int(r[14]) if r[15] > r[14] else F - 1 for r in gtab]
    if F < 3:
        assert nseg == 0
        return
    bnd = sorted(set([1, F - 1] + ends + starts))
    assert nseg == len(bnd) - 1
    np.testing.assert_array_equal(plan[4:4 + nseg + 1], bnd)
    ie, ib = plan[4 + F + 1:4 + F + 1 + G], plan[4 + F + 1 + gcap:4 + F + 1 + gcap + G]
    for g in range(G):
        assert bnd[ie[g]] == ends[g] and bnd[ib[g]] == starts[g]


def _layer_parity(run: Run, rows, kind_tol, check_states=True):
    s, inp = run.shape, run.inp
    F, T, C = s.frames, s.tokens_per_frame, s.chunk_frames
    o = oracle_inputs(inp)
    tdt = torch.float32 if run.dtype == "f32" else torch.bfloat16
    y = run.layer()
    Nv, H, D = run.Nv, run.H, run.D
    rows_t = torch.from_numpy(rows).cuda()
    A = to_numpy(run.intermediate(2, (Nv, 2 * H * D), tdt)[rows_t])
    yr = to_numpy(y[rows_t])
    _check_tables(run)
    # each step against the oracle of that step
    ref_os = vo.softmax_branch(o["q"], o["k"], o["v"], o["kt"], o["vt"], F, T, C, rows=rows)
    if run.kind == vdn.DELTA:
        ref_ol = vo.delta_branch(o["q"], o["k"], o["v"], o["kt"], o["vt"], o["beta"], F, T, C, rows=rows)
    else:
        ref_ol = vo.linear_branch(o["q"], o["k"], o["v"], o["kt"], o["vt"], F, T, C, rows=rows)
    if run.materialises_branches():
        Os = to_numpy(run.intermediate(0, (Nv, H, D), tdt)[rows_t])
        Ol = to_numpy(run.intermediate(1, (Nv, H, D), tdt)[rows_t])
        assert_close("O_s", Os, ref_os, kind_tol)
        assert_close("O_l", Ol, ref_ol, kind_tol)
        ref_a_dev = vo.hybrid_fuse(o["q"][rows], Os, Ol, o["w_gate_s"], o["w_gate_l"], o["gamma"], 1e-6)
        assert_close("A (fuse of device O_s, O_l)", A, ref_a_dev, kind_tol)
    else:
        # fused path: O_s and O_l never leave the kernels; each half of A is checked
        # against the oracle of its branch followed by the gate (and RMSNorm)
        ref_a = vo.hybrid_fuse(o["q"][rows], ref_os, ref_ol, o["w_gate_s"], o["w_gate_l"], o["gamma"], 1e-6)
        HD = H * D
        assert_close("A_s (softmax branch + gate)", A[:, :HD], ref_a[:, :HD], kind_tol)
        assert_close("A_l (linear branch + RMSNorm + gate)", A[:, HD:], ref_a[:, HD:], kind_tol)
    assert_close("y (projection of device A)", yr, vo.out_proj(A, o["w_os"], o["w_ol"]), kind_tol)
    # the whole layer, float64 from the inputs
    ref_a = vo.hybrid_fuse(o["q"][rows], ref_os, ref_ol, o["w_gate_s"], o["w_gate_l"], o["gamma"], 1e-6)
    assert_close("A (layer)", A, ref_a, kind_tol)
    assert_close("y (layer)", yr, vo.out_proj(ref_a, o["w_os"], o["w_ol"]), kind_tol)
    # the fused ELU1 layer keeps only S_fwd + S_bwd (bf16); A_l above checks it
    stored = vdn.hybrid_attn_intermediate(s, run.kind, run.cdt, run.ws, 3) != 0
    if check_states and run.kind == vdn.ELU1 and stored:
        _, gtab = vdn.mask_layout_build(s)
        G = len(gtab)
        num_f, num_b, den_f, den_b = vo.linear_memory(o["k"], o["v"], o["kt"], o["vt"], F, T, C)
        first = [int(r[0]) for r in gtab]
        Sf = run.intermediate(3, (G, H, D, D), torch.float32).cpu().numpy()
        Sb = run.intermediate(4, (G, H, D, D), torch.float32).cpu().numpy()
        # fp32 sums; on the tensor-core path phi(k) enters the MMA in bf16
        state_tol = 1e-5 if run.dtype == "f32" else 5e-3
        assert rel_l2(Sf, num_f[first]) <= state_tol
        assert rel_l2(Sb, num_b[first]) <= state_tol


# ----------------------------------------------------------------------------- configurations
def test_config1_tiny_f32_full():
    w = synth.CONFIGS[1]
    run = Run(w.shape, cfg_inputs(1), w.dtype)
    _layer_parity(run, np.arange(w.shape.n_video), "f32")


def test_config2_small_bf16_full():
    w = synth.CONFIGS[2]
    run = Run(w.shape, cfg_inputs(2), w.dtype)
    _layer_parity(run, np.arange(w.shape.n_video), "bf16")


def test_config3_medium_heavy_tailed_keys_sampled():
    w = synth.CONFIGS[3]
    run = Run(w.shape, cfg_inputs(3), w.dtype)
    _layer_parity(run, synth.sample_rows(w.shape), "bf16")


def test_config4_full_size_sampled():
    w = synth.CONFIGS[4]
    run = Run(w.shape, cfg_inputs(4), w.dtype)
    _layer_parity(run, synth.sample_rows(w.shape), "bf16")


# ----------------------------------------------------------------------------- edge shapes
EDGE = [
    # F, T, C, L, H, D, dtype
    (87, 40, 5, 16, 2, 64, "bf16"),    # ragged last chunk (87 = 17*5 + 2)
    (20, 100, 5, 0, 2, 128, "bf16"),   # no text; T not a multiple of 128
    (30, 50, 5, 8, 3, 64, "bf16"),     # T < 128: tiles hold several frames
    (12, 33, 5, 5, 2, 32, "bf16"),     # F <= 3C, every frame in the window; D = 32
    (12, 33, 5, 5, 4, 32, "bf16"),     # the same with four heads: one 128-feature head group
    (1, 70, 5, 3, 2, 64, "bf16"),      # a single frame (both anchors)
    (2, 70, 5, 0, 1, 64, "f32"),       # two anchors, no text
    (9, 17, 1, 2, 2, 32, "f32"),       # one-frame chunks, odd T
    (40, 129, 3, 130, 2, 128, "bf16"), # text longer than a tile; T = 128 + 1
]


@pytest.mark.parametrize("edge", EDGE)
def test_edge_shapes(edge):
    F, T, C, L, H, D, dt = edge
    shape = synth.Shape(F, T, C, L, H, D)
    inp = synth.make_inputs(shape, dt, seed=1000 + F * 7 + T)
    run = Run(shape, inp, dt)
    _layer_parity(run, np.arange(shape.n_video), dt)


def test_scalar_linear_gate():
    shape = synth.Shape(16, 64, 5, 8, 2, 64)
    inp = synth.make_inputs(shape, "bf16", seed=5, gate_l_cols=1)
    run = Run(shape, inp, "bf16")
    _layer_parity(run, np.arange(shape.n_video), "bf16")


# ----------------------------------------------------------------------------- step entry points
@pytest.mark.parametrize("shape", [None, (12, 300, 5, 40, 2, 128)])
def test_step_entry_points_match_oracle(shape):
    if shape is None:
        s, inp = synth.CONFIGS[2].shape, cfg_inputs(2)
    else:
        s = synth.Shape(*shape)
        inp = synth.make_inputs(s, "bf16", seed=4242)
    F, T, C, L, H, D = s.frames, s.tokens_per_frame, s.chunk_frames, s.text_tokens, s.heads, s.head_dim
    # states: fp32 sums; the tensor-core state build (bf16, D = 128, or D = 64 or 32 in whole
    # 128-feature head groups) feeds phi(k) to the MMA in bf16
    st_tol = 5e-3 if D == 128 or (D in (32, 64) and (H * D) % 128 == 0) else 1e-5
    Nv = s.n_video
    o = oracle_inputs(inp)
    d = {n: to_device(a) for n, a in inp.items()}
    ws = workspace(vdn.step_workspace_size(s))
    vdn.workspace_init(ws)
    o_s = empty((Nv, H, D), "bf16")
    lse = torch.empty((Nv, H), dtype=torch.float32, device="cuda")
    vdn.softmax_branch_fwd(s, vdn.BF16, d["q"], d["k"], d["v"], d["kt"], d["vt"], o_s, ws, lse=lse)
    ref = vo.softmax_branch(o["q"], o["k"], o["v"], o["kt"], o["vt"], F, T, C)
    assert_close("softmax_branch_fwd", to_numpy(o_s), ref, "bf16")
    # lse: log-sum-exp of the scaled scores, checked on a few rows by direct evaluation
    M = vo.frame_mask(F, C)
    for r in (0, 1, T * 7 + 3, Nv - 1):
        f = r // T
        tok = np.concatenate([np.arange(fk * T, (fk + 1) * T) for fk in np.nonzero(M[f] == vo.SOFT)[0]])
        for h in range(H):
            K = np.concatenate([o["kt"][:, h], o["k"][tok, h]]).astype(np.float64)
            sc = K @ o["q"][r, h].astype(np.float64) / np.sqrt(D)
            ref_lse = sc.max() + np.log(np.exp(sc - sc.max()).sum())
            assert abs(lse[r, h].item() - ref_lse) < 1e-3
    S = torch.empty((F, H, D, D), dtype=torch.float32, device="cuda")
    z = torch.empty((F, H, D), dtype=torch.float32, device="cuda")
    St = torch.empty((H, D, D), dtype=torch.float32, device="cuda")
    zt = torch.empty((H, D), dtype=torch.float32, device="cuda")
    vdn.linear_state_build(s, vdn.ELU1, vdn.BF16, d["k"], d["v"], d["kt"], d["vt"], S, z, St, zt, ws)
    rS, rz = vo.frame_states(o["k"], o["v"], F, T)
    rSt, rzt = vo.text_state(o["kt"], o["vt"])
    assert rel_l2(S.cpu().numpy(), rS) < st_tol and rel_l2(z.cpu().numpy(), rz) < 1e-5
    assert rel_l2(St.cpu().numpy(), rSt) < st_tol and rel_l2(zt.cpu().numpy(), rzt) < 1e-5
    G = vdn.max_groups(s)
    Sf, Sb = (torch.empty((G, H, D, D), dtype=torch.float32, device="cuda") for _ in range(2))
    zf, zb = (torch.empty((G, H, D), dtype=torch.float32, device="cuda") for _ in range(2))
    vdn.linear_state_scan(s, vdn.ELU1, S, z, St, zt, None, Sf, Sb, zf, zb, ws)
    _, gtab = vdn.mask_layout_build(s)
    first = [int(r[0]) for r in gtab]
    nf, nb, df, db = vo.linear_memory(o["k"], o["v"], o["kt"], o["vt"], F, T, C)
    ng = len(gtab)
    assert rel_l2(Sf[:ng].cpu().numpy(), nf[first]) < st_tol and rel_l2(Sb[:ng].cpu().numpy(), nb[first]) < st_tol
    assert rel_l2(zf[:ng].cpu().numpy(), df[first]) < 1e-5 and rel_l2(zb[:ng].cpu().numpy(), db[first]) < 1e-5
    o_l = empty((Nv, H, D), "bf16")
    vdn.linear_read(s, vdn.ELU1, vdn.BF16, d["q"], Sf, Sb, zf, zb, o_l, ws)
    ref_l = vo.linear_read(o["q"], nf, nb, df, db, T)
    assert_close("linear_read", to_numpy(o_l), ref_l, "bf16")
    a = empty((Nv, 2 * H * D), "bf16")
    vdn.hybrid_fuse(s, vdn.BF16, d["q"], o_s, o_l, d["w_gate_s"], d["w_gate_l"], D, d["gamma"], 1e-6, a)
    ref_a = vo.hybrid_fuse(o["q"], to_numpy(o_s), to_numpy(o_l), o["w_gate_s"], o["w_gate_l"], o["gamma"], 1e-6)
    assert_close("hybrid_fuse", to_numpy(a), ref_a, "bf16")
    y = empty((Nv, H * D), "bf16")
    vdn.out_proj(s, vdn.BF16, a, d["w_os"], d["w_ol"], y, ws)
    assert_close("out_proj", to_numpy(y), vo.out_proj(to_numpy(a), o["w_os"], o["w_ol"]), "bf16")
    vdn.check_device_status(ws)


@pytest.mark.parametrize("shape", [(130, 4, 1, 3, 1, 32),    # 127 segments: the per-frame walk
                                   (87, 6, 5, 2, 2, 64),     # ragged last chunk
                                   (3, 5, 1, 0, 1, 32),      # a single segment, no text
                                   (2, 5, 5, 4, 1, 32)])     # no frame outside the anchors
def test_state_scan_layouts(shape):
    s = synth.Shape(*shape)
    F, T, C, L, H, D = shape
    inp = synth.make_inputs(s, "f32", seed=77 + F)
    o = oracle_inputs(inp)
    d = {n: to_device(a) for n, a in inp.items()}
    ws = workspace(vdn.step_workspace_size(s))
    vdn.workspace_init(ws)
    S = torch.empty((F, H, D, D), dtype=torch.float32, device="cuda")
    z = torch.empty((F, H, D), dtype=torch.float32, device="cuda")
    St = torch.empty((H, D, D), dtype=torch.float32, device="cuda")
    zt = torch.empty((H, D), dtype=torch.float32, device="cuda")
    vdn.linear_state_build(s, vdn.ELU1, vdn.F32, d["k"], d["v"], d["kt"], d["vt"], S, z, St, zt, ws)
    G = vdn.max_groups(s)
    Sf, Sb = (torch.full((G, H, D, D), float("nan"), device="cuda") for _ in range(2))
    zf, zb = (torch.full((G, H, D), float("nan"), device="cuda") for _ in range(2))
    vdn.linear_state_scan(s, vdn.ELU1, S, z, St, zt, None, Sf, Sb, zf, zb, ws)
    vdn.check_device_status(ws)
    _, gtab = vdn.mask_layout_build(s)
    first = [int(r[0]) for r in gtab]
    nf, nb, df, db = vo.linear_memory(o["k"], o["v"], o["kt"], o["vt"], F, T, C)
    ng = len(gtab)
    for got, ref in ((Sf, nf), (Sb, nb), (zf, df), (zb, db)):
        assert rel_l2(got[:ng].cpu().numpy(), ref[first]) < 1e-5


# ----------------------------------------------------------------------------- bounded device wait
def test_bounded_wait_reports_timeout_and_context_survives():
    ws = workspace(4096)
    vdn.workspace_init(ws)
    vdn.debug_unset_flag_wait(ws, 2000)
    with pytest.raises(vdn.VdnError) as e:
        vdn.check_device_status(ws)
    assert e.value.status == 5
    vdn.check_device_status(ws)          # cleared after the read
    # the context still runs work afterwards
    w = synth.CONFIGS[1]
    run = Run(w.shape, cfg_inputs(1), w.dtype)
    y = run.layer()
    assert torch.isfinite(y).all()


# ----------------------------------------------------------------------------- host-buffer entry point
@pytest.mark.parametrize("kind_dtype", [(vdn.ELU1, vdn.BF16), (vdn.DELTA, vdn.E4M3)])
def test_host_entry_point_matches_device_entry_point(kind_dtype):
    kind, cdt = kind_dtype
    s = synth.Shape(12, 300, 5, 40, 2, 128)
    inp = synth.make_inputs(s, "bf16", seed=99, with_beta=kind == vdn.DELTA)
    run = Run(s, inp, "bf16", kind=kind, layer_dtype=cdt)
    y_dev = to_numpy(run.layer())
    names = ["q", "k", "v", "kt", "vt"] + (["beta"] if kind == vdn.DELTA else [])
    host = {n: torch.from_numpy(inp[n].view(np.int16) if inp[n].dtype == np.uint16 else inp[n]).pin_memory()
            for n in names}
    y_host = torch.empty((s.n_video, s.hidden), dtype=torch.int16).pin_memory()
    ws = workspace(vdn.hybrid_attn_host_workspace_size(s, kind, cdt))
    assert ws.numel() > vdn.hybrid_attn_workspace_size(s, kind, cdt)
    vdn.workspace_init(ws)
    stream = torch.cuda.Stream()
    d = run.dev
    vdn.hybrid_attn_fwd_host(s, kind, cdt, host["q"], host["k"], host["v"], host["kt"], host["vt"], host.get("beta"),
                             d["w_gate_s"], d["w_gate_l"], run.G_l, d["gamma"], 1e-6, d["w_os"], d["w_ol"], y_host, ws,
                             stream)
    stream.synchronize()
    vdn.check_device_status(ws)
    got = synth.bf16_bits_to_f32(y_host.numpy().view(np.uint16))
    assert np.array_equal(got, y_dev)  # the same kernels on the same inputs: the same bits
    ref = vo.layer(oracle_inputs(inp), s.frames, s.tokens_per_frame, s.chunk_frames, rows=np.arange(s.n_video),
                   linear="delta" if kind == vdn.DELTA else "elu1")
    assert rel_l2(got, ref["y"]) <= (3e-2 if cdt == vdn.E4M3 else 5e-3)


# ----------------------------------------------------------------------------- repeatability
@pytest.mark.parametrize("kind_dtype", [(vdn.ELU1, vdn.BF16), (vdn.DELTA, vdn.E4M3)])
def test_layer_repeats_bit_for_bit(kind_dtype):
    """Every reduction has a fixed order (no floating-point atomics), so the same call on the
    same inputs gives the same bits: 24 frames of 1008 tokens, 8 heads of 128."""
    kind, cdt = kind_dtype
    s = synth.Shape(24, 1008, 5, 128, 8, 128)
    inp = synth.make_inputs(s, "bf16", seed=31, with_beta=kind == vdn.DELTA)
    run = Run(s, inp, "bf16", kind=kind, layer_dtype=cdt)
    y0 = run.layer()
    for _ in range(2):
        y = run.layer()
        assert torch.equal(y.view(torch.int16), y0.view(torch.int16))


# ----------------------------------------------------------------------------- read-kernel modes
@pytest.mark.parametrize("kind", [vdn.ELU1, vdn.DELTA])
def test_scalar_linear_gate_tensor_core_path(kind):
    """G_l = 1 on the D = 128 tensor-core path (the scalar-gate instantiation of the read)."""
    shape = synth.Shape(12, 300, 5, 40, 2, 128)
    inp = synth.make_inputs(shape, "bf16", seed=6, gate_l_cols=1, with_beta=kind == vdn.DELTA)
    run = Run(shape, inp, "bf16", kind=kind)
    s = run.shape
    rows = np.arange(s.n_video)
    o = oracle_inputs(inp)
    y = run.layer()
    HD = s.heads * s.head_dim
    A = to_numpy(run.intermediate(2, (s.n_video, 2 * HD), torch.bfloat16))
    ref = vo.layer(o, s.frames, s.tokens_per_frame, s.chunk_frames, rows=rows,
                   linear="delta" if kind == vdn.DELTA else "elu1")
    assert_close("A_l (scalar gate)", A[:, HD:], ref["a"][:, HD:], "bf16")
    assert_close("y", to_numpy(y), ref["y"], "bf16")


def test_delta_plain_read_tensor_core_path():
    """vdn_linear_read with the delta rule at D = 128 (the plain delta instantiation)."""
    s = synth.Shape(12, 300, 5, 40, 2, 128)
    F, T, C, L, H, D = 12, 300, 5, 40, 2, 128
    inp = synth.make_inputs(s, "bf16", seed=23, with_beta=True)
    d = {n: to_device(a) for n, a in inp.items()}
    o = oracle_inputs(inp)
    ws = workspace(vdn.step_workspace_size(s))
    vdn.workspace_init(ws)
    rSf, rSb = vo.delta_memory(o["k"], o["v"], o["kt"], o["vt"], o["beta"], F, T, C)
    _, gtab = vdn.mask_layout_build(s)
    G = vdn.max_groups(s)
    Sf = torch.zeros((G, H, D, D), dtype=torch.float32, device="cuda")
    Sb = torch.zeros((G, H, D, D), dtype=torch.float32, device="cuda")
    first = [int(r[0]) for r in gtab]
    Sf[:len(gtab)] = torch.from_numpy(rSf[first].astype(np.float32)).cuda()
    Sb[:len(gtab)] = torch.from_numpy(rSb[first].astype(np.float32)).cuda()
    o_l = empty((s.n_video, H, D), "bf16")
    vdn.linear_read(s, vdn.DELTA, vdn.BF16, d["q"], Sf, Sb, None, None, o_l, ws)
    vdn.check_device_status(ws)
    assert_close("delta read (tensor cores)", to_numpy(o_l), vo.delta_read(o["q"], rSf, rSb, T), "bf16")
