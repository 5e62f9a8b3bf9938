"""CPU pin of the e4m3 error bound used for the softmax branch on the GPU.

Per-head e4m3 rounding (3 mantissa bits, about 2.6% RMS relative error per value) of Q,
K, V and P cannot reproduce a float64 softmax to 3e-2 on unit-Gaussian data: the
rounded scores shift the weights by about 3.7%, and the rounded V and P add about 2.6%
each.  This test measures that model error with torch's own CPU e4m3 conversion on a
query block with the key count and head size of the full-size workload (17,648 keys,
D = 128), and checks that the GPU bound of 7e-2 sits above it with margin.  The kernel
itself is held to 3e-2 against the oracle evaluated on its own e4m3 inputs.

The next tests fix the model error of the e4m3 output projection (per-column weight
scales; static per-head A scales from the branches' bounds) and of the whole e4m3 layer,
which set the bounds its GPU tests use (tests/test_e4m3_projection_gpu.py)."""
import numpy as np
import torch

GPU_BOUND = 7e-2


def _e4m3(x, amax):
    s = amax / 448.0
    return (x / s).float().to(torch.float8_e4m3fn).double() * s


def test_e4m3_attention_model_error():
    g = torch.Generator().manual_seed(0)
    n, nk, d = 128, 17648, 128
    q = torch.randn(n, d, generator=g, dtype=torch.float64)
    k = torch.randn(nk, d, generator=g, dtype=torch.float64)
    v = torch.randn(nk, d, generator=g, dtype=torch.float64)
    ref = torch.softmax(q @ k.T / d ** 0.5, -1) @ v
    q8, k8, v8 = (_e4m3(x, x.abs().max()) for x in (q, k, v))
    s = q8 @ k8.T / d ** 0.5
    p = torch.exp(s - s.max(-1, keepdim=True).values)
    p8 = p.float().to(torch.float8_e4m3fn).double()           # unit scale
    out = (p8 @ v8) / p.sum(-1, keepdim=True)
    err = ((out - ref).norm() / ref.norm()).item()
    assert 0.03 < err < 0.8 * GPU_BOUND, err                  # above the 3e-2 bar, below the bound
    # with only P rounded (the kernel's own arithmetic on e4m3 inputs) the error is inside 3e-2
    ref8 = torch.softmax(s, -1) @ v8
    err_p = (((p8 @ v8) / p.sum(-1, keepdim=True) - ref8).norm() / ref8.norm()).item()
    assert err_p < 0.03, err_p


PROJ_GPU_BOUND = 6e-2


def test_e4m3_projection_model_error():
    """The error model of an e4m3 output projection (the first of the next steps): A with one
    scale per row (its amax / 448), each output column of W_o with its own, products summed
    in fp32 or better.  On layer-sized rows (K = 2HD = 10240) the model error against the
    exact product is about 3.7% RMS, set by e4m3's 3 mantissa bits, well inside the bound
    such a kernel would be held to; the kernel's own arithmetic on the rounded operands is
    exact up to fp32 accumulation."""
    g = torch.Generator().manual_seed(1)
    n, k, m = 64, 10240, 256
    a = torch.randn(n, k, generator=g, dtype=torch.float64)
    a[:, : k // 2] *= 0.3                                   # the softmax half is smaller
    w = torch.randn(m, k, generator=g, dtype=torch.float64) * 0.02
    ref = a @ w.T
    a8 = torch.cat([_e4m3(r, r.abs().max()).unsqueeze(0) for r in a])
    w8 = torch.cat([_e4m3(c, c.abs().max()).unsqueeze(0) for c in w])
    err = ((a8 @ w8.T - ref).norm() / ref.norm()).item()
    assert 0.02 < err < 0.8 * PROJ_GPU_BOUND, err
    # one scale for the whole of A instead of one per row costs accuracy only when rows
    # differ in size; here they do not, so the two agree to within a few percent
    a8t = _e4m3(a, a.abs().max())
    err_t = ((a8t @ w8.T - ref).norm() / ref.norm()).item()
    assert abs(err_t - err) < 0.25 * err, (err_t, err)


def test_e4m3_projection_static_bounds_cost_nothing():
    """Static scales from the branches' bounds do as well as measured amaxes.  A_s is a
    gated convex combination of V rows, so |A_s| <= amax(V); A_l is a gated RMS-normalised
    vector, so |A_l| <= max|gamma| sqrt(D).  e4m3 keeps its relative step over 14 binades,
    so values far below such a bound round no worse.  The branch epilogues can therefore
    write A in e4m3 as they go, with no amax pass: model error as with per-row scales."""
    g = torch.Generator().manual_seed(2)
    n, hd, m = 64, 5120, 256
    a_s = 0.1 * torch.randn(n, hd, generator=g, dtype=torch.float64)    # softmax-averaged V, gated
    a_l = 0.5 * torch.randn(n, hd, generator=g, dtype=torch.float64)    # gated, RMS-normalised
    w = torch.randn(m, 2 * hd, generator=g, dtype=torch.float64) * 0.02
    a = torch.cat([a_s, a_l], 1)
    ref = a @ w.T
    w8 = torch.cat([_e4m3(c, c.abs().max()).unsqueeze(0) for c in w])
    a8_static = torch.cat([_e4m3(a_s, torch.tensor(5.0)), _e4m3(a_l, torch.tensor(128.0 ** 0.5))], 1)
    a8_row = torch.cat([_e4m3(r, r.abs().max()).unsqueeze(0) for r in a])
    err_static = ((a8_static @ w8.T - ref).norm() / ref.norm()).item()
    err_row = ((a8_row @ w8.T - ref).norm() / ref.norm()).item()
    assert err_static < 0.8 * PROJ_GPU_BOUND and abs(err_static - err_row) < 0.05 * err_row, (err_static, err_row)


LAYER_E4M3_BOUND = 6e-2


def test_e4m3_layer_model_error():
    """The whole e4m3 layer's model error on y: the e4m3 softmax (per-head Q/K/V scales,
    e4m3 P) feeds A_s, A is written as e4m3 codes with the static per-head scales (the V
    scale for A_s, max|gamma| sqrt(D) / 448 for A_l) and [W_os | W_ol] is rounded per output
    column.  Simulated here with torch's CPU e4m3 conversion on layer-shaped data (2 heads
    of 128, 17,648 keys per query, gates and RMSNorm as in the layer); y's error against
    the exact float64 layer must sit well inside the GPU bound LAYER_E4M3_BOUND."""
    g = torch.Generator().manual_seed(3)
    n, nk, d, H = 128, 17648, 128, 2
    hd = H * d
    q = torch.randn(H, n, d, generator=g, dtype=torch.float64)
    k = torch.randn(H, nk, d, generator=g, dtype=torch.float64)
    v = torch.randn(H, nk, d, generator=g, dtype=torch.float64)
    w_s = torch.randn(H, d, generator=g, dtype=torch.float64) * 0.02
    w_l = torch.randn(H, d, d, generator=g, dtype=torch.float64) * 0.02
    o_l = torch.randn(H, n, d, generator=g, dtype=torch.float64)          # any linear-branch output
    w = torch.randn(hd, 2 * hd, generator=g, dtype=torch.float64) * 0.02

    def layer_y(o_s, a8):
        gs = torch.sigmoid((q * w_s[:, None, :]).sum(-1, keepdim=True))
        gl = torch.sigmoid(torch.einsum("hnd,hde->hne", q, w_l))
        nrm = o_l / torch.sqrt((o_l ** 2).mean(-1, keepdim=True) + 1e-6)
        a_s, a_l = gs * o_s, gl * nrm                                        # gamma = 1
        if a8:
            vs = v.abs().amax((1, 2)) / 448.0                                # the V scale per head
            ls = torch.full((H,), d ** 0.5 / 448.0, dtype=torch.float64)     # max|gamma| sqrt(D) / 448
            a_s = (a_s / vs[:, None, None]).float().to(torch.float8_e4m3fn).double() * vs[:, None, None]
            a_l = (a_l / ls[:, None, None]).float().to(torch.float8_e4m3fn).double() * ls[:, None, None]
        a = torch.cat([a_s.permute(1, 0, 2).reshape(n, hd), a_l.permute(1, 0, 2).reshape(n, hd)], 1)
        ww = torch.cat([_e4m3(c, c.abs().max()).unsqueeze(0) for c in w]) if a8 else w
        return a @ ww.T

    exact_o = torch.softmax(q @ k.transpose(1, 2) / d ** 0.5, -1) @ v
    q8 = torch.stack([_e4m3(x, x.abs().max()) for x in q])
    k8 = torch.stack([_e4m3(x, x.abs().max()) for x in k])
    v8 = torch.stack([_e4m3(x, x.abs().max()) for x in v])
    s = q8 @ k8.transpose(1, 2) / d ** 0.5
    p = torch.exp(s - s.amax(-1, keepdim=True))
    o8 = (p.float().to(torch.float8_e4m3fn).double() @ v8) / p.sum(-1, keepdim=True)
    ref = layer_y(exact_o, False)
    err = ((layer_y(o8, True) - ref).norm() / ref.norm()).item()
    assert 0.02 < err < 0.8 * LAYER_E4M3_BOUND, err
