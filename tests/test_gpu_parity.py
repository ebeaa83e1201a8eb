"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bit-exact: packed weights, gamma, x_q, per-token scales, int32 accumulators.
Dequantised outputs and the ReLU^2 gate: relative error <= 1e-6 (zero exact).
Every kernel selection is exercised on the same inputs; ragged tails in M, N
and K (K % 128 == 64 gives a half-filled last k-stage) are covered.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_fwd_b200 as tw
from gpu_util import DEV, assert_rel_close, make_weights, make_x, sample_rows

pytestmark = pytest.mark.gpu

DECODE = [tw.BITNET_DISPATCH_DECODE_FUSED, tw.BITNET_DISPATCH_DECODE, tw.BITNET_DISPATCH_PREFILL]
DNAME = {0: "auto", 1: "decode_fused", 2: "decode", 3: "prefill"}


@pytest.fixture(autouse=True)
def _clean_state():
    prev = tw.bitnet_set_dispatch(tw.BITNET_DISPATCH_AUTO)
    yield
    tw.bitnet_set_dispatch(prev)
    assert tw.bitnet_device_status(clear=True) == 0


# ---------------------------------------------------------------- packing
@pytest.mark.parametrize("n,k", [(256, 256), (17, 64), (1000, 320), (2560, 2560), (6912, 2560), (2560, 6912)])
def test_pack_bit_exact(n, k):
    W = make_weights(n, k, 100 + n + k)
    assert np.float32(W["g"].cpu().numpy()[0]).view(np.uint32) == np.float32(W["g_ref"]).view(np.uint32)
    assert np.array_equal(W["p"].cpu().numpy(), W["p_ref"])


def test_pack_deterministic():
    W = make_weights(2560, 2560, 7)
    p2, g2 = tw.bitnet_pack_weights(torch.from_numpy(W["w"]).to(DEV))
    assert torch.equal(p2, W["p"]) and torch.equal(g2, W["g"])


# ---------------------------------------------------------------- activation quantiser
@pytest.mark.parametrize("m,k,kind,dtype", [
    (1, 256, "normal", "bf16"), (4, 256, "normal", "bf16"), (7, 320, "outliers", "bf16"),
    (64, 2560, "student_t_rows", "bf16"), (33, 6912, "outliers", "bf16"), (4096, 2560, "student_t_rows", "bf16"),
    (5, 2560, "normal", "f32"), (300, 6912, "normal", "f32"),
    # the streaming kernel (M >= 256, rows of up to 32 KB in shared memory): ragged grids, the
    # largest row it takes, and rows of a single 128-byte chunk per lane group
    (257, 6912, "outliers", "bf16"), (600, 8192, "normal", "f32"), (1024, 64, "student_t_rows", "bf16"),
    # row held by 8 warps (fp32, K = 16384) and the two-pass kernel for rows longer than that
    (3, 16384, "normal", "f32"), (2, 65536, "outliers", "bf16"), (9, 65536, "normal", "f32"),
])
def test_quant_act_bit_exact(m, k, kind, dtype):
    xd, xf = make_x(m, k, 200 + m + k, kind, dtype)
    x_q, s, rs = tw.bitnet_quant_act(xd)
    rq, rsc, rrs = oracle.quant_act(xf)
    assert np.array_equal(x_q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rsc.view(np.uint32))
    assert np.array_equal(rs.cpu().numpy(), rrs)


def test_quant_act_special_rows():
    x = np.zeros((4, 128), np.float32)
    x[1, :8] = [127.0, 2.5, -2.5, 3.5, 0.5, -0.5, 1.5, -126.5]   # s = 1, exact ties
    x[2, :5] = [1.0, 3.0, -5.0, -254.0, 7.0]                      # s = 0.5
    x[3, 7] = -3e-38                                               # tiny row (amax < 1e-5)
    for dt in (torch.float32, torch.bfloat16):
        xd = torch.from_numpy(x).to(DEV).to(dt)
        x_q, s, rs = tw.bitnet_quant_act(xd)
        xf = xd.float().cpu().numpy()
        rq, rsc, rrs = oracle.quant_act(xf)
        assert np.array_equal(x_q.cpu().numpy(), rq)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), rsc.view(np.uint32))
        assert np.array_equal(rs.cpu().numpy(), rrs)


# ---------------------------------------------------------------- BitLinear
def run_linear(xd, W, dispatch, m, k, n):
    tw.bitnet_set_dispatch(dispatch)
    acc = torch.full((m, n), -7, dtype=torch.int32, device=DEV)
    x_q = torch.empty((m, k), dtype=torch.int8, device=DEV)
    s = torch.empty(m, dtype=torch.float32, device=DEV)
    y = tw.bitnet_linear(xd, W["p"], W["g"], x_q_out=x_q, s_out=s, acc_out=acc)
    torch.cuda.synchronize()
    return y.cpu().numpy(), acc.cpu().numpy(), x_q.cpu().numpy(), s.cpu().numpy()


def weights_from(w):
    """Packed weights of a given latent matrix, by both sides."""
    p_ref, g_ref, w_q = oracle.pack_weights(w)
    p, g = tw.bitnet_pack_weights(torch.from_numpy(w).to(DEV))
    torch.cuda.synchronize()
    return dict(w=w, w_q=w_q, p_ref=p_ref, g_ref=g_ref, p=p, g=g)


@pytest.mark.parametrize("dispatch,m", [(d, 5) for d in DECODE] + [(tw.BITNET_DISPATCH_PREFILL, 130)],
                         ids=lambda v: DNAME[v] if v in DNAME and v < 4 else str(v))
def test_linear_degenerate_inputs(dispatch, m):
    """Degenerate cases of the method on every path: an all-zero latent matrix (gamma = 0, so
    every code is 0 and every output exactly 0), a matrix with one nonzero latent (gamma =
    |w| / (N K), W_q one-hot), and activation rows that are all zero (s = 127 / 1e-5, x_q = 0,
    y = 0) next to ordinary rows.  Integers bit-exact, outputs as the oracle (zero exact)."""
    k, n = 320, 200
    xd, xf = make_x(m, k, 4100 + m, "normal", "bf16")
    xd = xd.clone()
    xd[1].zero_()
    xd[m - 1].zero_()
    xf = xd.float().cpu().numpy()
    one = np.zeros((n, k), np.float32)
    one[37, 101] = -0.75
    for w in (np.zeros((n, k), np.float32), one):
        W = weights_from(w)
        assert np.array_equal(W["p"].cpu().numpy(), W["p_ref"])
        y, acc, x_q, s = run_linear(xd, W, dispatch, m, k, n)
        y_ref, acc_ref, xq_ref, s_ref = oracle.bitlinear(xf, W["p_ref"], W["g_ref"], k)
        assert np.array_equal(x_q, xq_ref)
        assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32))
        assert np.array_equal(acc.astype(np.int64), acc_ref)
        assert_rel_close(y, y_ref)
        assert not y[1].any() and not y[m - 1].any()
        if not w.any():
            assert not y.any() and not acc.any()


LINEAR_SHAPES = [
    # (M, K, N, kind, dtype)
    (4, 256, 256, "normal", "bf16"),          # small single BitLinear
    (1, 2560, 2560, "outliers", "bf16"),      # decode GEMV shapes, M = 1
    (1, 2560, 6912, "outliers", "bf16"),
    (1, 6912, 2560, "outliers", "bf16"),
    (8, 2560, 6912, "normal", "bf16"),
    (16, 6912, 2560, "normal", "f32"),        # down projection reads fp32 h
    (33, 320, 200, "outliers", "bf16"),       # ragged M, N; K % 128 == 64
    (64, 2560, 2560, "normal", "bf16"),
    (3, 64, 1, "normal", "bf16"),             # minimum K, single output column
    (5, 576, 300, "normal", "bf16"),          # 9 k-steps over a cluster of 8: ranks without k-steps
    (40, 1024, 1000, "outliers", "f32"),      # 5 token tiles, fp32 input
    (8, 2560, 640, "normal", "bf16"),         # K / V projections of the 2B4T layer (GQA, 5 KV heads)
    (8, 2560, 3840, "normal", "bf16"),        # fused q|k|v projection
    (32, 6912, 2560, "normal", "f32"),        # batched decode down projections (M = 32, 64)
    (64, 6912, 2560, "outliers", "f32"),
]


@pytest.mark.parametrize("dispatch", DECODE, ids=lambda d: DNAME[d])
@pytest.mark.parametrize("m,k,n,kind,dtype", LINEAR_SHAPES)
def test_linear_small_m(dispatch, m, k, n, kind, dtype):
    W = make_weights(n, k, 300 + n + k)
    xd, xf = make_x(m, k, 400 + m + k, kind, dtype)
    y, acc, x_q, s = run_linear(xd, W, dispatch, m, k, n)
    y_ref, acc_ref, xq_ref, s_ref = oracle.bitlinear(xf, W["p_ref"], W["g_ref"], k)
    assert np.array_equal(x_q, xq_ref)
    assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(acc.astype(np.int64), acc_ref)
    assert_rel_close(y, y_ref)


PREFILL_SHAPES = [
    (129, 192, 257, "student_t_rows", "bf16"),  # M = 128 + 1, N % 4 != 0, K % 128 == 64
    (300, 320, 300, "normal", "bf16"),
    (256, 2560, 512, "student_t_rows", "f32"),
    (1, 64, 5, "normal", "bf16"),
]


@pytest.mark.parametrize("m,k,n,kind,dtype", PREFILL_SHAPES)
def test_linear_prefill_ragged(m, k, n, kind, dtype):
    W = make_weights(n, k, 500 + n + k)
    xd, xf = make_x(m, k, 600 + m + k, kind, dtype)
    y, acc, x_q, s = run_linear(xd, W, tw.BITNET_DISPATCH_PREFILL, m, k, n)
    y_ref, acc_ref, xq_ref, s_ref = oracle.bitlinear(xf, W["p_ref"], W["g_ref"], k)
    assert np.array_equal(x_q, xq_ref)
    assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(acc.astype(np.int64), acc_ref)
    assert_rel_close(y, y_ref)


@pytest.mark.parametrize("k,n", [(2560, 6912), (6912, 2560), (2560, 3840), (2560, 640), (2560, 2560)])
def test_linear_prefill_full_size_sampled(k, n):
    """M = 4096 prefill at the 2B4T shapes; every output of 48 sampled rows.  N = 2560 and 3840
    leave a partly filled last wave of tiles, which runs as sub-tiles of 64 output columns."""
    m = 4096
    W = make_weights(n, k, 700 + k)
    xd, xf = make_x(m, k, 800 + k, "student_t_rows", "bf16")
    y, acc, x_q, s = run_linear(xd, W, tw.BITNET_DISPATCH_AUTO, m, k, n)
    # the quantiser on every row
    xq_all, s_all, _ = oracle.quant_act(xf)
    assert np.array_equal(x_q, xq_all)
    assert np.array_equal(s.view(np.uint32), s_all.view(np.uint32))
    # the contraction and epilogue on sampled rows: both ends and one random row of every 128-row tile
    rows = sample_rows(m, 48, 9)
    y_ref, acc_ref, xq_ref, s_ref = oracle.bitlinear(xf[rows], W["p_ref"], W["g_ref"], k)
    assert np.array_equal(acc[rows].astype(np.int64), acc_ref)
    assert_rel_close(y[rows], y_ref)
    # properties that hold for every output: |acc| <= 127 * K, and y == 0 iff acc == 0
    assert np.abs(acc).max() <= 127 * k
    assert np.array_equal(y == 0, acc == 0)


# ---------------------------------------------------------------- gated FFN
def run_ffn(xd, G, U, dispatch, m, n):
    tw.bitnet_set_dispatch(dispatch)
    ag = torch.full((m, n), -7, dtype=torch.int32, device=DEV)
    au = torch.full((m, n), -7, dtype=torch.int32, device=DEV)
    h = tw.bitnet_ffn_gate_up(xd, G["p"], G["g"], U["p"], U["g"], acc_g_out=ag, acc_u_out=au)
    torch.cuda.synchronize()
    return h.cpu().numpy(), ag.cpu().numpy(), au.cpu().numpy()


@pytest.mark.parametrize("dispatch,m", [(d, 5) for d in DECODE] + [(tw.BITNET_DISPATCH_PREFILL, 130)],
                         ids=lambda v: DNAME[v] if v in DNAME and v < 4 else str(v))
def test_ffn_degenerate_inputs(dispatch, m):
    """The gated FFN with an all-zero gate matrix (h = relu(0)^2 * u = 0) and with an all-zero
    up matrix (h = relu(g)^2 * 0 = 0), and all-zero activation rows, on every path: int32 sums
    bit-exact, h as the oracle and exactly zero where the definition makes it zero."""
    k, n = 320, 136
    xd, _ = make_x(m, k, 4200 + m, "normal", "bf16")
    xd = xd.clone()
    xd[0].zero_()
    xf = xd.float().cpu().numpy()
    rnd = make_weights(n, k, 4300)
    zero = weights_from(np.zeros((n, k), np.float32))
    for G, U in ((zero, rnd), (rnd, zero)):
        h, ag, au = run_ffn(xd, G, U, dispatch, m, n)
        h_ref, ag_ref, au_ref, _, _ = oracle.ffn_gate_up(xf, G["p_ref"], G["g_ref"], U["p_ref"], U["g_ref"], k)
        assert np.array_equal(ag.astype(np.int64), ag_ref)
        assert np.array_equal(au.astype(np.int64), au_ref)
        assert_rel_close(h, h_ref)
        assert not h.any()


FFN_SHAPES = [
    (12, 576, 136, "outliers"),
    (1, 2560, 6912, "normal"),
    (8, 2560, 6912, "normal"),
    (16, 2560, 6912, "outliers"),             # batched decode FFN at the 2B4T shape (M = 16, 32, 64)
    (32, 2560, 6912, "normal"),
    (64, 2560, 6912, "normal"),
    (32, 320, 200, "outliers"),
    (64, 256, 256, "normal"),
]


def token_rows(m):
    """All tokens up to 16; beyond, the first and last token of every 8-token tile."""
    if m <= 16:
        return np.arange(m)
    return np.array(sorted({r for t in range(0, m, 8) for r in (t, min(t + 7, m - 1))}))


@pytest.mark.parametrize("dispatch", DECODE, ids=lambda d: DNAME[d])
@pytest.mark.parametrize("m,k,n,kind", FFN_SHAPES)
def test_ffn_small_m(dispatch, m, k, n, kind):
    G = make_weights(n, k, 900 + n)
    U = make_weights(n, k, 950 + n)
    xd, xf = make_x(m, k, 1000 + m, kind)
    h, ag, au = run_ffn(xd, G, U, dispatch, m, n)
    rows = token_rows(m)
    h_ref, ag_ref, au_ref, _, _ = oracle.ffn_gate_up(xf[rows], G["p_ref"], G["g_ref"], U["p_ref"], U["g_ref"], k)
    assert np.array_equal(ag[rows].astype(np.int64), ag_ref)
    assert np.array_equal(au[rows].astype(np.int64), au_ref)
    assert_rel_close(h[rows], h_ref)


@pytest.mark.parametrize("m,k,n", [(4096, 2560, 6912), (200, 192, 130), (4096, 2560, 2560)])
def test_ffn_prefill(m, k, n):
    G = make_weights(n, k, 1100 + n)
    U = make_weights(n, k, 1150 + n)
    xd, xf = make_x(m, k, 1200 + m, "student_t_rows")
    h, ag, au = run_ffn(xd, G, U, tw.BITNET_DISPATCH_AUTO if m > 64 else tw.BITNET_DISPATCH_PREFILL, m, n)
    rows = sample_rows(m, 40, 11) if m > 512 else np.arange(m)
    h_ref, ag_ref, au_ref, _, _ = oracle.ffn_gate_up(xf[rows], G["p_ref"], G["g_ref"], U["p_ref"], U["g_ref"], k)
    assert np.array_equal(ag[rows].astype(np.int64), ag_ref)
    assert np.array_equal(au[rows].astype(np.int64), au_ref)
    assert_rel_close(h[rows], h_ref)


@pytest.mark.parametrize("m", [8, 4096])
def test_ffn_chain_down(m):
    """gate/up -> down: the down projection re-quantises the GPU's fp32 h per token
    (stage-wise parity: the oracle quantises the same h)."""
    k, n = 2560, 6912
    G = make_weights(n, k, 1300)
    U = make_weights(n, k, 1301)
    D = make_weights(k, n, 1302)
    xd, _ = make_x(m, k, 1303)
    h = tw.bitnet_ffn_gate_up(xd, G["p"], G["g"], U["p"], U["g"])
    acc = torch.empty((m, k), dtype=torch.int32, device=DEV)
    y = tw.bitnet_linear(h, D["p"], D["g"], acc_out=acc)
    torch.cuda.synchronize()
    rows = sample_rows(m, 24, 13) if m > 64 else np.arange(m)
    hf = h.cpu().numpy()[rows]
    y_ref, acc_ref, _, _ = oracle.bitlinear(hf, D["p_ref"], D["g_ref"], n)
    assert np.array_equal(acc.cpu().numpy()[rows].astype(np.int64), acc_ref)
    assert_rel_close(y.cpu().numpy()[rows], y_ref)


# ---------------------------------------------------------------- cross-checks
@pytest.mark.parametrize("dispatch,m,kernels", [
    (tw.BITNET_DISPATCH_AUTO, 8, 1),          # cluster kernel: quantiser fused in
    (tw.BITNET_DISPATCH_DECODE_FUSED, 64, 1),
    (tw.BITNET_DISPATCH_DECODE, 8, 2),        # quantiser kernel + row-split decode kernel
    (tw.BITNET_DISPATCH_PREFILL, 8, 2),       # quantiser kernel + tcgen05 kernel
    (tw.BITNET_DISPATCH_AUTO, 65, 2),
])
def test_kernels_per_call(dispatch, m, kernels):
    k, n = 2560, 2560
    W = make_weights(n, k, 1700)
    xd, _ = make_x(m, k, 1701)
    tw.bitnet_set_dispatch(dispatch)
    y = torch.empty((m, n), dtype=torch.float32, device=DEV)
    ws = torch.empty(tw.bitnet_workspace_size(m, n, k), dtype=torch.uint8, device=DEV)
    c0 = tw.bitnet_launch_count()
    tw.bitnet_linear(xd, W["p"], W["g"], y=y, workspace=ws)
    assert tw.bitnet_launch_count() - c0 == kernels
    torch.cuda.synchronize()



def test_all_kernels_agree_bitwise():
    m, k, n = 24, 2560, 6912
    W = make_weights(n, k, 1400)
    xd, _ = make_x(m, k, 1401)
    outs = [run_linear(xd, W, d, m, k, n)[0] for d in DECODE]
    for o in outs[1:]:
        assert np.array_equal(o.view(np.uint32), outs[0].view(np.uint32))


def test_acc_matches_library_int8_gemm():
    """Library special case: the int32 accumulators equal torch._int_mm on the
    unpacked int8 weights (run as a black box)."""
    m, k, n = 128, 2560, 2560
    W = make_weights(n, k, 1500)
    w_t = torch.from_numpy(W["w_q"]).to(DEV).t()   # [K][N], column-major
    xd, _ = make_x(m, k, 1501)
    for d, mm in ((tw.BITNET_DISPATCH_PREFILL, m), (tw.BITNET_DISPATCH_DECODE, 64)):
        _, acc, x_q, _ = run_linear(xd[:mm].contiguous(), W, d, mm, k, n)
        ref = torch._int_mm(torch.from_numpy(x_q).to(DEV), w_t)
        assert np.array_equal(acc, ref.cpu().numpy())


def test_repeat_calls_identical_and_graph_capture():
    m, k, n = 8, 2560, 2560
    W = make_weights(n, k, 1600)
    xd, _ = make_x(m, k, 1601)
    ws = torch.empty(tw.bitnet_workspace_size(m, n, k), dtype=torch.uint8, device=DEV)
    y1 = tw.bitnet_linear(xd, W["p"], W["g"], workspace=ws).clone()
    y2 = torch.empty_like(y1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            tw.bitnet_linear(xd, W["p"], W["g"], y=y2, workspace=ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    y2.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
