"""bitnet_decode_sequence on the GPU, through the C ABI.

Every op of a persistent sequence launch is compared
  * with the CPU oracle on the same inputs (integers exact, y within 1e-6
    relative), and
  * bitwise with the same op run alone (bitnet_linear / bitnet_ffn_gate_up),
and a sequence whose ops share buffers (read after write, write after read,
write after write) must leave every buffer exactly as running its ops one
after another does.  Both cluster sizes (4 and 8 CTAs splitting K) are run."""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_fwd_b200 as tw
from gpu_util import DEV, assert_rel_close, make_weights, make_x

pytestmark = pytest.mark.gpu

H, I = 2560, 6912


@pytest.fixture(autouse=True, params=[4, 8], ids=["c4", "c8"])
def cluster(request):
    prev = tw.bitnet_set_sequence_cluster(request.param)
    yield request.param
    tw.bitnet_set_sequence_cluster(prev)
    assert tw.bitnet_device_status(clear=True) == 0


def oracle_linear(xf, W, k):
    y, acc, _, _ = oracle.bitlinear(np.ascontiguousarray(xf, np.float32), W["p_ref"], W["g_ref"], k)
    return y


def oracle_ffn(xf, Wg, Wu, k):
    h, _, _, _, _ = oracle.ffn_gate_up(np.ascontiguousarray(xf, np.float32), Wg["p_ref"], Wg["g_ref"],
                                       Wu["p_ref"], Wu["g_ref"], k)
    return h


def run_seq(ops, m, ws=None):
    ws = tw.bitnet_sequence_workspace(DEV) if ws is None else ws
    tw.bitnet_decode_sequence(ops, m, ws)
    torch.cuda.synchronize()
    return ws


# ---------------------------------------------------------------- a decode step of a layer stack
@pytest.mark.parametrize("m", [1, 8, 13, 64])
def test_layer_stack(m, cluster):
    """Two layers of (q, o, gate/up + ReLU^2, down on h), private outputs."""
    layers = []
    for l in range(2):
        s = 1000 * (l + 1) + m
        L = dict(q=make_weights(H, H, s + 1), o=make_weights(H, H, s + 2), g=make_weights(I, H, s + 3),
                 u=make_weights(I, H, s + 4), d=make_weights(H, I, s + 5))
        L["x"] = [make_x(m, H, s + 10 + i, "outliers" if i == 0 else "normal") for i in range(3)]
        L["out"] = {k: torch.empty((m, n), dtype=torch.float32, device=DEV)
                    for k, n in (("q", H), ("o", H), ("h", I), ("down", H))}
        layers.append(L)
    ops = []
    for L in layers:
        (xq, _), (xo, _), (xg, _) = L["x"]
        o = L["out"]
        ops += [tw.linear_op(xq, L["q"]["p"], L["q"]["g"], o["q"]),
                tw.linear_op(xo, L["o"]["p"], L["o"]["g"], o["o"]),
                tw.ffn_gate_up_op(xg, L["g"]["p"], L["g"]["g"], L["u"]["p"], L["u"]["g"], o["h"]),
                tw.linear_op(o["h"], L["d"]["p"], L["d"]["g"], o["down"])]
    ws = run_seq(ops, m)
    assert torch.count_nonzero(ws) == 0, "counters must be left zeroed"

    rows = np.arange(m) if m <= 8 else np.array(sorted({0, 1, m // 2, m - 2, m - 1}))
    for L in layers:
        (xq, fq), (xo, fo), (xg, fg) = L["x"]
        o = {k: v.cpu().numpy() for k, v in L["out"].items()}
        # alone, through the per-op entry points: bit-identical
        ref_q = tw.bitnet_linear(xq, L["q"]["p"], L["q"]["g"])
        ref_o = tw.bitnet_linear(xo, L["o"]["p"], L["o"]["g"])
        ref_h = tw.bitnet_ffn_gate_up(xg, L["g"]["p"], L["g"]["g"], L["u"]["p"], L["u"]["g"])
        ref_d = tw.bitnet_linear(ref_h, L["d"]["p"], L["d"]["g"])
        for got, ref in ((o["q"], ref_q), (o["o"], ref_o), (o["h"], ref_h), (o["down"], ref_d)):
            assert np.array_equal(got.view(np.uint32), ref.cpu().numpy().view(np.uint32))
        # against the oracle (stage-wise: the down projection quantises the GPU's h)
        assert_rel_close(o["q"][rows], oracle_linear(fq[rows], L["q"], H))
        assert_rel_close(o["o"][rows], oracle_linear(fo[rows], L["o"], H))
        assert_rel_close(o["h"][rows], oracle_ffn(fg[rows], L["g"], L["u"], H))
        assert_rel_close(o["down"][rows], oracle_linear(o["h"][rows], L["d"], I))


# ---------------------------------------------------------------- shapes
SHAPES = [  # (kind, K, N, x dtype)
    ("linear", 64, 8, "bf16"), ("linear", 128, 300, "bf16"), ("linear", 256, 256, "f32"),
    ("linear", 576, 1000, "bf16"), ("linear", 8192, 256, "bf16"), ("linear", 6912, 2560, "f32"),
    ("linear", 2560, 640, "bf16"), ("linear", 2560, 3840, "bf16"), ("ffn", 256, 136, "bf16"),
    ("ffn", 2560, 6912, "bf16"), ("ffn", 320, 17, "f32"),
]


@pytest.mark.parametrize("kind,k,n,dtype", SHAPES)
@pytest.mark.parametrize("m", [1, 5, 8, 9])
def test_shapes_vs_oracle(kind, k, n, dtype, m, cluster):
    seed = 7 * k + n + m
    x, xf = make_x(m, k, seed, "normal", dtype)
    W0 = make_weights(n, k, seed + 1)
    if kind == "linear":
        y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
        ops = [tw.linear_op(x, W0["p"], W0["g"], y)]
        run_seq(ops, m)
        ref = tw.bitnet_linear(x, W0["p"], W0["g"])
        assert_rel_close(y.cpu().numpy(), oracle_linear(xf, W0, k))
    else:
        W1 = make_weights(n, k, seed + 2)
        y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
        ops = [tw.ffn_gate_up_op(x, W0["p"], W0["g"], W1["p"], W1["g"], y)]
        run_seq(ops, m)
        ref = tw.bitnet_ffn_gate_up(x, W0["p"], W0["g"], W1["p"], W1["g"])
        assert_rel_close(y.cpu().numpy(), oracle_ffn(xf, W0, W1, k))
    assert torch.equal(y.view(torch.int32), ref.view(torch.int32))


# ---------------------------------------------------------------- shared buffers
def test_hazards_match_sequential_execution(cluster):
    """Ops that read each other's outputs and overwrite each other's inputs."""
    m, k = 8, 256
    Ws = [make_weights(k, k, 500 + i) for i in range(6)]
    Wg, Wu = make_weights(k, k, 510), make_weights(k, k, 511)
    x0, _ = make_x(m, k, 520)
    x1, _ = make_x(m, k, 521)

    def program(A, B, C):
        return [
            ("lin", x0, Ws[0], A),          # A = L0(x0)
            ("lin", A, Ws[1], B),           # B = L1(A)          read after write
            ("lin", x1, Ws[2], A),          # A = L2(x1)         write after write, write after read
            ("lin", A, Ws[3], B),           # B = L3(A)          reads the new A
            ("ffn", x0, (Wg, Wu), C),       # C = FFN(x0)
            ("lin", C, Ws[4], A),           # A = L4(C)
            ("lin", B, Ws[5], C),           # C = L5(B)          write after read of C by L4
        ]

    def bufs():
        return [torch.full((m, k), float("nan"), dtype=torch.float32, device=DEV) for _ in range(3)]

    A, B, C = bufs()
    ops = []
    for kind, x, W, y in program(A, B, C):
        if kind == "lin":
            ops.append(tw.linear_op(x, W["p"], W["g"], y))
        else:
            ops.append(tw.ffn_gate_up_op(x, W[0]["p"], W[0]["g"], W[1]["p"], W[1]["g"], y))
    wx, wy = tw.bitnet_sequence_plan(ops, m)
    assert wx == [-1, 0, -1, 2, -1, 4, 3] and wy == [-1, -1, 1, 1, -1, 3, 5]
    run_seq(ops, m)

    rA, rB, rC = bufs()
    for kind, x, W, y in program(rA, rB, rC):
        if kind == "lin":
            tw.bitnet_linear(x, W["p"], W["g"], y=y)
        else:
            tw.bitnet_ffn_gate_up(x, W[0]["p"], W[0]["g"], W[1]["p"], W[1]["g"], h=y)
    torch.cuda.synchronize()
    for got, ref in ((A, rA), (B, rB), (C, rC)):
        assert torch.equal(got.view(torch.int32), ref.view(torch.int32))


# ---------------------------------------------------------------- launches
def test_one_launch_graph_and_repeat(cluster):
    m = 8
    W = make_weights(H, H, 600)
    Wd = make_weights(H, I, 601)
    Wg, Wu = make_weights(I, H, 602), make_weights(I, H, 603)
    x, _ = make_x(m, H, 604)
    q = torch.empty((m, H), dtype=torch.float32, device=DEV)
    h = torch.empty((m, I), dtype=torch.float32, device=DEV)
    d = torch.empty((m, H), dtype=torch.float32, device=DEV)
    ops = [tw.linear_op(x, W["p"], W["g"], q), tw.ffn_gate_up_op(x, Wg["p"], Wg["g"], Wu["p"], Wu["g"], h),
           tw.linear_op(h, Wd["p"], Wd["g"], d)]
    ws = tw.bitnet_sequence_workspace(DEV)
    c0 = tw.bitnet_launch_count()
    run_seq(ops, m, ws)
    assert tw.bitnet_launch_count() - c0 == 1
    first = [t.clone() for t in (q, h, d)]
    for t in (q, h, d):
        t.fill_(float("nan"))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(3):
                tw.bitnet_decode_sequence(ops, m, ws, stream=s)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(first, (q, h, d)):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    assert torch.count_nonzero(ws) == 0


def test_huge_projection_is_cut_into_row_slices(cluster):
    """A gated FFN with 60000 output rows: its weights exceed every CTA's ring,
    so the planner cuts it into row slices; the result is bit-identical to the
    per-op call and matches the oracle on sampled rows."""
    m, k, n = 8, 256, 60000
    x, xf = make_x(m, k, 700, "outliers")
    G, U = make_weights(n, k, 701), make_weights(n, k, 702)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    ws = tw.bitnet_sequence_workspace(DEV)
    c0 = tw.bitnet_launch_count()
    tw.bitnet_decode_sequence([tw.ffn_gate_up_op(x, G["p"], G["g"], U["p"], U["g"], y)], m, ws)
    torch.cuda.synchronize()
    assert tw.bitnet_launch_count() - c0 == 1
    ref = tw.bitnet_ffn_gate_up(x, G["p"], G["g"], U["p"], U["g"])
    assert torch.equal(y.view(torch.int32), ref.view(torch.int32))
    cols = np.random.default_rng(703).choice(n, 512, replace=False)
    Gs = dict(p_ref=G["p_ref"][cols], g_ref=G["g_ref"])
    Us = dict(p_ref=U["p_ref"][cols], g_ref=U["g_ref"])
    assert_rel_close(y.cpu().numpy()[:, cols], oracle_ffn(xf, Gs, Us, k))
    assert torch.count_nonzero(ws) == 0


def test_k_above_the_limit_is_rejected(cluster):
    m = 8
    x = torch.zeros((m, 8256), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((256, 8256 // 4), dtype=torch.uint8, device=DEV)
    g = torch.ones(4, dtype=torch.float32, device=DEV)
    y = torch.empty((m, 256), dtype=torch.float32, device=DEV)
    ws = tw.bitnet_sequence_workspace(DEV)
    c0 = tw.bitnet_launch_count()
    with pytest.raises(tw.BitnetError) as e:
        tw.bitnet_decode_sequence([tw.linear_op(x, w, g, y)], m, ws)
    assert e.value.status == tw.BITNET_ERR_UNSUPPORTED_SHAPE
    assert tw.bitnet_launch_count() == c0


# ---------------------------------------------------------------- partitions of independent layers
@pytest.mark.parametrize("parts", [0, 1, 2, 4, 8])
@pytest.mark.parametrize("m", [1, 8, 13])
def test_private_layer_stack_partitions_and_slices(m, parts, cluster):
    """Layers with their own output buffers are independent groups: they run on
    separate partitions, with projections cut into row slices to fit the
    smaller partitions.  Every partition count gives the per-op results bit for
    bit; the oracle checks the gate/up -> down chain on sampled rows."""
    nl = 4
    layers = []
    for l in range(nl):
        s = 3000 + 100 * l + m
        L = dict(q=make_weights(H, H, s + 1), o=make_weights(H, H, s + 2), g=make_weights(I, H, s + 3),
                 u=make_weights(I, H, s + 4), d=make_weights(H, I, s + 5))
        L["x"] = [make_x(m, H, s + 10 + i) for i in range(3)]
        L["out"] = {k: torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
                    for k, n in (("q", H), ("o", H), ("h", I), ("down", H))}
        layers.append(L)
    ops = []
    for L in layers:
        (xq, _), (xo, _), (xg, _) = L["x"]
        o = L["out"]
        ops += [tw.linear_op(xq, L["q"]["p"], L["q"]["g"], o["q"]),
                tw.linear_op(xo, L["o"]["p"], L["o"]["g"], o["o"]),
                tw.ffn_gate_up_op(xg, L["g"]["p"], L["g"]["g"], L["u"]["p"], L["u"]["g"], o["h"]),
                tw.linear_op(o["h"], L["d"]["p"], L["d"]["g"], o["down"])]
    prev = tw.bitnet_set_sequence_partitions(parts)
    try:
        lay = tw.bitnet_sequence_layout(ops, m, cluster, 33 if cluster == 4 else 16)
        ws = run_seq(ops, m)
    finally:
        tw.bitnet_set_sequence_partitions(prev)
    if parts:
        assert len(lay["part_clusters"]) == parts
    assert torch.count_nonzero(ws) == 0
    rows = np.arange(m) if m <= 8 else np.array([0, m // 2, m - 1])
    for L in layers:
        (xq, fq), (xo, fo), (xg, fg) = L["x"]
        o = {k: v.cpu().numpy() for k, v in L["out"].items()}
        ref_q = tw.bitnet_linear(xq, L["q"]["p"], L["q"]["g"])
        ref_o = tw.bitnet_linear(xo, L["o"]["p"], L["o"]["g"])
        ref_h = tw.bitnet_ffn_gate_up(xg, L["g"]["p"], L["g"]["g"], L["u"]["p"], L["u"]["g"])
        ref_d = tw.bitnet_linear(ref_h, L["d"]["p"], L["d"]["g"])
        for got, ref in ((o["q"], ref_q), (o["o"], ref_o), (o["h"], ref_h), (o["down"], ref_d)):
            assert np.array_equal(got.view(np.uint32), ref.cpu().numpy().view(np.uint32))
        assert_rel_close(o["h"][rows], oracle_ffn(fg[rows], L["g"], L["u"], H))
        assert_rel_close(o["down"][rows], oracle_linear(o["h"][rows], L["d"], I))
