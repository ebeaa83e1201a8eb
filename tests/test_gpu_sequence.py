"""bitnet_decode_sequence on the GPU, through the C ABI.

Every op of a persistent sequence launch is compared
  * with the CPU oracle on the same inputs (integers exact, y within 1e-6
    relative), and
  * bitwise with the same op run alone (bitnet_linear / bitnet_ffn_gate_up,
    and their _norm forms),
and a sequence whose ops share buffers (read after write, write after read,
write after write) must leave every buffer exactly as running its ops one
after another does.  The full decode step the benchmark times (30 layers,
M = 8, every projection of every layer in one launch) is checked the same way."""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_fwd_b200 as tw
from gpu_util import DEV, assert_rel_close, f32_to_dev, make_weights, make_x
import synth

pytestmark = pytest.mark.gpu

H, I = 2560, 6912


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert tw.bitnet_device_status(clear=True) == 0


def oracle_linear(xf, W, k):
    y, acc, _, _ = oracle.bitlinear(np.ascontiguousarray(xf, np.float32), W["p_ref"], W["g_ref"], k)
    return y


def oracle_ffn(xf, Wg, Wu, k):
    h, _, _, _, _ = oracle.ffn_gate_up(np.ascontiguousarray(xf, np.float32), Wg["p_ref"], Wg["g_ref"],
                                       Wu["p_ref"], Wu["g_ref"], k)
    return h


def workspace(n_ops, m, k_max=I):
    return tw.bitnet_sequence_workspace(DEV, n_ops, m, k_max)


def counters_zero(ws, n_ops):
    return torch.count_nonzero(ws[:4 * (2 + 2 * n_ops)]) == 0


def run_seq(ops, m, ws=None):
    ws = workspace(len(ops), m, max(o.K for o in ops)) if ws is None else ws
    tw.bitnet_decode_sequence(ops, m, ws)
    torch.cuda.synchronize()
    assert counters_zero(ws, len(ops)), "counters must be left zeroed"
    return ws


def same_bits(a, b):
    a = a.cpu().numpy() if torch.is_tensor(a) else a
    b = b.cpu().numpy() if torch.is_tensor(b) else b
    return np.array_equal(np.ascontiguousarray(a).view(np.uint32), np.ascontiguousarray(b).view(np.uint32))


# ---------------------------------------------------------------- a decode step of a layer stack
def make_layer(seed, m, kinds=("outliers", "normal", "normal")):
    L = dict(q=make_weights(H, H, seed + 1), o=make_weights(H, H, seed + 2), g=make_weights(I, H, seed + 3),
             u=make_weights(I, H, seed + 4), d=make_weights(H, I, seed + 5))
    L["x"] = [make_x(m, H, seed + 10 + i, kinds[i]) for i in range(3)]
    L["out"] = {k: torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
                for k, n in (("q", H), ("o", H), ("h", I), ("down", H))}
    return L


def layer_ops(L, out=None):
    (xq, _), (xo, _), (xg, _) = L["x"]
    o = L["out"] if out is None else out
    return [tw.linear_op(xq, L["q"]["p"], L["q"]["g"], o["q"]),
            tw.linear_op(xo, L["o"]["p"], L["o"]["g"], o["o"]),
            tw.ffn_gate_up_op(xg, L["g"]["p"], L["g"]["g"], L["u"]["p"], L["u"]["g"], o["h"]),
            tw.linear_op(o["h"], L["d"]["p"], L["d"]["g"], o["down"])]


def check_layer(L, m, rows):
    (xq, fq), (xo, fo), (xg, fg) = L["x"]
    o = {k: v.cpu().numpy() for k, v in L["out"].items()}
    # alone, through the per-op entry points: bit-identical
    ref_q = tw.bitnet_linear(xq, L["q"]["p"], L["q"]["g"])
    ref_o = tw.bitnet_linear(xo, L["o"]["p"], L["o"]["g"])
    ref_h = tw.bitnet_ffn_gate_up(xg, L["g"]["p"], L["g"]["g"], L["u"]["p"], L["u"]["g"])
    ref_d = tw.bitnet_linear(ref_h, L["d"]["p"], L["d"]["g"])
    for got, ref in ((o["q"], ref_q), (o["o"], ref_o), (o["h"], ref_h), (o["down"], ref_d)):
        assert same_bits(got, ref)
    # against the oracle (stage-wise: the down projection quantises the GPU's h)
    assert_rel_close(o["q"][rows], oracle_linear(fq[rows], L["q"], H))
    assert_rel_close(o["o"][rows], oracle_linear(fo[rows], L["o"], H))
    assert_rel_close(o["h"][rows], oracle_ffn(fg[rows], L["g"], L["u"], H))
    assert_rel_close(o["down"][rows], oracle_linear(o["h"][rows], L["d"], I))


@pytest.mark.parametrize("m", [1, 8, 13, 64])
def test_layer_stack(m):
    """Two layers of (q, o, gate/up + ReLU^2, down on h), private outputs."""
    layers = [make_layer(1000 * (l + 1) + m, m) for l in range(2)]
    ops = sum((layer_ops(L) for L in layers), [])
    run_seq(ops, m)
    rows = np.arange(m) if m <= 8 else np.array(sorted({0, 1, m // 2, m - 2, m - 1}))
    for L in layers:
        check_layer(L, m, rows)


# ---------------------------------------------------------------- shapes
SHAPES = [  # (kind, K, N, x dtype)
    ("linear", 64, 8, "bf16"), ("linear", 128, 300, "bf16"), ("linear", 256, 256, "f32"),
    ("linear", 576, 1000, "bf16"), ("linear", 8192, 256, "bf16"), ("linear", 8192, 130, "f32"),
    ("linear", 6912, 2560, "f32"), ("linear", 2560, 640, "bf16"), ("linear", 2560, 3840, "bf16"),
    ("linear", 2560, 2560, "bf16"), ("ffn", 256, 136, "bf16"), ("ffn", 2560, 6912, "bf16"),
    ("ffn", 320, 17, "f32"), ("ffn", 704, 65, "bf16"),
]


def run_one(kind, k, n, dtype, m, seed, norm=False):
    x, xf = make_x(m, k, seed, "outliers" if m > 1 else "normal", dtype)
    W0 = make_weights(n, k, seed + 1)
    g = None
    if norm:
        g = np.ascontiguousarray(synth.activations_f32(1, k, seed + 3)[0] * np.float32(0.3) + np.float32(1.0))
    gd = None if g is None else f32_to_dev(g)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    if kind == "linear":
        run_seq([tw.linear_op(x, W0["p"], W0["g"], y, norm_g=gd)], m)
        ref = tw.bitnet_linear(x, W0["p"], W0["g"]) if gd is None else tw.bitnet_linear_norm(x, gd, W0["p"], W0["g"])
        xo = xf if g is None else oracle.rmsnorm(xf, g)[0]
        want = oracle_linear(xo, W0, k)
    else:
        W1 = make_weights(n, k, seed + 2)
        run_seq([tw.ffn_gate_up_op(x, W0["p"], W0["g"], W1["p"], W1["g"], y, norm_g=gd)], m)
        ref = (tw.bitnet_ffn_gate_up(x, W0["p"], W0["g"], W1["p"], W1["g"]) if gd is None else
               tw.bitnet_ffn_gate_up_norm(x, gd, W0["p"], W0["g"], W1["p"], W1["g"]))
        xo = xf if g is None else oracle.rmsnorm(xf, g)[0]
        want = oracle_ffn(xo, W0, W1, k)
    torch.cuda.synchronize()
    assert_rel_close(y.cpu().numpy(), want)
    assert same_bits(y, ref)


@pytest.mark.parametrize("kind,k,n,dtype", SHAPES)
@pytest.mark.parametrize("m", [1, 5, 8, 9])
def test_shapes_vs_oracle(kind, k, n, dtype, m):
    run_one(kind, k, n, dtype, m, 7 * k + n + m)


@pytest.mark.parametrize("kind,k,n,dtype", [("linear", 2560, 2560, "bf16"), ("ffn", 2560, 6912, "bf16"),
                                            ("linear", 6912, 2560, "f32"), ("ffn", 320, 17, "f32")])
@pytest.mark.parametrize("m", [16, 17, 32, 33, 64])
def test_token_tiles_vs_oracle(kind, k, n, dtype, m):
    """2, 4 and 8 tiles of 8 tokens, full and ragged."""
    run_one(kind, k, n, dtype, m, 11 * k + n + m)


@pytest.mark.parametrize("kind,k,n,dtype", [("linear", 2560, 2560, "bf16"), ("ffn", 2560, 6912, "bf16"),
                                            ("linear", 6912, 2560, "f32"), ("linear", 8192, 200, "f32"),
                                            ("ffn", 576, 100, "bf16")])
@pytest.mark.parametrize("m", [1, 8, 13])
def test_norm_ops_vs_oracle(kind, k, n, dtype, m):
    """Ops with an RMS-normalised input: bitwise equal to bitnet_linear_norm /
    bitnet_ffn_gate_up_norm, within 1e-6 of the oracle."""
    run_one(kind, k, n, dtype, m, 13 * k + n + m, norm=True)


# ---------------------------------------------------------------- shared buffers
def test_hazards_match_sequential_execution():
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
    for _ in range(3):  # repeated launches on one workspace
        run_seq(ops, m)

    rA, rB, rC = bufs()
    for kind, x, W, y in program(rA, rB, rC):
        if kind == "lin":
            tw.bitnet_linear(x, W["p"], W["g"], y=y)
        else:
            tw.bitnet_ffn_gate_up(x, W[0]["p"], W[0]["g"], W[1]["p"], W[1]["g"], h=y)
    torch.cuda.synchronize()
    for got, ref in ((A, rA), (B, rB), (C, rC)):
        assert same_bits(got, ref)


# ---------------------------------------------------------------- launches
def test_one_launch_graph_and_repeat():
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
    ws = workspace(3, m)
    c0 = tw.bitnet_launch_count()
    run_seq(ops, m, ws)
    assert tw.bitnet_launch_count() - c0 == 2  # the weights' tensor maps, then the sequence
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
        assert same_bits(a, b)
    assert counters_zero(ws, 3)


def test_huge_projection():
    """A gated FFN with 60000 output rows (938 row tasks): bit-identical to the per-op call and
    within 1e-6 of the oracle on sampled output columns."""
    m, k, n = 8, 256, 60000
    x, xf = make_x(m, k, 700, "outliers")
    G, U = make_weights(n, k, 701), make_weights(n, k, 702)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    c0 = tw.bitnet_launch_count()
    run_seq([tw.ffn_gate_up_op(x, G["p"], G["g"], U["p"], U["g"], y)], m)
    assert tw.bitnet_launch_count() - c0 == 2
    ref = tw.bitnet_ffn_gate_up(x, G["p"], G["g"], U["p"], U["g"])
    assert same_bits(y, ref)
    cols = np.random.default_rng(703).choice(n, 512, replace=False)
    Gs = dict(p_ref=G["p_ref"][cols], g_ref=G["g_ref"])
    Us = dict(p_ref=U["p_ref"][cols], g_ref=U["g_ref"])
    assert_rel_close(y.cpu().numpy()[:, cols], oracle_ffn(xf, Gs, Us, k))


def test_k_above_the_limit_is_rejected():
    m = 8
    x = torch.zeros((m, 8256), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((256, 8256 // 4), dtype=torch.uint8, device=DEV)
    g = torch.ones(4, dtype=torch.float32, device=DEV)
    y = torch.empty((m, 256), dtype=torch.float32, device=DEV)
    ws = workspace(1, m, 8192)
    c0 = tw.bitnet_launch_count()
    with pytest.raises(tw.BitnetError) as e:
        tw.bitnet_decode_sequence([tw.linear_op(x, w, g, y)], m, ws)
    assert e.value.status == tw.BITNET_ERR_UNSUPPORTED_SHAPE
    assert tw.bitnet_launch_count() == c0


def test_workspace_too_small_is_rejected():
    m = 8
    L = make_layer(800, m)
    ops = layer_ops(L)
    up = lambda v: (v + 255) // 256 * 256  # noqa: E731
    need = up(4 * (2 + 2 * 4)) + up(256 * 4 + 128) + sum(up(o.K * 8) + 512 for o in ops)  # documented exact size
    assert need < tw.bitnet_sequence_workspace_size(4, m, I)
    tw.bitnet_decode_sequence(ops, m, torch.zeros(need, dtype=torch.uint8, device=DEV))  # exactly enough
    torch.cuda.synchronize()
    ws = torch.zeros(need - 256, dtype=torch.uint8, device=DEV)
    c0 = tw.bitnet_launch_count()
    with pytest.raises(tw.BitnetError) as e:
        tw.bitnet_decode_sequence(ops, m, ws)
    assert e.value.status == tw.BITNET_ERR_WORKSPACE
    assert tw.bitnet_launch_count() == c0


# ---------------------------------------------------------------- the benchmark's decode step
def device_layer(seed, m, gen):
    """A layer whose latent weights and activations are drawn on the device (seeded torch
    generator) and packed by the library, as the benchmark does."""
    def w(n, k):
        lat = torch.randn((n, k), generator=gen, device=DEV, dtype=torch.float32) * 0.02
        p, g = tw.bitnet_pack_weights(lat)
        return dict(p=p, g=g)

    L = dict(q=w(H, H), o=w(H, H), g=w(I, H), u=w(I, H), d=w(H, I))
    L["x"] = [(torch.randn((m, H), generator=gen, device=DEV).to(torch.bfloat16), None) for _ in range(3)]
    L["out"] = {k: torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
                for k, n in (("q", H), ("o", H), ("h", I), ("down", H))}
    return L


def test_full_decode_step_of_the_benchmark():
    """The launch the benchmark times: 30 layers of (q, o, gate/up + ReLU^2, down on h) at
    M = 8 with per-layer outputs, 120 ops in one launch.  Every output of every layer is
    bitwise equal to the per-op calls; layers 0, 13 and 29 (weights and inputs from the seeded
    CPU generator) also match the oracle on every token.  Run twice on one workspace."""
    m, nl = 8, 30
    oracle_layers = (0, 13, 29)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(4242)
    layers = [make_layer(9000 + 10 * l, m) if l in oracle_layers else device_layer(l, m, gen) for l in range(nl)]
    ops = sum((layer_ops(L) for L in layers), [])
    groups = tw.bitnet_sequence_tasks(ops, m, tw.bitnet_num_sms())
    assert len(groups) == 2 * len(ops)
    ws = workspace(len(ops), m)
    for _ in range(2):
        run_seq(ops, m, ws)
    rows = np.arange(m)
    for l, L in enumerate(layers):
        if l in oracle_layers:
            check_layer(L, m, rows)
            continue
        (xq, _), (xo, _), (xg, _) = L["x"]
        o = L["out"]
        ref_q = tw.bitnet_linear(xq, L["q"]["p"], L["q"]["g"])
        ref_o = tw.bitnet_linear(xo, L["o"]["p"], L["o"]["g"])
        ref_h = tw.bitnet_ffn_gate_up(xg, L["g"]["p"], L["g"]["g"], L["u"]["p"], L["u"]["g"])
        ref_d = tw.bitnet_linear(ref_h, L["d"]["p"], L["d"]["g"])
        for got, ref in ((o["q"], ref_q), (o["o"], ref_o), (o["h"], ref_h), (o["down"], ref_d)):
            assert same_bits(got, ref), l


@pytest.mark.parametrize("m", [8, 13])
def test_list_longer_than_one_launch(m):
    """45 layers: 180 ops in one call, run as two launches of 128 and 52 ops.  Layer 32's q
    reads layer 31's down output, so the first op of the second launch reads what the last op
    of the first launch wrote.  Every output is bitwise equal to per-op calls in list order,
    and the counters of both workspace parts are left zeroed.  M = 13 takes the two-token-tile
    kernel and its larger workspace parts."""
    nl = 45
    gen = torch.Generator(device=DEV)
    gen.manual_seed(777)
    layers = [device_layer(l, m, gen) for l in range(nl)]
    spec = []
    for l, L in enumerate(layers):
        (xq, _), (xo, _), (xg, _) = L["x"]
        o = L["out"]
        if l == 32:
            xq = layers[31]["out"]["down"]
        spec += [("lin", xq, L["q"], o["q"]), ("lin", xo, L["o"], o["o"]), ("ffn", xg, (L["g"], L["u"]), o["h"]),
                 ("lin", o["h"], L["d"], o["down"])]
    ops = [tw.linear_op(x, w["p"], w["g"], y) if k == "lin" else
           tw.ffn_gate_up_op(x, w[0]["p"], w[0]["g"], w[1]["p"], w[1]["g"], y) for k, x, w, y in spec]
    n, cap = len(ops), tw.BITNET_SEQ_MAX_OPS
    assert n == 180 and spec[cap][1] is spec[cap - 1][3]
    ws = workspace(n, m)
    c0 = tw.bitnet_launch_count()
    tw.bitnet_decode_sequence(ops, m, ws)
    torch.cuda.synchronize()
    assert tw.bitnet_launch_count() - c0 == 4  # two launches of (tensor maps, sequence)
    assert tw.bitnet_device_status() == 0
    part0 = tw.bitnet_sequence_workspace_size(cap, m, I)
    assert counters_zero(ws, cap) and counters_zero(ws[part0:], n - cap)
    ref = {}
    for k, x, w, y in spec:
        xin = ref.get(x.data_ptr(), x)
        ref[y.data_ptr()] = (tw.bitnet_linear(xin, w["p"], w["g"]) if k == "lin" else
                             tw.bitnet_ffn_gate_up(xin, w[0]["p"], w[0]["g"], w[1]["p"], w[1]["g"]))
    for i, (k, x, w, y) in enumerate(spec):
        assert same_bits(y, ref[y.data_ptr()]), i


def test_degenerate_weights_in_a_sequence():
    """A sequence whose q projection has all-zero latents (gamma = 0) and whose gated FFN has
    an all-zero gate matrix, with one all-zero activation row: every output equals the per-op
    call bit for bit and is exactly zero where the definition makes it zero."""
    m = 8
    L = make_layer(860, m)
    zero = tw.bitnet_pack_weights(torch.zeros((H, H), device=DEV))
    zero_g = tw.bitnet_pack_weights(torch.zeros((I, H), device=DEV))
    (xq, _), (xo, _), (xg, _) = L["x"]
    xo = xo.clone()
    xo[3].zero_()
    o = L["out"]
    ops = [tw.linear_op(xq, zero[0], zero[1], o["q"]), tw.linear_op(xo, L["o"]["p"], L["o"]["g"], o["o"]),
           tw.ffn_gate_up_op(xg, zero_g[0], zero_g[1], L["u"]["p"], L["u"]["g"], o["h"]),
           tw.linear_op(o["h"], L["d"]["p"], L["d"]["g"], o["down"])]
    run_seq(ops, m)
    assert not o["q"].any() and not o["h"].any() and not o["down"].any() and not o["o"][3].any()
    assert same_bits(o["o"], tw.bitnet_linear(xo, L["o"]["p"], L["o"]["g"]))


def test_one_workspace_for_different_lists():
    """One workspace serves a 4-layer list, then a 45-layer list (two launches whose counters sit
    where the first list kept tensor maps and activations), then the 4-layer list again, then
    the 45-layer list after the workspace was filled with 0xff: every run gives the per-op
    results bit for bit."""
    m = 8
    gen = torch.Generator(device=DEV)
    gen.manual_seed(779)
    layers = [device_layer(l, m, gen) for l in range(45)]
    short = sum((layer_ops(L) for L in layers[:4]), [])
    long_ = sum((layer_ops(L) for L in layers), [])
    ws = torch.empty(max(tw.bitnet_sequence_workspace_size(len(short), m, I),
                         tw.bitnet_sequence_workspace_size(len(long_), m, I)), dtype=torch.uint8, device=DEV)
    ws.fill_(0xff)

    def check(ls):
        for L in ls:
            (xq, _), (xo, _), (xg, _) = L["x"]
            o = L["out"]
            ref_h = tw.bitnet_ffn_gate_up(xg, L["g"]["p"], L["g"]["g"], L["u"]["p"], L["u"]["g"])
            for got, ref in ((o["q"], tw.bitnet_linear(xq, L["q"]["p"], L["q"]["g"])),
                             (o["o"], tw.bitnet_linear(xo, L["o"]["p"], L["o"]["g"])), (o["h"], ref_h),
                             (o["down"], tw.bitnet_linear(ref_h, L["d"]["p"], L["d"]["g"]))):
                assert same_bits(got, ref)
            for t in o.values():
                t.fill_(float("nan"))

    for ops, ls in ((short, layers[:4]), (long_, layers), (short, layers[:4])):
        tw.bitnet_decode_sequence(ops, m, ws)
        torch.cuda.synchronize()
        assert tw.bitnet_device_status() == 0
        check(ls)
    ws.fill_(0xff)
    tw.bitnet_decode_sequence(long_, m, ws)
    torch.cuda.synchronize()
    assert tw.bitnet_device_status() == 0
    check(layers)


# ---------------------------------------------------------------- failure detection (no GPU fault)
def test_bounded_wait_runs_out_and_the_next_launch_is_correct():
    """A host-armed stall makes one op's weight-row tasks wait for a quantisation task that
    never runs.  With a 20 ms wait limit the launch ends by itself with BITNET_ERR_TIMEOUT in
    the device status word and leaves the workspace counters zeroed; the next launch, with the
    stall removed, gives the per-op results bit for bit and a clean status."""
    m = 8
    L = make_layer(850, m)
    ops = layer_ops(L)
    ws = workspace(len(ops), m)
    prev_limit = tw.bitnet_set_wait_limit_ns(20_000_000)
    prev_stall = tw.bitnet_set_sequence_test_stall(2)  # the gate/up op
    try:
        tw.bitnet_decode_sequence(ops, m, ws)
        torch.cuda.synchronize()
        assert tw.bitnet_device_status(clear=True) == tw.BITNET_ERR_TIMEOUT
        assert counters_zero(ws, len(ops))
    finally:
        tw.bitnet_set_sequence_test_stall(prev_stall)
        tw.bitnet_set_wait_limit_ns(prev_limit)
    run_seq(ops, m, ws)
    assert tw.bitnet_device_status(clear=False) == tw.BITNET_OK
    check_layer(L, m, np.arange(m))


def test_bounded_wait_in_the_second_launch_of_a_long_list():
    """A 132-op list (two launches) with the stall on op 130, the gate/up op of the last layer,
    in the second launch: the first launch completes and its outputs equal the per-op calls;
    the second ends by itself with BITNET_ERR_TIMEOUT; the counters of both workspace parts
    are left zeroed, and the next call without the stall is correct throughout."""
    m, nl = 8, 33
    gen = torch.Generator(device=DEV)
    gen.manual_seed(778)
    layers = [device_layer(l, m, gen) for l in range(nl)]
    ops = sum((layer_ops(L) for L in layers), [])
    n, cap = len(ops), tw.BITNET_SEQ_MAX_OPS
    ws = workspace(n, m)
    part0 = tw.bitnet_sequence_workspace_size(cap, m, I)

    def check(upto):
        for L in layers[:upto]:
            (xq, _), (xo, _), (xg, _) = L["x"]
            o = L["out"]
            ref_h = tw.bitnet_ffn_gate_up(xg, L["g"]["p"], L["g"]["g"], L["u"]["p"], L["u"]["g"])
            for got, ref in ((o["q"], tw.bitnet_linear(xq, L["q"]["p"], L["q"]["g"])),
                             (o["o"], tw.bitnet_linear(xo, L["o"]["p"], L["o"]["g"])), (o["h"], ref_h),
                             (o["down"], tw.bitnet_linear(ref_h, L["d"]["p"], L["d"]["g"]))):
                assert same_bits(got, ref)

    prev_limit = tw.bitnet_set_wait_limit_ns(20_000_000)
    prev_stall = tw.bitnet_set_sequence_test_stall(130)
    try:
        tw.bitnet_decode_sequence(ops, m, ws)
        torch.cuda.synchronize()
        assert tw.bitnet_device_status(clear=True) == tw.BITNET_ERR_TIMEOUT
        assert counters_zero(ws, cap) and counters_zero(ws[part0:], n - cap)
    finally:
        tw.bitnet_set_sequence_test_stall(prev_stall)
        tw.bitnet_set_wait_limit_ns(prev_limit)
    check(cap // 4)  # the 32 layers of the first launch
    run_seq(ops, m, ws)
    assert counters_zero(ws[part0:], n - cap)
    assert tw.bitnet_device_status(clear=False) == tw.BITNET_OK
    check(nl)


# ---------------------------------------------------------------- independent layers
@pytest.mark.parametrize("m", [1, 8, 13])
def test_private_layer_stack(m):
    """Layers with their own output buffers share no memory: their tasks interleave freely.
    Every op gives the per-op results bit for bit; the oracle checks the gate/up -> down chain."""
    layers = [make_layer(3000 + 100 * l + m, m, ("normal",) * 3) for l in range(4)]
    ops = sum((layer_ops(L) for L in layers), [])
    run_seq(ops, m)
    rows = np.arange(m) if m <= 8 else np.array([0, m // 2, m - 1])
    for L in layers:
        check_layer(L, m, rows)
