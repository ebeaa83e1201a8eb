"""bf16 outputs, emitted per-token maxima and given maxima (bitnet_linear_ex /
bitnet_ffn_gate_up_ex) on the GPU, through the C ABI, against the oracle.

The oracle fixes the stored fp32 value as fl(acc * fl(gamma / s)) (gated:
fl(fl(p * p) * u)), so every comparison here is exact:
  * fp32 outputs bit-identical to the oracle's fp32 epilogue value (and to the
    plain entry points);
  * bf16 outputs bit-identical to the oracle's nearest-even rounding of it;
  * emitted maxima bit-identical to the oracle's maxima of the stored values;
  * a BitLinear fed the emitted maxima bit-identical to one that reduces x
    itself.
Every kernel path is run: the fused cluster decode kernel, the quantiser +
row-split decode kernel, and the quantiser + tcgen05 prefill kernel (TMA
stores for 16-byte rows, plain stores otherwise)."""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_fwd_b200 as tw
from gpu_util import DEV, make_weights, make_x, sample_rows

pytestmark = pytest.mark.gpu

PATHS = {"cluster": tw.BITNET_DISPATCH_DECODE_FUSED, "decode": tw.BITNET_DISPATCH_DECODE,
         "prefill": tw.BITNET_DISPATCH_PREFILL}


@pytest.fixture(autouse=True)
def reset_dispatch():
    prev = tw.bitnet_set_dispatch(tw.BITNET_DISPATCH_AUTO)
    yield
    tw.bitnet_set_dispatch(prev)
    assert tw.bitnet_device_status(clear=True) == 0


def bits16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def bits32(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def oracle_out(xf, W, k, y_dtype, U=None, x_amax=None, rows=None):
    xs = xf if rows is None else xf[rows]
    xa = None if x_amax is None else (x_amax if rows is None else x_amax[rows])
    if U is None:
        return oracle.bitlinear_ex(xs, W["p_ref"], W["g_ref"], k, y_dtype, x_amax=xa)
    return oracle.bitlinear_ex(xs, W["p_ref"], W["g_ref"], k, y_dtype, x_amax=xa, packed_u=U["p_ref"],
                               gamma_u=U["g_ref"])


def run(x, W, U, y_dtype, want_amax, x_amax=None):
    m = x.shape[0]
    amax = torch.full((m,), float("nan"), dtype=torch.float32, device=DEV) if want_amax else None
    if U is None:
        y = tw.bitnet_linear_ex(x, W["p"], W["g"], x_amax=x_amax, y_dtype=y_dtype, y_amax=amax)
    else:
        y = tw.bitnet_ffn_gate_up_ex(x, W["p"], W["g"], U["p"], U["g"], x_amax=x_amax, h_dtype=y_dtype, h_amax=amax)
    torch.cuda.synchronize()
    return y, amax


CASES = [  # (path, m, k, n)
    ("cluster", 1, 2560, 2560), ("cluster", 5, 512, 1000), ("cluster", 8, 2560, 640), ("cluster", 13, 1024, 777),
    ("cluster", 64, 512, 384),
    ("decode", 3, 512, 1000), ("decode", 9, 2560, 640), ("decode", 64, 256, 136),
    ("prefill", 200, 512, 1000), ("prefill", 300, 1024, 777), ("prefill", 129, 256, 260), ("prefill", 4, 512, 264),
]


@pytest.mark.parametrize("ffn", [False, True], ids=["linear", "ffn"])
@pytest.mark.parametrize("path,m,k,n", CASES)
def test_outputs_and_maxima_vs_oracle(path, m, k, n, ffn):
    tw.bitnet_set_dispatch(PATHS[path])
    seed = 31 * m + k + 7 * n + (1 if ffn else 0)
    x, xf = make_x(m, k, seed, "outliers" if m % 2 else "normal")
    W = make_weights(n, k, seed + 1)
    U = make_weights(n, k, seed + 2) if ffn else None
    rows = None if m * k * n <= 300 * 1024 * 1000 else sample_rows(m, 24, seed)
    sel = slice(None) if rows is None else rows

    y32, a32 = run(x, W, U, torch.float32, True)
    yb, ab = run(x, W, U, torch.bfloat16, True)
    ref32, ref_a32 = oracle_out(xf, W, k, "f32", U, rows=rows)
    refb, ref_ab = oracle_out(xf, W, k, "bf16", U, rows=rows)

    assert np.array_equal(bits32(y32.cpu().numpy()[sel]), bits32(ref32)), "fp32 output differs from the oracle"
    assert np.array_equal(bits32(a32.cpu().numpy()[sel]), bits32(ref_a32)), "fp32 output maxima differ"
    assert np.array_equal(bits16(yb)[sel], refb), "bf16 output differs from the oracle"
    assert np.array_equal(bits32(ab.cpu().numpy()[sel]), bits32(ref_ab)), "bf16 output maxima differ"
    # the plain entry points store the same fp32 values
    plain = (tw.bitnet_linear(x, W["p"], W["g"]) if U is None
             else tw.bitnet_ffn_gate_up(x, W["p"], W["g"], U["p"], U["g"]))
    assert torch.equal(plain.view(torch.int32), y32.view(torch.int32))
    # every row: maxima = max |stored| computed from the GPU's own outputs
    assert torch.equal(ab, yb.float().abs().amax(dim=1)) and torch.equal(a32, y32.abs().amax(dim=1))


@pytest.mark.parametrize("path", ["cluster", "decode", "prefill"])
@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_chain_through_emitted_maxima(path, y_dtype):
    """gate/up emits h and its maxima; the down projection fed those maxima
    equals the one that reduces h itself, and the oracle's."""
    tw.bitnet_set_dispatch(PATHS[path])
    m = 200 if path == "prefill" else 8
    H, I = 512, 1024
    x, xf = make_x(m, H, 900 + m)
    G, U = make_weights(I, H, 901), make_weights(I, H, 902)
    D = make_weights(H, I, 903)
    h, h_amax = run(x, G, U, y_dtype, True)
    d_given, d_amax = run(h, D, None, y_dtype, True, x_amax=h_amax)
    d_self, d_amax_self = run(h, D, None, y_dtype, True)
    assert torch.equal(d_given.view(torch.int16 if y_dtype == torch.bfloat16 else torch.int32),
                       d_self.view(torch.int16 if y_dtype == torch.bfloat16 else torch.int32))
    assert torch.equal(d_amax, d_amax_self)
    hf = h.float().cpu().numpy()
    ref, ref_a = oracle_out(hf, D, I, "bf16" if y_dtype == torch.bfloat16 else "f32",
                            x_amax=h_amax.cpu().numpy())
    got = bits16(d_given) if y_dtype == torch.bfloat16 else bits32(d_given.cpu().numpy())
    assert np.array_equal(got, ref if y_dtype == torch.bfloat16 else bits32(ref))
    assert np.array_equal(bits32(d_amax.cpu().numpy()), bits32(ref_a))


@pytest.mark.parametrize("path", ["cluster", "decode", "prefill"])
def test_given_maxima_are_used(path):
    """A given maximum larger than the true one changes the scale exactly as
    the oracle's quantiser with that maximum does."""
    tw.bitnet_set_dispatch(PATHS[path])
    m = 130 if path == "prefill" else 6
    k, n = 512, 384
    x, xf = make_x(m, k, 950)
    W = make_weights(n, k, 951)
    given = (np.abs(xf).max(axis=1) * np.float32(2.5)).astype(np.float32)
    y, _ = run(x, W, None, torch.float32, False, x_amax=torch.from_numpy(given).to(DEV))
    ref, _ = oracle_out(xf, W, k, "f32", x_amax=given)
    assert np.array_equal(bits32(y.cpu().numpy()), bits32(ref))


@pytest.mark.parametrize("path", ["cluster", "decode", "prefill"])
def test_maxima_are_rezeroed_every_call(path):
    """Large outputs first, then small ones into the same maxima buffer, also
    replayed from a CUDA graph: each call's maxima are its own."""
    tw.bitnet_set_dispatch(PATHS[path])
    m = 140 if path == "prefill" else 8
    k, n = 256, 512
    xb, _ = make_x(m, k, 960)
    xs = (xb.float() * 1e-3).to(torch.bfloat16)
    W = make_weights(n, k, 961)
    amax = torch.empty(m, dtype=torch.float32, device=DEV)
    out = torch.empty((m, n), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(tw.bitnet_workspace_size(m, n, k), dtype=torch.uint8, device=DEV)
    for x in (xb, xs):
        tw.bitnet_linear_ex(x, W["p"], W["g"], y=out, y_amax=amax, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(amax, out.float().abs().amax(dim=1))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        tw.bitnet_linear_ex(xb, W["p"], W["g"], y=out, y_amax=amax, workspace=ws, stream=s)  # warm-up
        with torch.cuda.graph(g, stream=s):
            tw.bitnet_linear_ex(xb, W["p"], W["g"], y=out, y_amax=amax, workspace=ws, stream=s)
            tw.bitnet_linear_ex(xs, W["p"], W["g"], y=out, y_amax=amax, workspace=ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(amax, out.float().abs().amax(dim=1))
    ref = tw.bitnet_linear_ex(xs, W["p"], W["g"], y_dtype=torch.bfloat16)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("m", [4, 200])
def test_norm_with_bf16_output_and_maxima(m):
    """RMS normalisation in front, bf16 output and emitted maxima together."""
    k, n = 1024, 640
    x, xf = make_x(m, k, 970 + m)
    g = np.random.default_rng(971).uniform(0.5, 1.5, k).astype(np.float32)
    W = make_weights(n, k, 972)
    amax = torch.empty(m, dtype=torch.float32, device=DEV)
    y = tw.bitnet_linear_ex(x, W["p"], W["g"], norm_g=torch.from_numpy(g).to(DEV), y_dtype=torch.bfloat16,
                            y_amax=amax)
    torch.cuda.synchronize()
    xn, _ = oracle.rmsnorm(xf, g)
    ref, ref_a = oracle.bitlinear_ex(xn, W["p_ref"], W["g_ref"], k, "bf16")
    assert np.array_equal(bits16(y), ref)
    assert np.array_equal(bits32(amax.cpu().numpy()), bits32(ref_a))
