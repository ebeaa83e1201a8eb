"""RMS normalisation fused in front of the quantiser, on the GPU through the C ABI.

Bit-exact against the oracle: x_q, per-token scales, row sums and int32
accumulators; BitLinear / FFN outputs within 1e-6 relative.  Both sides use
the correctly rounded sum of squares (the exact sum rounded once), so no
reduction order enters and equality is exact."""
import math

import numpy as np
import pytest
import torch

import oracle
import ternary_weight_fwd_b200 as tw
from gpu_util import DEV, assert_rel_close, f32_to_dev, make_weights, make_x
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_state():
    prev = tw.bitnet_set_dispatch(tw.BITNET_DISPATCH_AUTO)
    yield
    tw.bitnet_set_dispatch(prev)
    assert tw.bitnet_device_status(clear=True) == 0


def norm_weight(k, seed):
    """Per-feature weights around 1 with some negative entries."""
    g = synth.activations_f32(1, k, seed)[0] * np.float32(0.3) + np.float32(1.0)
    return np.ascontiguousarray(g, np.float32)


@pytest.mark.parametrize("m,k,kind,dtype,eps", [
    (1, 64, "normal", "bf16", 1e-5), (7, 320, "outliers", "bf16", 1e-5), (64, 2560, "outliers", "bf16", 1e-5),
    (4096, 2560, "student_t_rows", "bf16", 1e-5), (33, 6912, "normal", "f32", 1e-5), (5, 8192, "normal", "bf16", 1e-5),
    (9, 2560, "normal", "bf16", 0.0), (3, 256, "normal", "f32", 0.5),
])
def test_rmsnorm_quant_bit_exact(m, k, kind, dtype, eps):
    xd, xf = make_x(m, k, 900 + m + k, kind, dtype)
    g = norm_weight(k, 901 + k)
    x_q, s, rs = tw.bitnet_rmsnorm_quant(xd, f32_to_dev(g), eps)
    torch.cuda.synchronize()
    rq, rsc, rrs, _, _ = oracle.rmsnorm_quant_act(xf, g, eps)
    assert np.array_equal(x_q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rsc.view(np.uint32))
    assert np.array_equal(rs.cpu().numpy(), rrs)


def test_rmsnorm_quant_special_rows():
    """Tiny rows (eps dominates), a zero row and a constant row."""
    k = 512
    x = synth.activations_f32(4, k, 902) * np.float32(1e-4)
    x[1] = 0.0
    x[2] = np.float32(-2.5)
    g = norm_weight(k, 903)
    x_q, s, rs = tw.bitnet_rmsnorm_quant(f32_to_dev(x), f32_to_dev(g))
    torch.cuda.synchronize()
    rq, rsc, rrs, _, _ = oracle.rmsnorm_quant_act(x, g)
    assert np.array_equal(x_q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rsc.view(np.uint32))
    assert np.all(x_q.cpu().numpy()[1] == 0)


def _sq_terms(p):
    """binary32 values whose squares add up to exactly 2^p."""
    return [2.0 ** (p // 2)] if p % 2 == 0 else [2.0 ** ((p - 1) // 2)] * 2


def _range_rows(k, seed):
    """Rows whose sums of squares need more than a 128-bit window (a value more than 33
    binades below the largest), rows sitting exactly on a rounding tie of the sum, rows of
    subnormals, and ordinary rows next to them (two rows share a CTA at K <= 4096)."""
    rng = np.random.default_rng(seed)
    rows = []
    rows.append((rng.standard_normal(k) * 2.0 ** rng.integers(-70, 60, k)).astype(np.float32))
    rows.append(rng.standard_normal(k).astype(np.float32))
    r = rng.standard_normal(k).astype(np.float32)
    r[k // 3] = np.float32(2.0 ** -60)  # one value 60 binades down: long accumulator
    rows.append(r)
    rows.append((rng.standard_normal(k) * 2.0 ** rng.integers(-149, -120, k)).astype(np.float32))
    for v0 in rng.uniform(1.0, 2.0, 3).astype(np.float32):
        e = math.frexp(float(v0) * float(v0))[1] - 1
        for terms in (_sq_terms(e - 53), _sq_terms(e - 52) + _sq_terms(e - 53), _sq_terms(e - 53) + [2.0 ** -40]):
            row = np.zeros(k, np.float32)
            vals = [v0] + terms
            row[rng.choice(k, len(vals), replace=False)] = vals
            rows.append(row)
    r = np.zeros(k, np.float32)
    r[0] = 1.0
    r[1:4096 if k > 4096 else k] = 2.0 ** -27  # one large square among many tiny ones
    rows.append(r)
    return np.stack(rows).astype(np.float32)


@pytest.mark.parametrize("k", [256, 2560, 6912])
def test_rmsnorm_sumsq_wide_range_and_ties(k):
    """Exact sums of squares on rows of every path: the 128-bit window, the long accumulator
    (values more than 33 binades below the row's largest), exact ties and subnormals."""
    x_all = _range_rows(k, 950 + k)
    g = norm_weight(k, 951)
    for eps in (1e-5, 0.0):
        # with eps = 0 the subnormal row (index 3) would give 1/rms beyond binary32
        x = x_all if eps else np.delete(x_all, 3, axis=0)
        x_q, s, rs = tw.bitnet_rmsnorm_quant(f32_to_dev(x), f32_to_dev(g), eps)
        torch.cuda.synchronize()
        rq, rsc, rrs, _, _ = oracle.rmsnorm_quant_act(x, g, eps)
        assert np.array_equal(x_q.cpu().numpy(), rq)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), rsc.view(np.uint32))
        assert np.array_equal(rs.cpu().numpy(), rrs)


@pytest.mark.parametrize("m,k,n", [(1, 2560, 2560), (8, 2560, 640), (8, 6912, 2560), (300, 2560, 512), (4096, 2560, 256)])
def test_linear_norm_vs_oracle(m, k, n):
    dtype = "f32" if k == 6912 else "bf16"
    xd, xf = make_x(m, k, 910 + m + n, "outliers" if m < 64 else "student_t_rows", dtype)
    g = norm_weight(k, 911 + k)
    W = make_weights(n, k, 912 + n)
    acc = torch.full((m, n), -7, dtype=torch.int32, device=DEV)
    y = tw.bitnet_linear_norm(xd, f32_to_dev(g), W["p"], W["g"], acc_out=acc)
    torch.cuda.synchronize()
    rows = np.arange(m) if m <= 300 else np.array([0, 1, 127, 128, 2048, m - 1])
    y_ref, acc_ref, _, _ = oracle.bitlinear_norm(xf[rows], g, W["p_ref"], W["g_ref"], k)
    assert np.array_equal(acc.cpu().numpy()[rows].astype(np.int64), acc_ref)
    assert_rel_close(y.cpu().numpy()[rows], y_ref)


@pytest.mark.parametrize("m", [8, 200])
def test_ffn_gate_up_norm_vs_oracle(m):
    k, n = 2560, 6912
    xd, xf = make_x(m, k, 920 + m)
    g = norm_weight(k, 921)
    G, U = make_weights(n, k, 922), make_weights(n, k, 923)
    h = tw.bitnet_ffn_gate_up_norm(xd, f32_to_dev(g), G["p"], G["g"], U["p"], U["g"])
    torch.cuda.synchronize()
    rows = np.arange(min(m, 8))
    xn, _ = oracle.rmsnorm(xf[rows], g)
    h_ref = oracle.ffn_gate_up(xn, G["p_ref"], G["g_ref"], U["p_ref"], U["g_ref"], k)[0]
    assert_rel_close(h.cpu().numpy()[rows], h_ref)


def test_norm_matches_separate_norm_then_linear():
    """The fused path equals normalising first (oracle, to fp32) and calling bitnet_linear."""
    m, k, n = 16, 2560, 2560
    xd, xf = make_x(m, k, 930)
    g = norm_weight(k, 931)
    W = make_weights(n, k, 932)
    y1 = tw.bitnet_linear_norm(xd, f32_to_dev(g), W["p"], W["g"])
    xn, _ = oracle.rmsnorm(xf, g)
    y2 = tw.bitnet_linear(f32_to_dev(xn), W["p"], W["g"])
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))


def test_fused_decode_dispatch_is_rejected_with_norm():
    tw.bitnet_set_dispatch(tw.BITNET_DISPATCH_DECODE_FUSED)
    xd, _ = make_x(4, 256, 940)
    W = make_weights(256, 256, 941)
    with pytest.raises(tw.BitnetError) as e:
        tw.bitnet_linear_norm(xd, f32_to_dev(norm_weight(256, 942)), W["p"], W["g"])
    assert e.value.status == tw.BITNET_ERR_UNSUPPORTED_SHAPE
