"""CPU oracle for the BitLinear forward (W1.58A8) -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The product path (the CUDA library and its Python
binding) never does, and shares no code with it.

Each function is a thin numpy/ctypes wrapper over the plain C in
``bitnet_oracle.c``; the C file states which passage of the BitNet model page
each step follows and which reading was taken where the page is silent.
Every function here is pinned by ``tests/test_oracle_pins.py``.
"""
import ctypes
import numpy as np

from . import build as _build

_lib = None


def _bind(path):
    """Load a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int64
    F = ctypes.c_float
    sig = {
        "oracle_bf16_to_f32": ([P, I, P], None),
        "oracle_absmean_f64": ([P, I, I], ctypes.c_double),
        "oracle_gamma": ([P, I, I], F),
        "oracle_ternarize": ([P, I, I, F, F, P], None),
        "oracle_pack": ([P, I, I, P], None),
        "oracle_unpack": ([P, I, I, P], I),
        "oracle_quant_act": ([P, I, I, P, P, P], None),
        "oracle_int_matmul": ([P, P, I, I, I, P], None),
        "oracle_int_dot_samples": ([P, P, I, P, P, I, P], None),
        "oracle_dequant": ([P, P, F, I, I, P], None),
        "oracle_relu2_gate": ([P, P, I, P], None),
        "oracle_sumsq": ([P, I], ctypes.c_double),
        "oracle_rmsnorm": ([P, P, I, I, F, P, P], None),
        "oracle_quant_act_amax": ([P, I, I, P, P, P, P], None),
        "oracle_epilogue_f32": ([P, P, P, F, F, I, I, P], None),
        "oracle_f32_to_bf16": ([P, I, P], None),
        "oracle_row_absmax": ([P, I, I, P], None),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(_build.build())
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


QUANT_EPS = 1e-5  # eps of gamma + eps and floor of max|x| (as fp32)


def bf16_to_f32(bits):
    """bf16 bit patterns (uint16) -> float32, exactly."""
    src, p = _c(bits, np.uint16)
    out = np.empty(src.shape, np.float32)
    _load().oracle_bf16_to_f32(p, src.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


def absmean_f64(w):
    w, p = _c(w, np.float32)
    n, k = w.shape
    return float(_load().oracle_absmean_f64(p, n, k))


def gamma(w):
    """gamma = mean|W| (binary64 in canonical row order, rounded to fp32)."""
    w, p = _c(w, np.float32)
    n, k = w.shape
    return np.float32(_load().oracle_gamma(p, n, k))


def ternarize(w, gamma_, eps=QUANT_EPS):
    w, p = _c(w, np.float32)
    n, k = w.shape
    out = np.empty((n, k), np.int8)
    _load().oracle_ternarize(p, n, k, float(gamma_), float(np.float32(eps)),
                             out.ctypes.data_as(ctypes.c_void_p))
    return out


def pack(w_q):
    w_q, p = _c(w_q, np.int8)
    n, k = w_q.shape
    assert k % 16 == 0
    out = np.empty((n, k // 4), np.uint8)
    _load().oracle_pack(p, n, k, out.ctypes.data_as(ctypes.c_void_p))
    return out


def unpack(packed, k):
    packed, p = _c(packed, np.uint8)
    n = packed.shape[0]
    out = np.empty((n, k), np.int8)
    bad = _load().oracle_unpack(p, n, k, out.ctypes.data_as(ctypes.c_void_p))
    return out, int(bad)


def pack_weights(w, eps=QUANT_EPS):
    """Whole offline step: returns (packed uint8 [N][K/4], gamma fp32, W_q int8)."""
    g = gamma(w)
    w_q = ternarize(w, g, eps)
    return pack(w_q), g, w_q


def quant_act(x, amax=None):
    """x: float32 [M][K] (exact bf16 values or fp32). Returns (x_q, s, rowsum).

    amax: optional float32 [M] per-token maxima used instead of max|x|."""
    x, p = _c(x, np.float32)
    m, k = x.shape
    x_q = np.empty((m, k), np.int8)
    s = np.empty(m, np.float32)
    rs = np.empty(m, np.int32)
    out = (x_q.ctypes.data_as(ctypes.c_void_p), s.ctypes.data_as(ctypes.c_void_p),
           rs.ctypes.data_as(ctypes.c_void_p))
    if amax is None:
        _load().oracle_quant_act(p, m, k, *out)
    else:
        a, pa = _c(amax, np.float32)
        assert a.shape == (m,)
        _load().oracle_quant_act_amax(p, m, k, pa, *out)
    return x_q, s, rs


def int_matmul(x_q, w_q):
    x_q, px = _c(x_q, np.int8)
    w_q, pw = _c(w_q, np.int8)
    m, k = x_q.shape
    n, k2 = w_q.shape
    assert k == k2
    acc = np.empty((m, n), np.int64)
    _load().oracle_int_matmul(px, pw, m, n, k, acc.ctypes.data_as(ctypes.c_void_p))
    return acc


def int_dot_samples(x_q, w_q, m_idx, n_idx):
    x_q, px = _c(x_q, np.int8)
    w_q, pw = _c(w_q, np.int8)
    mi, pm = _c(m_idx, np.int64)
    ni, pn = _c(n_idx, np.int64)
    assert mi.shape == ni.shape
    acc = np.empty(mi.shape, np.int64)
    _load().oracle_int_dot_samples(px, pw, x_q.shape[1], pm, pn, mi.size,
                                   acc.ctypes.data_as(ctypes.c_void_p))
    return acc


def dequant(acc, s, gamma_):
    acc, pa = _c(acc, np.int64)
    s, ps = _c(s, np.float32)
    m, n = acc.shape
    y = np.empty((m, n), np.float64)
    _load().oracle_dequant(pa, ps, float(gamma_), m, n, y.ctypes.data_as(ctypes.c_void_p))
    return y


def relu2_gate(g, u):
    g, pg = _c(g, np.float64)
    u, pu = _c(u, np.float64)
    assert g.shape == u.shape
    h = np.empty(g.shape, np.float64)
    _load().oracle_relu2_gate(pg, pu, g.size, h.ctypes.data_as(ctypes.c_void_p))
    return h


def bitlinear(x, packed, gamma_, k):
    """Full forward from already-packed weights: (y fp64, acc int64, x_q, s)."""
    w_q, bad = unpack(packed, k)
    assert bad == 0
    x_q, s, _ = quant_act(x)
    acc = int_matmul(x_q, w_q)
    return dequant(acc, s, gamma_), acc, x_q, s


def ffn_gate_up(x, packed_g, gamma_g, packed_u, gamma_u, k):
    """Fused gate/up forward: (h fp64, acc_g, acc_u, x_q, s)."""
    yg, acc_g, x_q, s = bitlinear(x, packed_g, gamma_g, k)
    yu, acc_u, _, _ = bitlinear(x, packed_u, gamma_u, k)
    return relu2_gate(yg, yu), acc_g, acc_u, x_q, s


RMS_EPS = 1e-5  # rms_norm_eps of BitNetConfig


def sumsq(row):
    """Sum of squares of one row (binary64, the fixed partial/pairing order)."""
    row, p = _c(row, np.float32)
    return float(_load().oracle_sumsq(p, row.shape[0]))


def rmsnorm(x, g, eps=RMS_EPS):
    """x: float32 [M][K], g: float32 [K]. Returns (y float32 [M][K], r float32 [M])."""
    x, px = _c(x, np.float32)
    g, pg = _c(g, np.float32)
    m, k = x.shape
    y = np.empty((m, k), np.float32)
    r = np.empty(m, np.float32)
    _load().oracle_rmsnorm(px, pg, m, k, float(eps), y.ctypes.data_as(ctypes.c_void_p),
                           r.ctypes.data_as(ctypes.c_void_p))
    return y, r


def rmsnorm_quant_act(x, g, eps=RMS_EPS):
    """RMS normalisation followed by the per-token absmax quantiser: (x_q, s, rowsum, y, r)."""
    y, r = rmsnorm(x, g, eps)
    x_q, s, rs = quant_act(y)
    return x_q, s, rs, y, r


def bitlinear_norm(x, g, packed, gamma_, k, eps=RMS_EPS):
    """BitLinear of the RMS-normalised input: (y fp64, acc, x_q, s)."""
    xn, _ = rmsnorm(x, g, eps)
    return bitlinear(xn, packed, gamma_, k)


def epilogue_f32(acc_g, s, gamma_g, acc_u=None, gamma_u=0.0):
    """The fp32 epilogue value of every output (y32, or h32 when acc_u is given)."""
    ag, pg = _c(acc_g, np.int64)
    sv, ps = _c(s, np.float32)
    m, n = ag.shape
    pu = None
    if acc_u is not None:
        au, pu = _c(acc_u, np.int64)
        assert au.shape == ag.shape
    y = np.empty((m, n), np.float32)
    _load().oracle_epilogue_f32(pg, pu, ps, float(gamma_g), float(gamma_u), m, n,
                                y.ctypes.data_as(ctypes.c_void_p))
    return y


def f32_to_bf16(v):
    """float32 -> bf16 bit patterns (uint16), round to nearest even."""
    src, p = _c(v, np.float32)
    out = np.empty(src.shape, np.uint16)
    _load().oracle_f32_to_bf16(p, src.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


def row_absmax(v):
    """float32 [M][N] -> float32 [M], max |v| of each row."""
    src, p = _c(v, np.float32)
    m, n = src.shape
    out = np.empty(m, np.float32)
    _load().oracle_row_absmax(p, m, n, out.ctypes.data_as(ctypes.c_void_p))
    return out


def bitlinear_ex(x, packed, gamma_, k, y_dtype="f32", x_amax=None, packed_u=None, gamma_u=None):
    """BitLinear (or, with packed_u, the gated FFN) with its output as stored.

    Returns (y, y_amax): y float32 [M][N] (y_dtype "f32") or bf16 bit patterns
    uint16 (y_dtype "bf16"); y_amax float32 [M] = max |stored value| per row.
    x_amax: optional per-token maxima handed to the quantiser."""
    w_q, bad = unpack(packed, k)
    assert bad == 0
    x_q, s, _ = quant_act(x, x_amax)
    acc = int_matmul(x_q, w_q)
    acc_u = None
    if packed_u is not None:
        wu, bad = unpack(packed_u, k)
        assert bad == 0
        acc_u = int_matmul(x_q, wu)
    y32 = epilogue_f32(acc, s, gamma_, acc_u, 0.0 if gamma_u is None else gamma_u)
    if y_dtype == "f32":
        return y32, row_absmax(y32)
    assert y_dtype == "bf16"
    yb = f32_to_bf16(y32)
    return yb, row_absmax(bf16_to_f32(yb))
