"""The C-ABI library builds, loads and exports every declared entry point; host-side
argument validation works without a GPU (no compute is launched here)."""
import ctypes
import os
import re
import subprocess

import pytest

import ternary_weight_fwd_b200 as tw
from ternary_weight_fwd_b200 import build as tw_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(bitnet_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    tw_build.build()
    return tw.load_library()


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("bitnet_pack_weights", "bitnet_quant_act", "bitnet_linear", "bitnet_ffn_gate_up"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", tw.LIB_PATH]).decode()
    exported = set(re.findall(r"\bT (bitnet_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert getattr(lib, n) is not None


def test_build_targets_sm100a_only():
    cmd = tw_build.nvcc_cmd("out.so")
    gencodes = [cmd[i + 1] for i, c in enumerate(cmd) if c == "-gencode"]
    assert gencodes == ["arch=compute_100a,code=sm_100a"]


def test_status_strings(lib):
    for code, name in [(0, "BITNET_OK"), (1, "BITNET_ERR_INVALID_ARG"), (2, "BITNET_ERR_UNSUPPORTED_SHAPE"),
                       (3, "BITNET_ERR_MISALIGNED"), (4, "BITNET_ERR_CUDA"), (5, "BITNET_ERR_TIMEOUT"),
                       (6, "BITNET_ERR_WORKSPACE")]:
        assert tw.bitnet_status_string(code) == name
    assert tw.bitnet_status_string(99) == "BITNET_ERR_UNKNOWN"


def test_workspace_sizes(lib):
    assert tw.bitnet_pack_workspace_size(2560, 6912) == 2560 * 8
    # x_q (M*K rounded to 256) + scales + row sums (each M*4 rounded to 256)
    assert tw.bitnet_workspace_size(1, 2560, 2560) == 2560 + 256 + 256
    assert tw.bitnet_workspace_size(4096, 6912, 2560) == 4096 * 2560 + 2 * 16384
    assert tw.bitnet_workspace_size(0, 1, 64) == 0


def test_dispatch_setter(lib):
    prev = lib.bitnet_set_dispatch(tw.BITNET_DISPATCH_PREFILL)
    try:
        assert lib.bitnet_set_dispatch(7) == -1
        assert lib.bitnet_set_dispatch(tw.BITNET_DISPATCH_DECODE) == tw.BITNET_DISPATCH_PREFILL
    finally:
        lib.bitnet_set_dispatch(prev)


FAKE = 1 << 20  # a 16-byte aligned non-null "device" address; never dereferenced


@pytest.mark.parametrize("case,expect", [
    (dict(M=0), tw.BITNET_ERR_INVALID_ARG),
    (dict(N=0), tw.BITNET_ERR_INVALID_ARG),
    (dict(K=96), tw.BITNET_ERR_UNSUPPORTED_SHAPE),
    (dict(K=0), tw.BITNET_ERR_INVALID_ARG),
    (dict(K=65536 + 64), tw.BITNET_ERR_UNSUPPORTED_SHAPE),
    (dict(x=0), tw.BITNET_ERR_INVALID_ARG),
    (dict(w=0), tw.BITNET_ERR_INVALID_ARG),
    (dict(gamma=0), tw.BITNET_ERR_INVALID_ARG),
    (dict(y=0), tw.BITNET_ERR_INVALID_ARG),
    (dict(dtype=5), tw.BITNET_ERR_INVALID_ARG),
    (dict(x=FAKE + 8), tw.BITNET_ERR_MISALIGNED),
    (dict(y=FAKE + 4), tw.BITNET_ERR_MISALIGNED),
    (dict(ws=0), tw.BITNET_ERR_WORKSPACE),
    (dict(ws_bytes=10), tw.BITNET_ERR_WORKSPACE),
])
def test_linear_rejects_before_launch(lib, case, expect):
    a = dict(M=4, N=256, K=256, x=FAKE, w=FAKE, gamma=FAKE, y=FAKE, dtype=0, ws=FAKE, ws_bytes=1 << 20)
    a.update(case)
    P = ctypes.c_void_p
    st = lib.bitnet_linear(P(a["x"] or None), a["dtype"], a["M"], a["K"], P(a["w"] or None),
                           P(a["gamma"] or None), a["N"], P(a["y"] or None), None, None, None,
                           P(a["ws"] or None), a["ws_bytes"], None)
    assert st == expect


def test_ffn_and_quant_and_pack_reject_before_launch(lib):
    P = ctypes.c_void_p
    assert lib.bitnet_ffn_gate_up(P(FAKE), 0, 4, 256, P(FAKE), P(FAKE), None, P(FAKE), 256, P(FAKE), None, None,
                                  P(FAKE), 1 << 20, None) == tw.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_quant_act(P(FAKE), 0, 4, 100, P(FAKE), P(FAKE), None, None) == tw.BITNET_ERR_UNSUPPORTED_SHAPE
    assert lib.bitnet_quant_act(None, 0, 4, 128, P(FAKE), P(FAKE), None, None) == tw.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_pack_weights(P(FAKE), 16, 64, 1e-5, P(FAKE), P(FAKE), None, 0, None) == tw.BITNET_ERR_WORKSPACE
    assert lib.bitnet_pack_weights(P(FAKE), 16, 64, -1.0, P(FAKE), P(FAKE), P(FAKE), 4096, None) == \
        tw.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_pack_weights(P(FAKE + 4), 16, 64, 1e-5, P(FAKE), P(FAKE), P(FAKE), 4096, None) == \
        tw.BITNET_ERR_MISALIGNED


def test_norm_entry_points_reject_before_launch(lib):
    """bitnet_rmsnorm_quant / bitnet_linear_norm validate on the host (no GPU needed)."""
    P = 1 << 40
    st = lib.bitnet_rmsnorm_quant
    assert st(None, 0, 4, 256, P, 1e-5, P, P, None, None) == tw.BITNET_ERR_INVALID_ARG
    assert st(P, 0, 4, 256, None, 1e-5, P, P, None, None) == tw.BITNET_ERR_INVALID_ARG
    assert st(P, 0, 4, 256, P, -1.0, P, P, None, None) == tw.BITNET_ERR_INVALID_ARG
    assert st(P, 0, 4, 256, P, float("nan"), P, P, None, None) == tw.BITNET_ERR_INVALID_ARG
    assert st(P, 0, 4, 96, P, 1e-5, P, P, None, None) == tw.BITNET_ERR_UNSUPPORTED_SHAPE
    assert st(P, 0, 4, 8256, P, 1e-5, P, P, None, None) == tw.BITNET_ERR_UNSUPPORTED_SHAPE
    assert st(P + 4, 0, 4, 256, P, 1e-5, P, P, None, None) == tw.BITNET_ERR_MISALIGNED
    assert st(P, 0, 4, 256, P + 8, 1e-5, P, P, None, None) == tw.BITNET_ERR_MISALIGNED
    assert st(P, 7, 4, 256, P, 1e-5, P, P, None, None) == tw.BITNET_ERR_INVALID_ARG
    ln = lib.bitnet_linear_norm
    ws = tw.bitnet_workspace_size(4, 256, 256)
    assert ln(P, 0, 4, 256, None, 1e-5, P, P, 256, P, None, None, None, P, ws, None) == tw.BITNET_ERR_INVALID_ARG
    assert ln(P, 0, 4, 8256, P, 1e-5, P, P, 256, P, None, None, None, P, ws, None) == \
        tw.BITNET_ERR_UNSUPPORTED_SHAPE
    assert ln(P, 0, 4, 256, P + 4, 1e-5, P, P, 256, P, None, None, None, P, ws, None) == tw.BITNET_ERR_MISALIGNED
    fn = lib.bitnet_ffn_gate_up_norm
    assert fn(P, 0, 4, 256, None, 1e-5, P, P, P, P, 256, P, None, None, P, ws, None) == tw.BITNET_ERR_INVALID_ARG


def test_ex_entry_points_reject_before_launch(lib):
    """bitnet_linear_ex / bitnet_ffn_gate_up_ex: bad output dtype, given maxima
    together with normalisation, given and emitted maxima sharing memory, and
    misaligned maxima are rejected on the host."""
    P = 1 << 40
    A = P + (1 << 20)  # a second, disjoint address
    ws = tw.bitnet_workspace_size(4, 256, 256)
    lx = lib.bitnet_linear_ex
    ok_args = dict(x=P, xd=0, xa=None, g=None, eps=1e-5, m=4, k=256, w=P, gam=P, n=256, y=P, yd=0, ya=None)

    def call(**kw):
        a = dict(ok_args, **kw)
        return lx(a["x"], a["xd"], a["xa"], a["g"], a["eps"], a["m"], a["k"], a["w"], a["gam"], a["n"], a["y"],
                  a["yd"], a["ya"], P, ws, None)

    assert call(yd=7) == tw.BITNET_ERR_INVALID_ARG
    assert call(xd=7) == tw.BITNET_ERR_INVALID_ARG
    assert call(xa=A, g=P) == tw.BITNET_ERR_INVALID_ARG
    assert call(xa=A, ya=A + 8) == tw.BITNET_ERR_INVALID_ARG
    assert call(xa=A, ya=A) == tw.BITNET_ERR_INVALID_ARG
    assert call(ya=A + 4) == tw.BITNET_ERR_MISALIGNED
    assert call(xa=A + 4) == tw.BITNET_ERR_MISALIGNED
    assert call(y=None) == tw.BITNET_ERR_INVALID_ARG
    assert call(k=96) == tw.BITNET_ERR_UNSUPPORTED_SHAPE
    fx = lib.bitnet_ffn_gate_up_ex
    assert fx(P, 0, None, None, 1e-5, 4, 256, P, P, P, P, 256, P, 5, None, P, ws, None) == tw.BITNET_ERR_INVALID_ARG
    assert fx(P, 0, A, P, 1e-5, 4, 256, P, P, P, P, 256, P, 0, None, P, ws, None) == tw.BITNET_ERR_INVALID_ARG
    assert fx(P, 0, None, None, 1e-5, 4, 256, P, P, None, P, 256, P, 0, None, P, ws, None) == \
        tw.BITNET_ERR_INVALID_ARG
