"""B200-native BitLinear forward (BitNet b1.58, W1.58A8).

Thin Python binding over the C ABI in ``include/bitnet.h`` (library
``libbitnet_b200.so`` built in-tree by ``ternary_weight_fwd_b200.build``).
The functions keep the C names; this module only marshals arguments:
PyTorch tensors are used for device memory and streams, every step of the
computation runs in the library's CUDA kernels.  There is no fallback: if the
library is missing the call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitnet_b200.so")

BITNET_OK = 0
BITNET_ERR_INVALID_ARG = 1
BITNET_ERR_UNSUPPORTED_SHAPE = 2
BITNET_ERR_MISALIGNED = 3
BITNET_ERR_CUDA = 4
BITNET_ERR_TIMEOUT = 5
BITNET_ERR_WORKSPACE = 6

BITNET_DTYPE_BF16 = 0
BITNET_DTYPE_F32 = 1

BITNET_DISPATCH_AUTO = 0
BITNET_DISPATCH_DECODE_FUSED = 1
BITNET_DISPATCH_DECODE = 2
BITNET_DISPATCH_PREFILL = 3

BITNET_OP_LINEAR = 0
BITNET_OP_FFN_GATE_UP = 1
BITNET_SEQ_MAX_OPS = 128         # ops of one launch
BITNET_SEQ_MAX_OPS_TOTAL = 1024  # ops of one bitnet_decode_sequence call (consecutive launches)
BITNET_SEQ_MAX_M = 64

QUANT_EPS = 1e-5

_lib = None


class bitnet_op_t(ctypes.Structure):
    """One op of bitnet_decode_sequence (mirrors the C struct)."""
    _fields_ = [("kind", ctypes.c_int32), ("x_dtype", ctypes.c_int32), ("x", ctypes.c_void_p),
                ("K", ctypes.c_int64), ("N", ctypes.c_int64), ("w0", ctypes.c_void_p),
                ("gamma0", ctypes.c_void_p), ("w1", ctypes.c_void_p), ("gamma1", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("norm_g", ctypes.c_void_p), ("norm_eps", ctypes.c_float)]


class BitnetError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {bitnet_status_string(status)} ({status})")


def load_library(path: str = LIB_PATH):
    """Load and declare the C ABI.  Raises if the library has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing; build it with "
                           "`python -m ternary_weight_fwd_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    P, I64, SZ, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    sig = {
        "bitnet_status_string": ([I], ctypes.c_char_p),
        "bitnet_version": ([], I),
        "bitnet_pack_workspace_size": ([I64, I64], SZ),
        "bitnet_pack_weights": ([P, I64, I64, F, P, P, P, SZ, P], I),
        "bitnet_quant_act": ([P, I, I64, I64, P, P, P, P], I),
        "bitnet_workspace_size": ([I64, I64, I64], SZ),
        "bitnet_linear": ([P, I, I64, I64, P, P, I64, P, P, P, P, P, SZ, P], I),
        "bitnet_ffn_gate_up": ([P, I, I64, I64, P, P, P, P, I64, P, P, P, P, SZ, P], I),
        "bitnet_device_status": ([I, ctypes.POINTER(ctypes.c_int), P], I),
        "bitnet_num_sms": ([], I),
        "bitnet_set_dispatch": ([I], I),
        "bitnet_launch_count": ([], ctypes.c_uint64),
        "bitnet_linear_noalloc": ([P, I, I64, I64, P, P, I64, P, P], I),
        "bitnet_rmsnorm_quant": ([P, I, I64, I64, P, F, P, P, P, P], I),
        "bitnet_linear_norm": ([P, I, I64, I64, P, F, P, P, I64, P, P, P, P, P, SZ, P], I),
        "bitnet_ffn_gate_up_norm": ([P, I, I64, I64, P, F, P, P, P, P, I64, P, P, P, P, SZ, P], I),
        "bitnet_sequence_workspace_size": ([ctypes.c_int32, I64, I64], SZ),
        "bitnet_sequence_plan": ([ctypes.POINTER(bitnet_op_t), ctypes.c_int32, I64,
                                  ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)], I),
        "bitnet_decode_sequence": ([ctypes.POINTER(bitnet_op_t), ctypes.c_int32, I64, P, SZ, P], I),
        "bitnet_sequence_schedule": ([ctypes.POINTER(bitnet_op_t), ctypes.c_int32, I64,
                                      ctypes.POINTER(ctypes.c_int32)], I),
        "bitnet_sequence_tasks": ([ctypes.POINTER(bitnet_op_t), ctypes.c_int32, I64, ctypes.c_int32,
                                   P, P, P, P, P], I),
        "bitnet_set_sequence_test_stall": ([I], I),
        "bitnet_set_wait_limit_ns": ([ctypes.c_uint64], ctypes.c_uint64),
        "bitnet_linear_ex": ([P, I, P, P, F, I64, I64, P, P, I64, P, I, P, P, SZ, P], I),
        "bitnet_ffn_gate_up_ex": ([P, I, P, P, F, I64, I64, P, P, P, P, I64, P, I, P, P, SZ, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(status, where):
    if status != BITNET_OK:
        raise BitnetError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(x):
    if x.dtype == torch.bfloat16:
        return BITNET_DTYPE_BF16
    if x.dtype == torch.float32:
        return BITNET_DTYPE_F32
    raise TypeError(f"activations must be bfloat16 or float32, got {x.dtype}")


def bitnet_status_string(status: int) -> str:
    return load_library().bitnet_status_string(int(status)).decode()


def bitnet_version() -> int:
    return load_library().bitnet_version()


def bitnet_num_sms() -> int:
    return load_library().bitnet_num_sms()


def bitnet_set_dispatch(dispatch: int) -> int:
    prev = load_library().bitnet_set_dispatch(int(dispatch))
    if prev < 0:
        raise ValueError(f"invalid dispatch {dispatch}")
    return prev


def bitnet_launch_count() -> int:
    return load_library().bitnet_launch_count()


def bitnet_pack_workspace_size(n: int, k: int) -> int:
    return load_library().bitnet_pack_workspace_size(n, k)


def bitnet_workspace_size(m: int, n: int, k: int) -> int:
    return load_library().bitnet_workspace_size(m, n, k)


def bitnet_pack_weights(w, eps=QUANT_EPS, *, w_packed=None, gamma=None, workspace=None, stream=None):
    """fp32 latent [N][K] -> (packed uint8 [N][K/4], gamma fp32 [1])."""
    lib = load_library()
    n, k = w.shape
    if w_packed is None:
        w_packed = torch.empty((n, k // 4), dtype=torch.uint8, device=w.device)
    if gamma is None:
        gamma = torch.empty(4, dtype=torch.float32, device=w.device)[:1]
    ws_bytes = lib.bitnet_pack_workspace_size(n, k)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=w.device)
    _check(lib.bitnet_pack_weights(_ptr(w), n, k, float(eps), _ptr(w_packed), _ptr(gamma), _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "bitnet_pack_weights")
    return w_packed, gamma


def bitnet_quant_act(x, *, x_q=None, s=None, rowsum=None, want_rowsum=True, stream=None):
    """[M][K] bf16/fp32 -> (x_q int8 [M][K], s fp32 [M], rowsum int32 [M] or None)."""
    lib = load_library()
    m, k = x.shape
    if x_q is None:
        x_q = torch.empty((m, k), dtype=torch.int8, device=x.device)
    if s is None:
        s = torch.empty(m, dtype=torch.float32, device=x.device)
    if rowsum is None and want_rowsum:
        rowsum = torch.empty(m, dtype=torch.int32, device=x.device)
    _check(lib.bitnet_quant_act(_ptr(x), _dtype_code(x), m, k, _ptr(x_q), _ptr(s), _ptr(rowsum),
                                _stream(stream)), "bitnet_quant_act")
    return x_q, s, rowsum


def _workspace(workspace, m, n, k, device):
    need = load_library().bitnet_workspace_size(m, n, k)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    return workspace


def bitnet_linear(x, w_packed, gamma, *, y=None, x_q_out=None, s_out=None, acc_out=None, workspace=None,
                  stream=None):
    """y [M][N] fp32 = BitLinear(x) with packed ternary weights."""
    lib = load_library()
    m, k = x.shape
    n = w_packed.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    workspace = _workspace(workspace, m, n, k, x.device)
    _check(lib.bitnet_linear(_ptr(x), _dtype_code(x), m, k, _ptr(w_packed), _ptr(gamma), n, _ptr(y),
                             _ptr(x_q_out), _ptr(s_out), _ptr(acc_out), _ptr(workspace), workspace.numel(),
                             _stream(stream)), "bitnet_linear")
    return y


def bitnet_linear_noalloc(x, w_packed, gamma, *, y=None, stream=None):
    """bitnet_linear using the library's fixed device scratch instead of a workspace,
    for callers that cannot allocate at call time.  Only the output may be
    allocated here, and only when `y` is not given; calls sharing the scratch
    must not overlap on the GPU."""
    lib = load_library()
    m, k = x.shape
    n = w_packed.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    _check(lib.bitnet_linear_noalloc(_ptr(x), _dtype_code(x), m, k, _ptr(w_packed), _ptr(gamma), n, _ptr(y),
                                     _stream(stream)), "bitnet_linear_noalloc")
    return y


def bitnet_ffn_gate_up(x, wg_packed, gamma_g, wu_packed, gamma_u, *, h=None, acc_g_out=None, acc_u_out=None,
                       workspace=None, stream=None):
    """h [M][N] fp32 = relu(BitLinear_g(x))^2 * BitLinear_u(x)."""
    lib = load_library()
    m, k = x.shape
    n = wg_packed.shape[0]
    if h is None:
        h = torch.empty((m, n), dtype=torch.float32, device=x.device)
    workspace = _workspace(workspace, m, n, k, x.device)
    _check(lib.bitnet_ffn_gate_up(_ptr(x), _dtype_code(x), m, k, _ptr(wg_packed), _ptr(gamma_g), _ptr(wu_packed),
                                  _ptr(gamma_u), n, _ptr(h), _ptr(acc_g_out), _ptr(acc_u_out), _ptr(workspace),
                                  workspace.numel(), _stream(stream)), "bitnet_ffn_gate_up")
    return h


RMS_EPS = 1e-5


def bitnet_rmsnorm_quant(x, g, eps=RMS_EPS, *, x_q=None, s=None, rowsum=None, want_rowsum=True, stream=None):
    """(x_q int8 [M][K], s fp32 [M], rowsum int32 [M] or None) of RMSNorm(x) with weight g."""
    lib = load_library()
    m, k = x.shape
    if x_q is None:
        x_q = torch.empty((m, k), dtype=torch.int8, device=x.device)
    if s is None:
        s = torch.empty(m, dtype=torch.float32, device=x.device)
    if rowsum is None and want_rowsum:
        rowsum = torch.empty(m, dtype=torch.int32, device=x.device)
    _check(lib.bitnet_rmsnorm_quant(_ptr(x), _dtype_code(x), m, k, _ptr(g), float(eps), _ptr(x_q), _ptr(s),
                                    _ptr(rowsum), _stream(stream)), "bitnet_rmsnorm_quant")
    return x_q, s, rowsum


def bitnet_linear_norm(x, g, w_packed, gamma, eps=RMS_EPS, *, y=None, x_q_out=None, s_out=None, acc_out=None,
                       workspace=None, stream=None):
    """y [M][N] fp32 = BitLinear(RMSNorm(x, g))."""
    lib = load_library()
    m, k = x.shape
    n = w_packed.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    workspace = _workspace(workspace, m, n, k, x.device)
    _check(lib.bitnet_linear_norm(_ptr(x), _dtype_code(x), m, k, _ptr(g), float(eps), _ptr(w_packed), _ptr(gamma), n,
                                  _ptr(y), _ptr(x_q_out), _ptr(s_out), _ptr(acc_out), _ptr(workspace),
                                  workspace.numel(), _stream(stream)), "bitnet_linear_norm")
    return y


def bitnet_ffn_gate_up_norm(x, g, wg_packed, gamma_g, wu_packed, gamma_u, eps=RMS_EPS, *, h=None, acc_g_out=None,
                            acc_u_out=None, workspace=None, stream=None):
    """h [M][N] fp32 = relu(BitLinear_g(RMSNorm(x, g)))^2 * BitLinear_u(RMSNorm(x, g))."""
    lib = load_library()
    m, k = x.shape
    n = wg_packed.shape[0]
    if h is None:
        h = torch.empty((m, n), dtype=torch.float32, device=x.device)
    workspace = _workspace(workspace, m, n, k, x.device)
    _check(lib.bitnet_ffn_gate_up_norm(_ptr(x), _dtype_code(x), m, k, _ptr(g), float(eps), _ptr(wg_packed),
                                       _ptr(gamma_g), _ptr(wu_packed), _ptr(gamma_u), n, _ptr(h), _ptr(acc_g_out),
                                       _ptr(acc_u_out), _ptr(workspace), workspace.numel(), _stream(stream)),
           "bitnet_ffn_gate_up_norm")
    return h


def _out(y, m, n, y_dtype, device):
    if y is None:
        y = torch.empty((m, n), dtype=y_dtype, device=device)
    return y, _dtype_code(y)


def bitnet_linear_ex(x, w_packed, gamma, *, x_amax=None, norm_g=None, eps=RMS_EPS, y=None,
                     y_dtype=torch.float32, y_amax=None, workspace=None, stream=None):
    """y [M][N] (fp32 or bf16) = BitLinear(x), optionally RMS-normalised first
    (norm_g), with the per-token maxima of x given (x_amax [M]) and/or those of
    y emitted into y_amax [M] fp32.  Returns y."""
    lib = load_library()
    m, k = x.shape
    n = w_packed.shape[0]
    y, yc = _out(y, m, n, y_dtype, x.device)
    workspace = _workspace(workspace, m, n, k, x.device)
    _check(lib.bitnet_linear_ex(_ptr(x), _dtype_code(x), _ptr(x_amax), _ptr(norm_g), float(eps), m, k,
                                _ptr(w_packed), _ptr(gamma), n, _ptr(y), yc, _ptr(y_amax), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "bitnet_linear_ex")
    return y


def bitnet_ffn_gate_up_ex(x, wg_packed, gamma_g, wu_packed, gamma_u, *, x_amax=None, norm_g=None, eps=RMS_EPS,
                          h=None, h_dtype=torch.float32, h_amax=None, workspace=None, stream=None):
    """h [M][N] (fp32 or bf16) = relu(BitLinear_g(x))^2 * BitLinear_u(x) with the
    options of bitnet_linear_ex.  Returns h."""
    lib = load_library()
    m, k = x.shape
    n = wg_packed.shape[0]
    h, hc = _out(h, m, n, h_dtype, x.device)
    workspace = _workspace(workspace, m, n, k, x.device)
    _check(lib.bitnet_ffn_gate_up_ex(_ptr(x), _dtype_code(x), _ptr(x_amax), _ptr(norm_g), float(eps), m, k,
                                     _ptr(wg_packed), _ptr(gamma_g), _ptr(wu_packed), _ptr(gamma_u), n, _ptr(h), hc,
                                     _ptr(h_amax), _ptr(workspace), workspace.numel(), _stream(stream)),
           "bitnet_ffn_gate_up_ex")
    return h


def bitnet_device_status(clear=True, stream=None) -> int:
    out = ctypes.c_int(0)
    _check(load_library().bitnet_device_status(1 if clear else 0, ctypes.byref(out), _stream(stream)),
           "bitnet_device_status")
    return out.value


# ---- decode sequences -------------------------------------------------------
def linear_op(x, w_packed, gamma, y, norm_g=None, eps=RMS_EPS):
    """Describe y = BitLinear(x) (of RMSNorm(x) when norm_g is given) as one op of a decode sequence."""
    return bitnet_op_t(BITNET_OP_LINEAR, _dtype_code(x), x.data_ptr(), x.shape[1], w_packed.shape[0],
                       w_packed.data_ptr(), gamma.data_ptr(), None, None, y.data_ptr(),
                       None if norm_g is None else norm_g.data_ptr(), float(eps))


def ffn_gate_up_op(x, wg_packed, gamma_g, wu_packed, gamma_u, h, norm_g=None, eps=RMS_EPS):
    """Describe h = relu(BitLinear_g(x))^2 * BitLinear_u(x) as one op of a decode sequence."""
    return bitnet_op_t(BITNET_OP_FFN_GATE_UP, _dtype_code(x), x.data_ptr(), x.shape[1], wg_packed.shape[0],
                       wg_packed.data_ptr(), gamma_g.data_ptr(), wu_packed.data_ptr(), gamma_u.data_ptr(),
                       h.data_ptr(), None if norm_g is None else norm_g.data_ptr(), float(eps))


def _op_array(ops):
    arr = (bitnet_op_t * max(1, len(ops)))()
    for i, o in enumerate(ops):
        arr[i] = o
    return arr


def bitnet_sequence_workspace_size(n_ops: int, m: int, k_max: int) -> int:
    return load_library().bitnet_sequence_workspace_size(int(n_ops), int(m), int(k_max))


def bitnet_sequence_workspace(device, n_ops=BITNET_SEQ_MAX_OPS, m=BITNET_SEQ_MAX_M, k_max=8192):
    """A workspace for bitnet_decode_sequence (each launch zeroes its counters before use)."""
    return torch.zeros(bitnet_sequence_workspace_size(n_ops, m, k_max), dtype=torch.uint8, device=device)


def bitnet_sequence_plan(ops, m):
    """Host-only: validate `ops` (bitnet_op_t records) for M = m tokens and return
    (wait_x, wait_y), the earlier op each one waits for before reading x / writing y."""
    n = len(ops)
    wx = (ctypes.c_int32 * max(1, n))()
    wy = (ctypes.c_int32 * max(1, n))()
    _check(load_library().bitnet_sequence_plan(_op_array(ops), n, m, wx, wy), "bitnet_sequence_plan")
    return list(wx[:n]), list(wy[:n])


def bitnet_sequence_schedule(ops, m):
    """Host-only: the order (indices into `ops`) in which bitnet_decode_sequence takes them up."""
    n = len(ops)
    order = (ctypes.c_int32 * max(1, n))()
    _check(load_library().bitnet_sequence_schedule(_op_array(ops), n, m, order), "bitnet_sequence_schedule")
    return list(order[:n])


def bitnet_sequence_tasks(ops, m, ctas):
    """Host-only task order of a sequence launch on `ctas` CTAs: list of groups
    dict(op, kind ('quant' | 'rows'), tasks, deps (positions of earlier groups))."""
    import numpy as np
    n = len(ops)
    g_op = np.zeros(2 * n, np.int32)
    g_kind = np.zeros(2 * n, np.int32)
    g_tasks = np.zeros(2 * n, np.int32)
    d_cnt = np.zeros(2 * n, np.int32)
    deps = np.zeros(18 * n, np.int32)
    _check(load_library().bitnet_sequence_tasks(_op_array(ops), n, m, int(ctas), g_op.ctypes.data, g_kind.ctypes.data,
                                                g_tasks.ctypes.data, d_cnt.ctypes.data, deps.ctypes.data),
           "bitnet_sequence_tasks")
    return [dict(op=int(g_op[k]), kind="rows" if g_kind[k] else "quant", tasks=int(g_tasks[k]),
                 deps=[int(d) for d in deps[9 * k:9 * k + d_cnt[k]]]) for k in range(2 * n)]


def bitnet_decode_sequence(ops, m, workspace, stream=None):
    """Run `ops` (bitnet_op_t records over the same m tokens) in one persistent launch per
    BITNET_SEQ_MAX_OPS ops."""
    _check(load_library().bitnet_decode_sequence(_op_array(ops), len(ops), m, _ptr(workspace), workspace.numel(),
                                                 _stream(stream)), "bitnet_decode_sequence")


def bitnet_set_sequence_test_stall(op: int) -> int:
    """Tests only: op (list index) whose weight-row tasks wait for a quantisation task that never
    runs, so the launch ends in a device-side timeout; -1 = off.  Returns the previous value."""
    prev = load_library().bitnet_set_sequence_test_stall(int(op))
    if prev < -1:
        raise ValueError(f"op index out of range: {op}")
    return prev


def bitnet_set_wait_limit_ns(ns: int) -> int:
    """Limit of every bounded device-side wait (0 = default, 2 s).  Returns the previous value."""
    prev = load_library().bitnet_set_wait_limit_ns(int(ns))
    if prev == 0:
        raise RuntimeError("could not set the wait limit")
    return prev
