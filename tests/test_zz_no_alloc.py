"""bitnet_linear_noalloc: the entry point for callers that cannot allocate device
memory when they call (an engine that has reserved all free HBM for its own
pool, a plugin host that forbids allocation after start-up, a latency-critical
loop that cannot afford an allocation's implicit synchronisation).  It uses the
library's fixed device scratch instead of a caller workspace.

Checked through the C ABI against bitnet_linear (which takes a caller
workspace) on the same inputs, twice in a row, for a decode-sized call
(quantiser kernel + decode kernel, both using the scratch) and a prefill-sized
call (quantiser kernel + tcgen05 kernel); shapes whose scratch exceeds the
fixed size are refused before launch.  This file sorts last so that a run that
stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import ternary_weight_fwd_b200 as tw
from gpu_util import DEV, assert_rel_close, make_weights, make_x

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, xd, W, y, m, k, n):
    P = ctypes.c_void_p
    code = tw.BITNET_DTYPE_BF16 if xd.dtype == torch.bfloat16 else tw.BITNET_DTYPE_F32
    return lib.bitnet_linear_noalloc(P(xd.data_ptr()), code, m, k, P(W["p"].data_ptr()), P(W["g"].data_ptr()),
                                     n, P(y.data_ptr()), P(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("m,k,n,dispatch", [
    (8, 2560, 2560, tw.BITNET_DISPATCH_DECODE),   # decode kernel reading x_q from the scratch
    (256, 2560, 512, tw.BITNET_DISPATCH_AUTO),    # tcgen05 kernel reading x_q from the scratch
])
def test_noalloc_matches_workspace_entry_point(m, k, n, dispatch):
    lib = tw.load_library()
    prev = tw.bitnet_set_dispatch(dispatch)
    try:
        W = make_weights(n, k, 2000 + m)
        xd, _ = make_x(m, k, 2100 + m, "student_t_rows")
        ref = tw.bitnet_linear(xd, W["p"], W["g"]).cpu().numpy()
        for _ in range(2):
            y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
            assert _call_noalloc(lib, xd, W, y, m, k, n) == tw.BITNET_OK
            torch.cuda.synchronize()
            got = y.cpu().numpy()
            assert_rel_close(got, ref)
            assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    finally:
        tw.bitnet_set_dispatch(prev)
    assert tw.bitnet_device_status() == 0


def test_noalloc_refuses_oversized_scratch():
    lib = tw.load_library()
    m, k, n = 4096, 6912, 64     # x_q alone is 27 MiB > 8 MiB of fixed scratch
    W = make_weights(n, k, 2200)
    xd = torch.zeros((m, k), dtype=torch.bfloat16, device=DEV)
    y = torch.zeros((m, n), dtype=torch.float32, device=DEV)
    before = tw.bitnet_launch_count()
    assert _call_noalloc(lib, xd, W, y, m, k, n) == tw.BITNET_ERR_WORKSPACE
    assert tw.bitnet_launch_count() == before
