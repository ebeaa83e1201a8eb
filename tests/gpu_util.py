"""Helpers for the GPU parity tests: upload seeded inputs, compare against the oracle."""
import numpy as np
import torch

import oracle
import ternary_weight_fwd_b200 as tw
import synth

DEV = "cuda"
REL_TOL = 1e-6  # dequantised outputs: |y - y_ref| <= 1e-6 |y_ref|; y_ref == 0 -> y == 0


def bf16_to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def f32_to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def make_weights(n, k, seed):
    """Latent weights packed by both sides; returns oracle and device results."""
    w = synth.latent_weights(n, k, seed)
    p_ref, g_ref, w_q = oracle.pack_weights(w)
    p, g = tw.bitnet_pack_weights(f32_to_dev(w))
    torch.cuda.synchronize()
    return dict(w=w, w_q=w_q, p_ref=p_ref, g_ref=g_ref, p=p, g=g)


def make_x(m, k, seed, kind="normal", dtype="bf16"):
    """Returns (device tensor, fp32 values the oracle sees)."""
    if dtype == "bf16":
        bits = synth.activations(m, k, seed, kind)
        return bf16_to_dev(bits), synth.bf16_bits_to_f32(bits)
    x = synth.activations_f32(m, k, seed)
    return f32_to_dev(x), x


def assert_rel_close(y_gpu, y_ref, rel=REL_TOL):
    y = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == y_ref.shape
    zero = y_ref == 0
    assert np.all(y[zero] == 0), "nonzero where the oracle gives 0"
    nz = ~zero
    if nz.any():
        err = np.abs(y[nz] - y_ref[nz]) / np.abs(y_ref[nz])
        worst = float(err.max())
        assert worst <= rel, f"max relative error {worst:.3e} > {rel:.1e}"


def sample_rows(m, count, seed):
    """Row indices for spot checks: the first and last row of every 128-row tile, one random
    row inside every tile, plus random rows up to `count`."""
    r = np.random.default_rng(seed)
    fixed = [0, 1, m - 1, m // 2]
    for t in range(0, m, 128):
        fixed += [t, min(t + 127, m - 1), int(r.integers(t, min(t + 128, m)))]
    rows = set(i for i in fixed if 0 <= i < m)
    while len(rows) < min(count, m):
        rows.add(int(r.integers(0, m)))
    return np.array(sorted(rows), dtype=np.int64)
