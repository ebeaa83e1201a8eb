"""Host logic of bitnet_decode_sequence, without a GPU: argument validation and the
hazard analysis that decides which earlier op each op waits for.

The rule checked here is the one that makes a sequence equal to running its ops
one after another: op j must not read x before the latest earlier op that writes
any byte of it has finished (read after write), and must not write y before the
latest earlier op that reads or writes any byte of it has finished (write after
read / write after write).  Pointers are synthetic addresses: planning never
touches memory."""
import random

import numpy as np
import pytest

import ternary_weight_fwd_b200 as tw
from ternary_weight_fwd_b200 import build as tw_build

BASE = 1 << 40


@pytest.fixture(scope="module", autouse=True)
def lib():
    tw_build.build()
    return tw.load_library()


def op(kind, x, k, n, y, w0, g0, w1=None, g1=None, f32=False):
    return tw.bitnet_op_t(kind, tw.BITNET_DTYPE_F32 if f32 else tw.BITNET_DTYPE_BF16, x, k, n, w0, g0, w1, g1, y)


def lin(x, k, n, y, w, g=None, f32=False):
    return op(tw.BITNET_OP_LINEAR, x, k, n, y, w, g if g is not None else w + (n * k // 4 + 255) // 256 * 256,
              f32=f32)


def brute_force(ops, m):
    """Reference hazard analysis written from the rule above."""
    def xr(o):
        return o.x, o.x + m * o.K * (4 if o.x_dtype == tw.BITNET_DTYPE_F32 else 2)

    def yr(o):
        return o.y, o.y + m * o.N * 4

    def ov(a, b):
        return a[0] < b[1] and b[0] < a[1]

    wx, wy = [], []
    for j, oj in enumerate(ops):
        rx = [i for i in range(j) if ov(yr(ops[i]), xr(oj))]
        ry = [i for i in range(j) if ov(yr(ops[i]), yr(oj)) or ov(xr(ops[i]), yr(oj))]
        wx.append(max(rx) if rx else -1)
        wy.append(max(ry) if ry else -1)
    return wx, wy


def layer_stack(layers, m, shared_outputs=True):
    """The decode step of a BitNet layer stack: q, o, gate/up (+ReLU^2), down on h."""
    H, I = 2560, 6912
    addr = [BASE]

    def alloc(nbytes):
        a = addr[0]
        addr[0] += (nbytes + 4095) // 4096 * 4096
        return a

    ops = []
    outs = {k: alloc(m * n * 4) for k, n in (("q", H), ("o", H), ("h", I), ("down", H))}
    for _ in range(layers):
        xs = [alloc(m * H * 2) for _ in range(3)]
        if not shared_outputs:
            outs = {k: alloc(m * n * 4) for k, n in (("q", H), ("o", H), ("h", I), ("down", H))}
        ops.append(lin(xs[0], H, H, outs["q"], alloc(H * H // 4), alloc(16)))
        ops.append(lin(xs[1], H, H, outs["o"], alloc(H * H // 4), alloc(16)))
        ops.append(op(tw.BITNET_OP_FFN_GATE_UP, xs[2], H, I, outs["h"], alloc(I * H // 4), alloc(16),
                      alloc(I * H // 4), alloc(16)))
        ops.append(lin(outs["h"], I, H, outs["down"], alloc(H * I // 4), alloc(16), f32=True))
    return ops


def test_layer_stack_dependencies():
    ops = layer_stack(30, 8)
    wx, wy = tw.bitnet_sequence_plan(ops, 8)
    for l in range(30):
        q, o, gu, dn = 4 * l, 4 * l + 1, 4 * l + 2, 4 * l + 3
        assert wx[q] == wx[o] == wx[gu] == -1          # fresh inputs
        assert wx[dn] == gu                            # down reads h
        if l == 0:
            assert wy[q] == wy[o] == wy[dn] == -1 and wy[gu] == -1
        else:
            assert wy[q] == q - 4 and wy[o] == o - 4   # same output buffers as the previous layer
            assert wy[gu] == gu - 3                    # h is still read by the previous down
            assert wy[dn] == dn - 4
    assert (wx, wy) == brute_force(ops, 8)


def test_private_outputs_have_no_write_hazards():
    ops = layer_stack(4, 3, shared_outputs=False)
    wx, wy = tw.bitnet_sequence_plan(ops, 3)
    assert wy == [-1] * len(ops)
    assert wx == [-1 if j % 4 != 3 else j - 1 for j in range(len(ops))]


@pytest.mark.parametrize("seed", range(12))
def test_random_overlaps_match_brute_force(seed):
    """Random ops over a small arena, so partial overlaps of every kind occur."""
    r = random.Random(seed)
    m = r.choice([1, 2, 8, 13, 64])
    arena = BASE
    ops = []
    wbase = BASE + (1 << 30)  # weights live apart from activations
    for j in range(r.randint(1, 40)):
        k = 64 * r.randint(1, 8)
        n = r.randint(1, 300)
        f32 = r.random() < 0.3
        x = arena + 16 * r.randint(0, 4000)
        y = arena + 16 * r.randint(0, 4000)
        xb = m * k * (4 if f32 else 2)
        if x < y + m * n * 4 and y < x + xb:  # an op may not overwrite its own input
            y = x + xb + 16 * r.randint(0, 64)
        w = wbase + j * (1 << 20)
        ops.append(lin(x, k, n, y, w, w + (1 << 19), f32=f32))
    got = tw.bitnet_sequence_plan(ops, m)
    assert got == brute_force(ops, m)


def simulate(ops, m, order, arena_lo, arena_hi):
    """Run the ops' memory effects in `order` on a byte-stamp model of the activation
    arena: each op records the stamps it reads and stamps the bytes it writes."""
    mem = np.zeros(arena_hi - arena_lo, np.int32)
    reads = {}
    for j in order:
        o = ops[j]
        xb = m * o.K * (4 if o.x_dtype == tw.BITNET_DTYPE_F32 else 2)
        reads[j] = mem[o.x - arena_lo: o.x - arena_lo + xb].copy()
        mem[o.y - arena_lo: o.y - arena_lo + m * o.N * 4] = j + 1
    return reads, mem


def is_topological(ops, m, order):
    pos = {j: k for k, j in enumerate(order)}
    wx, wy = brute_force(ops, m)
    def xr(o):
        return o.x, o.x + m * o.K * (4 if o.x_dtype == tw.BITNET_DTYPE_F32 else 2)
    def yr(o):
        return o.y, o.y + m * o.N * 4
    def ov(a, b):
        return a[0] < b[1] and b[0] < a[1]
    for j in range(len(ops)):
        for i in range(j):
            if ov(yr(ops[i]), xr(ops[j])) or ov(yr(ops[i]), yr(ops[j])) or ov(xr(ops[i]), yr(ops[j])):
                if pos[i] > pos[j]:
                    return False
    return True


def test_schedule_layer_stack_moves_consumers_away_from_producers():
    ops = layer_stack(30, 8)
    order = tw.bitnet_sequence_schedule(ops, 8)
    assert sorted(order) == list(range(len(ops)))
    assert is_topological(ops, 8, order)
    # no down projection runs right after the gate/up whose h it reads, except in the
    # last layer, where no independent op is left to put between them
    for k in range(1, len(order)):
        j, prev = order[k], order[k - 1]
        if j % 4 == 3 and j < len(ops) - 4:
            assert prev != j - 1, (k, j, prev)
    assert order[-2:] == [len(ops) - 2, len(ops) - 1]


@pytest.mark.parametrize("seed", range(12))
def test_schedule_preserves_every_read_and_the_final_memory(seed):
    """Random ops over a small arena: the scheduled order reads and leaves exactly
    what list order does (byte-stamp model), and is a topological order."""
    r = random.Random(100 + seed)
    m = r.choice([1, 2, 8])
    arena = BASE
    size = 16 * 6000
    ops = []
    wbase = BASE + (1 << 30)
    for j in range(r.randint(2, 48)):
        k = 64 * r.randint(1, 4)
        n = r.randint(1, 120)
        f32 = r.random() < 0.3
        xb = m * k * (4 if f32 else 2)
        yb = m * n * 4
        x = arena + 16 * r.randint(0, (size - xb) // 16)
        y = arena + 16 * r.randint(0, (size - yb) // 16)
        if x < y + yb and y < x + xb:
            continue
        w = wbase + j * (1 << 20)
        ops.append(lin(x, k, n, y, w, w + (1 << 19), f32=f32))
    if not ops:
        return
    order = tw.bitnet_sequence_schedule(ops, m)
    assert sorted(order) == list(range(len(ops)))
    assert is_topological(ops, m, order)
    r0, mem0 = simulate(ops, m, range(len(ops)), arena, arena + size)
    r1, mem1 = simulate(ops, m, order, arena, arena + size)
    assert np.array_equal(mem0, mem1)
    for j in range(len(ops)):
        assert np.array_equal(r0[j], r1[j]), j


def _status(ops, m, n=None):
    lib = tw.load_library()
    arr = tw._op_array(ops)
    return lib.bitnet_sequence_plan(arr, len(ops) if n is None else n, m, None, None)


def test_rejections():
    good = lin(BASE, 256, 256, BASE + (1 << 20), BASE + (2 << 20))
    assert _status([good], 4) == tw.BITNET_OK
    assert _status([good], 0) == tw.BITNET_ERR_INVALID_ARG
    assert _status([good], 65) == tw.BITNET_ERR_UNSUPPORTED_SHAPE
    assert _status([good], 4, n=0) == tw.BITNET_ERR_INVALID_ARG
    assert _status([good] * 129, 4) == tw.BITNET_ERR_INVALID_ARG
    assert _status([good] * 128, 4) == tw.BITNET_OK
    # K not a multiple of 64, K above the sequence kernel's limit
    assert _status([lin(BASE, 96, 256, BASE + (1 << 20), BASE + (2 << 20))], 4) == tw.BITNET_ERR_UNSUPPORTED_SHAPE
    assert _status([lin(BASE, 8256, 256, BASE + (1 << 22), BASE + (2 << 22))], 4) == \
        tw.BITNET_ERR_UNSUPPORTED_SHAPE
    assert _status([lin(BASE, 8192, 256, BASE + (1 << 22), BASE + (2 << 22))], 4) == tw.BITNET_OK
    # misaligned pointers
    assert _status([lin(BASE + 8, 256, 256, BASE + (1 << 20), BASE + (2 << 20))], 4) == tw.BITNET_ERR_MISALIGNED
    assert _status([lin(BASE, 256, 256, BASE + (1 << 20) + 4, BASE + (2 << 20))], 4) == tw.BITNET_ERR_MISALIGNED
    # null pointers, bad kind / dtype, FFN without its up projection
    assert _status([lin(0, 256, 256, BASE + (1 << 20), BASE + (2 << 20))], 4) == tw.BITNET_ERR_INVALID_ARG
    bad = lin(BASE, 256, 256, BASE + (1 << 20), BASE + (2 << 20))
    bad.kind = 7
    assert _status([bad], 4) == tw.BITNET_ERR_INVALID_ARG
    bad = lin(BASE, 256, 256, BASE + (1 << 20), BASE + (2 << 20))
    bad.x_dtype = 5
    assert _status([bad], 4) == tw.BITNET_ERR_INVALID_ARG
    ffn = op(tw.BITNET_OP_FFN_GATE_UP, BASE, 256, 256, BASE + (1 << 20), BASE + (2 << 20), BASE + (3 << 20))
    assert _status([ffn], 4) == tw.BITNET_ERR_INVALID_ARG
    # an op overwriting its own input
    assert _status([lin(BASE, 256, 256, BASE + 256, BASE + (2 << 20))], 4) == tw.BITNET_ERR_INVALID_ARG
    # an output overwriting weights or a gamma of any op (they are read ahead of every wait)
    w1 = BASE + (2 << 20)
    ops = [lin(BASE, 256, 256, BASE + (1 << 20), w1, w1 + (1 << 16)),
           lin(BASE + (4 << 20), 256, 256, w1 + 1024, BASE + (3 << 20))]
    assert _status(ops, 4) == tw.BITNET_ERR_INVALID_ARG
    ops[1] = lin(BASE + (4 << 20), 256, 256, w1 + (1 << 16), BASE + (3 << 20))
    assert _status(ops, 4) == tw.BITNET_ERR_INVALID_ARG


def test_run_rejects_before_launch():
    """bitnet_decode_sequence validates like the plan and checks the workspace
    before it looks for a GPU; a valid call without a GPU fails with a CUDA status."""
    lib = tw.load_library()
    good = [lin(BASE, 256, 256, BASE + (1 << 20), BASE + (2 << 20))]
    arr = tw._op_array(good)
    ws = BASE + (8 << 20)
    size = tw.bitnet_sequence_workspace_size()
    assert size >= 4 * (tw.BITNET_SEQ_MAX_OPS + 1)
    assert lib.bitnet_decode_sequence(arr, 1, 4, None, size, None) == tw.BITNET_ERR_WORKSPACE
    assert lib.bitnet_decode_sequence(arr, 1, 4, ws, size - 1, None) == tw.BITNET_ERR_WORKSPACE
    assert lib.bitnet_decode_sequence(arr, 1, 4, ws + 8, size, None) == tw.BITNET_ERR_MISALIGNED
    # the workspace may not overlap any operand
    assert lib.bitnet_decode_sequence(arr, 1, 4, BASE + (1 << 20), size, None) == tw.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_decode_sequence(arr, 1, 4, BASE + (2 << 20), size, None) == tw.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_decode_sequence(arr, 0, 4, ws, size, None) == tw.BITNET_ERR_INVALID_ARG
    import torch
    if not torch.cuda.is_available():
        assert lib.bitnet_decode_sequence(arr, 1, 4, ws, size, None) == tw.BITNET_ERR_CUDA


def test_cluster_size_setter():
    prev = tw.bitnet_set_sequence_cluster(8)
    try:
        assert tw.bitnet_set_sequence_cluster(4) == 8
        for bad in (0, 1, 2, 3, 16):
            with pytest.raises(ValueError):
                tw.bitnet_set_sequence_cluster(bad)
        assert tw.bitnet_set_sequence_cluster(4) == 4
    finally:
        tw.bitnet_set_sequence_cluster(prev)


# ---------------------------------------------------------------- partitions and row slices
def producers(ops, m):
    wx, wy = brute_force(ops, m)
    return [{w for w in (wx[j], wy[j]) if w >= 0} for j in range(len(ops))]


def check_layout(ops, m, L, clusters):
    n = len(ops)
    order, part_of, slices = L["order"], L["part_of"], L["slices"]
    assert sorted(order) == list(range(n)), "order is a permutation of the ops"
    assert sum(L["part_clusters"]) == clusters and min(L["part_clusters"]) >= 1
    assert sum(slices) <= 320 and min(slices) >= 1  # kernel ops per launch
    pos = {i: k for k, i in enumerate(order)}
    for j, pre in enumerate(producers(ops, m)):
        for i in pre:
            # every earlier conflicting op runs first, in the same partition
            assert pos[i] < pos[j] and part_of[pos[i]] == part_of[pos[j]]
    # partitions never share memory: ops of different partitions never conflict
    wx, wy = brute_force([ops[i] for i in order], m)
    for j in range(n):
        for w in (wx[j], wy[j]):
            assert w < 0 or part_of[w] == part_of[j]


@pytest.mark.parametrize("forced", [0, 1, 2, 3, 4, 8])
@pytest.mark.parametrize("shared", [True, False], ids=["shared_outputs", "private_outputs"])
def test_layout_of_the_layer_stack(forced, shared):
    ops = layer_stack(30, 8, shared_outputs=shared)
    prev = tw.bitnet_set_sequence_partitions(forced)
    try:
        try:
            L = tw.bitnet_sequence_layout(ops, 8, 4, 33)
        except tw.BitnetError as e:
            # more partitions than slices allow (every op cut to fit 4 clusters): refused, never wrong
            assert forced >= 6 and e.status == tw.BITNET_ERR_UNSUPPORTED_SHAPE
            return
    finally:
        tw.bitnet_set_sequence_partitions(prev)
    check_layout(ops, 8, L, 33)
    n_parts = len(L["part_clusters"])
    if shared:
        assert n_parts <= 3  # the gate/up -> down chain, the q chain and the o chain
    if forced:
        assert n_parts == min(forced, 3 if shared else 120)
    # a gate/up op and the down op that reads its h share a partition
    for l in range(30):
        k_gu, k_dn = L["order"].index(4 * l + 2), L["order"].index(4 * l + 3)
        assert L["part_of"][k_gu] == L["part_of"][k_dn] and k_gu < k_dn


def test_layout_private_outputs_runs_layers_side_by_side():
    ops = layer_stack(30, 8, shared_outputs=False)
    L = tw.bitnet_sequence_layout(ops, 8, 4, 33)
    assert len(L["part_clusters"]) >= 2
    # big projections are cut into row slices on the smaller partitions
    k_gu = L["order"].index(2)
    assert L["slices"][k_gu] >= 2


def test_layout_cuts_one_huge_projection_into_slices():
    m, k, n = 8, 256, 60000
    ops = [op(tw.BITNET_OP_FFN_GATE_UP, BASE, k, n, BASE + (1 << 30), BASE + (2 << 30), BASE + (3 << 30),
              BASE + (4 << 30), BASE + (5 << 30))]
    L = tw.bitnet_sequence_layout(ops, m, 4, 33)
    assert L["part_clusters"] == [33] and L["slices"][0] >= 2
    # rows per cluster of each slice within 8 row groups per warp (1024 rows of both matrices)
    assert 2 * ((-(-(n // L["slices"][0] + 1) // 33) + 15) // 16) <= 64


def test_partition_setter():
    assert tw.bitnet_set_sequence_partitions(2) == 0
    assert tw.bitnet_set_sequence_partitions(0) == 2
    with pytest.raises(ValueError):
        tw.bitnet_set_sequence_partitions(9)
    assert tw.bitnet_set_sequence_partitions(0) == 0


def test_layout_auto_choice_for_the_bench_decode_step():
    """The plan the bench times (30 layers, per-layer outputs, M = 8, 33 clusters of 4): eight
    partitions of ~4 layers, q / o whole, gate/up in 4-5 row slices, down in 2, 266 kernel ops.
    Measured on B200: 3, 4, 5, 6, 7, 8 partitions -> 434, 432, 404, 385, 405, 368 us per step."""
    ops = layer_stack(30, 8, shared_outputs=False)
    L = tw.bitnet_sequence_layout(ops, 8, 4, 33)
    assert L["part_clusters"] == [5, 4, 4, 4, 4, 4, 4, 4]
    assert sum(L["slices"]) == 266
    kinds = {}
    for k, i in enumerate(L["order"]):
        kinds.setdefault(i % 4, set()).add(L["slices"][k])
    assert kinds[0] == {1} and kinds[1] == {1} and kinds[2] <= {4, 5} and kinds[3] == {2}


@pytest.mark.parametrize("seed", range(12))
def test_random_layouts_keep_every_hazard_inside_a_partition(seed):
    """Random op lists over a shared arena (partial overlaps of every kind) and random
    large projections: whatever partitions and row slices the planner picks, every op
    runs after, and in the same partition as, every earlier op it conflicts with, and
    the execution order leaves every read and the final memory as list order does."""
    r = random.Random(1000 + seed)
    m = r.choice([1, 8, 13, 64])
    arena = BASE
    ops = []
    wbase = BASE + (1 << 34)
    for j in range(r.randint(2, 60)):
        k = 64 * r.randint(1, 40)
        n = r.choice([r.randint(1, 300), r.randint(2000, 9000)])
        f32 = r.random() < 0.3
        x = arena + 16 * r.randint(0, 200000)
        y = arena + 16 * r.randint(0, 200000)
        xb = m * k * (4 if f32 else 2)
        if x < y + m * n * 4 and y < x + xb:
            y = x + xb + 16 * r.randint(0, 64)
        w = wbase + j * (1 << 26)
        if r.random() < 0.3:
            ops.append(op(tw.BITNET_OP_FFN_GATE_UP, x, k, n, y, w, w + (1 << 25), w + (1 << 24), w + (3 << 23),
                          f32=f32))
        else:
            ops.append(lin(x, k, n, y, w, w + (1 << 25), f32=f32))
    prev = tw.bitnet_set_sequence_partitions(r.choice([0, 0, 2, 4, 8]))
    try:
        L = tw.bitnet_sequence_layout(ops, m, r.choice([4, 8]), r.choice([16, 33]))
    except tw.BitnetError as e:
        assert e.status == tw.BITNET_ERR_UNSUPPORTED_SHAPE  # more row slices than one launch holds
        return
    finally:
        tw.bitnet_set_sequence_partitions(prev)
    n_ops = len(ops)
    assert sorted(L["order"]) == list(range(n_ops))
    pos = {i: k for k, i in enumerate(L["order"])}
    for j, pre in enumerate(producers(ops, m)):
        for i in pre:
            assert pos[i] < pos[j] and L["part_of"][pos[i]] == L["part_of"][pos[j]]
    lo = arena
    hi = max(max(o.x + m * o.K * 4, o.y + m * o.N * 4) for o in ops) + 16
    reads_a, mem_a = simulate(ops, m, list(range(n_ops)), lo, hi)
    reads_b, mem_b = simulate(ops, m, L["order"], lo, hi)
    assert np.array_equal(mem_a, mem_b)
    for j in range(n_ops):
        assert np.array_equal(reads_a[j], reads_b[j])
