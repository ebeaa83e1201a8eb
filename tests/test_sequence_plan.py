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
    size = tw.bitnet_sequence_workspace_size(1, 4, 256)
    assert size >= 4 * 4 + 256 * 8
    assert lib.bitnet_decode_sequence(arr, 1, 4, None, size, None) == tw.BITNET_ERR_WORKSPACE
    assert lib.bitnet_decode_sequence(arr, 1, 4, ws + 8, size, None) == tw.BITNET_ERR_MISALIGNED
    # the workspace may not overlap any operand
    assert lib.bitnet_decode_sequence(arr, 1, 4, BASE + (1 << 20), size, None) == tw.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_decode_sequence(arr, 1, 4, BASE + (2 << 20), size, None) == tw.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_decode_sequence(arr, 0, 4, ws, size, None) == tw.BITNET_ERR_INVALID_ARG
    import torch
    if not torch.cuda.is_available():
        assert lib.bitnet_decode_sequence(arr, 1, 4, ws, size, None) == tw.BITNET_ERR_CUDA


def test_workspace_size():
    one = tw.bitnet_sequence_workspace_size(1, 8, 2560)
    assert one >= 2560 * 8 + 8 * 8
    assert tw.bitnet_sequence_workspace_size(120, 8, 6912) >= 120 * 6912 * 8
    assert tw.bitnet_sequence_workspace_size(2, 8, 2560) > one
    assert tw.bitnet_sequence_workspace_size(1, 9, 2560) > one       # 16 token rows of x_q
    assert tw.bitnet_sequence_workspace_size(1, 64, 8192) >= 64 * 8192
    for bad in ((0, 8, 256), (tw.BITNET_SEQ_MAX_OPS_TOTAL + 1, 8, 256), (1, 0, 256), (1, 65, 256), (1, 8, 32),
                (1, 8, 8256)):
        assert tw.bitnet_sequence_workspace_size(*bad) == 0
    # the documented size: counters (2 per op + 2), tensor maps (2 x 128 bytes per op, 128-byte
    # alignment slack), then per op x_q [K/64][Mp][64] + 512 bytes of scales and row sums
    up = lambda v: (v + 255) // 256 * 256  # noqa: E731
    for n, m, k in ((1, 1, 256), (4, 8, 2560), (120, 8, 6912), (128, 64, 8192), (3, 13, 640)):
        mp = 8 if m <= 8 else 16 if m <= 16 else 32 if m <= 32 else 64
        want = up(4 * (2 + 2 * n)) + up(256 * n + 128) + n * (up(k * mp) + 512)
        assert tw.bitnet_sequence_workspace_size(n, m, k) == want
    # longer lists: one part per launch of at most BITNET_SEQ_MAX_OPS ops, laid out as above
    part = lambda n, k: up(4 * (2 + 2 * n)) + up(256 * n + 128) + n * (up(k * 8) + 512)  # noqa: E731
    cap = tw.BITNET_SEQ_MAX_OPS
    for n in (cap + 1, 180, 2 * cap, tw.BITNET_SEQ_MAX_OPS_TOTAL):
        want = sum(part(min(cap, n - c0), 6912) for c0 in range(0, n, cap))
        assert tw.bitnet_sequence_workspace_size(n, 8, 6912) == want


def test_long_lists_are_validated_before_any_launch():
    """A list longer than one launch is validated as a whole first: an invalid op in its
    second part is refused before the first part is launched (here: before the missing
    GPU is noticed); a valid list without a GPU fails with a CUDA status."""
    lib = tw.load_library()
    n, m = tw.BITNET_SEQ_MAX_OPS + 50, 4
    good = [lin(BASE + (2 * i << 20), 256, 256, BASE + ((2 * i + 1) << 20), BASE + ((1 << 12) + i << 20))
            for i in range(n)]
    size = tw.bitnet_sequence_workspace_size(n, m, 256)
    ws = BASE + (1 << 34)
    bad = list(good)
    bad[tw.BITNET_SEQ_MAX_OPS + 10] = lin(BASE, 256, 256, BASE + 16, BASE + (8 << 30))  # y overlaps its own x
    assert lib.bitnet_decode_sequence(tw._op_array(bad), n, m, ws, size, None) == tw.BITNET_ERR_INVALID_ARG
    over = list(good)
    over[-1] = lin(BASE + (2 * (n - 1) << 20), 256, 256, ws + 4096, BASE + (8 << 30))   # writes the workspace
    assert lib.bitnet_decode_sequence(tw._op_array(over), n, m, ws, size, None) == tw.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_decode_sequence(tw._op_array(good), n, m, ws, size - 256, None) == tw.BITNET_ERR_WORKSPACE
    assert lib.bitnet_decode_sequence(tw._op_array(good), tw.BITNET_SEQ_MAX_OPS_TOTAL + 1, m, ws, size,
                                      None) == tw.BITNET_ERR_INVALID_ARG
    import torch
    if not torch.cuda.is_available():
        assert lib.bitnet_decode_sequence(tw._op_array(good), n, m, ws, size, None) == tw.BITNET_ERR_CUDA


def test_norm_fields_are_validated():
    x, y, w = BASE, BASE + (1 << 20), BASE + (2 << 20)
    good = lin(x, 256, 256, y, w)
    good.norm_g = BASE + (3 << 20)
    good.norm_eps = 1e-5
    assert _status([good], 4) == tw.BITNET_OK
    bad = lin(x, 256, 256, y, w)
    bad.norm_g = BASE + (3 << 20) + 4
    assert _status([bad], 4) == tw.BITNET_ERR_MISALIGNED
    bad.norm_g = BASE + (3 << 20)
    bad.norm_eps = -1.0
    assert _status([bad], 4) == tw.BITNET_ERR_INVALID_ARG
    bad.norm_eps = float("inf")
    assert _status([bad], 4) == tw.BITNET_ERR_INVALID_ARG
    # an output may not overwrite a norm weight (read ahead of every wait)
    other = lin(BASE + (4 << 20), 256, 256, BASE + (3 << 20), BASE + (5 << 20))
    assert _status([good, other], 4) == tw.BITNET_ERR_INVALID_ARG


def test_test_stall_setter():
    assert tw.bitnet_set_sequence_test_stall(3) == -1
    assert tw.bitnet_set_sequence_test_stall(-1) == 3
    # an index of a list longer than one launch is accepted (it names an op of the whole list)
    assert tw.bitnet_set_sequence_test_stall(tw.BITNET_SEQ_MAX_OPS + 5) == -1
    assert tw.bitnet_set_sequence_test_stall(-1) == tw.BITNET_SEQ_MAX_OPS + 5
    with pytest.raises(ValueError):
        tw.bitnet_set_sequence_test_stall(tw.BITNET_SEQ_MAX_OPS_TOTAL)


# ---------------------------------------------------------------- task groups and their order
def rows_per_task(o, m):
    """Packed rows of a task: 128 (a gated FFN: 64 outputs) per 16-row group of each of the 8
    compute warps; two groups per warp when the tokens fit one 8-token tile."""
    rg = 2 if m <= 8 else 1
    return (64 if o.kind == tw.BITNET_OP_FFN_GATE_UP else 128) * rg


def ranges(o, m):
    return ((o.x, o.x + m * o.K * (4 if o.x_dtype == tw.BITNET_DTYPE_F32 else 2)), (o.y, o.y + m * o.N * 4))


def ov(a, b):
    return a[0] < b[1] and b[0] < a[1]


def check_tasks(ops, m, groups):
    """The task groups a launch claims, in order: every op's quant group (a task per token for
    M <= 8, else per 8 tokens) and rows group; dependencies point backwards, include every
    ordering the byte ranges require (transitively), and none is implied by another."""
    n = len(ops)
    assert len(groups) == 2 * n
    pos = {}
    for k, gr in enumerate(groups):
        o = ops[gr["op"]]
        key = (gr["op"], gr["kind"])
        assert key not in pos
        pos[key] = k
        want = (m if m <= 8 else -(-m // 8)) if gr["kind"] == "quant" else -(-o.N // rows_per_task(o, m))
        assert gr["tasks"] == want
        assert all(0 <= d < k for d in gr["deps"])
        assert len(gr["deps"]) <= (9 if gr["kind"] == "rows" else 8)
    # transitive closure of the reported dependencies
    anc = [set() for _ in groups]
    for k, gr in enumerate(groups):
        for d in gr["deps"]:
            anc[k] |= anc[d] | {d}
    # reduced: no reported dependency is an ancestor of another one
    for k, gr in enumerate(groups):
        for d in gr["deps"]:
            assert not any(d in anc[e] for e in gr["deps"] if e != d), (k, d)
    for j in range(n):
        xj, yj = ranges(ops[j], m)
        assert pos[(j, "quant")] in anc[pos[(j, "rows")]]
        for i in range(j):
            xi, yi = ranges(ops[i], m)
            if ov(yi, xj):
                assert pos[(i, "rows")] in anc[pos[(j, "quant")]], ("read after write", i, j)
            if ov(xi, yj):
                assert pos[(i, "quant")] in anc[pos[(j, "rows")]], ("write after read", i, j)
            if ov(yi, yj):
                assert pos[(i, "rows")] in anc[pos[(j, "rows")]], ("write after write", i, j)
    return pos


def random_linear_extension(groups, r):
    """A random order in which the groups could complete, given only their dependencies."""
    left = [len(g["deps"]) for g in groups]
    succ = [[] for _ in groups]
    for k, g in enumerate(groups):
        for d in g["deps"]:
            succ[d].append(k)
    ready = [k for k in range(len(groups)) if left[k] == 0]
    out = []
    while ready:
        k = ready.pop(r.randrange(len(ready)))
        out.append(k)
        for v in succ[k]:
            left[v] -= 1
            if left[v] == 0:
                ready.append(v)
    assert len(out) == len(groups)
    return out


def simulate_groups(ops, m, groups, order, arena_lo, arena_hi):
    """Byte-stamp model of a launch: a quant group reads its op's x, a rows group writes its y."""
    mem = np.zeros(arena_hi - arena_lo, np.int32)
    reads = {}
    for k in order:
        gr = groups[k]
        j = gr["op"]
        (xlo, xhi), (ylo, yhi) = ranges(ops[j], m)
        if gr["kind"] == "quant":
            reads[j] = mem[xlo - arena_lo: xhi - arena_lo].copy()
        else:
            mem[ylo - arena_lo: yhi - arena_lo] = j + 1
    return reads, mem


def test_tasks_of_the_bench_decode_step():
    """30 layers with private outputs at M = 8 on 148 CTAs: every input is fresh except down's
    (h of the same layer), so a down's quant group waits only for its gate/up rows, and rows
    groups wait only for their own quant group.  The order starts the longest chains (gate/up
    -> down) first and leaves the short independent q / o rows for the end."""
    ops = layer_stack(30, 8, shared_outputs=False)
    groups = tw.bitnet_sequence_tasks(ops, 8, 148)
    pos = check_tasks(ops, 8, groups)
    assert [g["op"] % 4 for g in groups[:30]] == [2] * 30 and all(g["kind"] == "quant" for g in groups[:30])
    assert all(g["kind"] == "rows" and g["op"] % 4 in (0, 1) for g in groups[-20:])
    for l in range(30):
        assert pos[(4 * l + 3, "rows")] < pos[(4 * l, "rows")]  # each down before its layer's q
    for l in range(30):
        gu, dn = 4 * l + 2, 4 * l + 3
        assert groups[pos[(dn, "quant")]]["deps"] == [pos[(gu, "rows")]]
        for j in (4 * l, 4 * l + 1, gu, dn):
            assert groups[pos[(j, "rows")]]["deps"] == [pos[(j, "quant")]]
    assert sum(g["tasks"] for g in groups) == 30 * (4 * 8 + 10 + 10 + 54 + 10)  # 256-row tasks at M = 8


def test_tasks_of_a_stack_sharing_its_output_buffers():
    ops = layer_stack(6, 8, shared_outputs=True)
    groups = tw.bitnet_sequence_tasks(ops, 8, 148)
    pos = check_tasks(ops, 8, groups)
    for l in range(1, 6):
        q, gu = 4 * l, 4 * l + 2
        # q overwrites the previous layer's q output: waits for those rows
        assert pos[(q - 4, "rows")] in groups[pos[(q, "rows")]]["deps"]
        # gate/up overwrites h, which the previous down's quant group still reads
        assert pos[(gu + 1 - 4, "quant")] in groups[pos[(gu, "rows")]]["deps"]


def test_too_many_dependencies_are_refused():
    """An op whose output overwrites the inputs of 9 independent earlier readers would wait
    on 9 groups (more than a task records): refused, never run with a wait missing."""
    m, k = 1, 64
    y = BASE
    readers = [lin(y + 128 * i, k, 16, BASE + (1 << 20) + 4096 * i, BASE + (1 << 30) + (1 << 20) * i)
               for i in range(9)]
    writer = lin(BASE + (2 << 20), k, 9 * 32, y, BASE + (1 << 31))
    with pytest.raises(tw.BitnetError) as e:
        tw.bitnet_sequence_tasks(readers + [writer], m, 148)
    assert e.value.status == tw.BITNET_ERR_UNSUPPORTED_SHAPE
    groups = tw.bitnet_sequence_tasks(readers[:8] + [writer], m, 148)  # 8 readers: fine
    check_tasks(readers[:8] + [writer], m, groups)


@pytest.mark.parametrize("seed", range(16))
def test_random_task_orders_preserve_every_read_and_the_final_memory(seed):
    """Random op lists over a shared arena (partial overlaps of every kind): the task groups'
    dependencies cover every required ordering, and ANY order in which the groups could
    complete under those dependencies reads and leaves exactly what list order does."""
    r = random.Random(1000 + seed)
    m = r.choice([1, 8, 13, 64])
    arena = BASE
    size = 16 * 20000
    ops = []
    wbase = BASE + (1 << 34)
    for j in range(r.randint(2, 40)):
        k = 64 * r.randint(1, 8)
        n = r.randint(1, 300)
        f32 = r.random() < 0.3
        xb, yb = m * k * (4 if f32 else 2), m * n * 4
        if xb > size or yb > size:
            continue
        x = arena + 16 * r.randint(0, (size - xb) // 16)
        y = arena + 16 * r.randint(0, (size - yb) // 16)
        if x < y + yb and y < x + xb:
            continue
        w = wbase + j * (1 << 26)
        if r.random() < 0.3:
            ops.append(op(tw.BITNET_OP_FFN_GATE_UP, x, k, n, y, w, w + (1 << 25), w + (1 << 24), w + (3 << 23),
                          f32=f32))
        else:
            ops.append(lin(x, k, n, y, w, w + (1 << 25), f32=f32))
    if not ops:
        return
    try:
        groups = tw.bitnet_sequence_tasks(ops, m, r.choice([1, 7, 148]))
    except tw.BitnetError as e:
        assert e.status == tw.BITNET_ERR_UNSUPPORTED_SHAPE  # an op with more than 8 waits
        return
    check_tasks(ops, m, groups)
    n_ops = len(ops)
    lo, hi = arena, arena + size
    reads_a, mem_a = simulate(ops, m, list(range(n_ops)), lo, hi)
    for _ in range(6):
        order = random_linear_extension(groups, r)
        reads_b, mem_b = simulate_groups(ops, m, groups, order, lo, hi)
        assert np.array_equal(mem_a, mem_b)
        for j in range(n_ops):
            assert np.array_equal(reads_a[j], reads_b[j])
