"""Pins of the oracle's bf16 rounding and ring collectives (CPU only).

What fixes the expected values: the pages' N=4 AllGather step tables and before/after examples
(tests/golden), the definition of round-to-nearest-even, IEEE binary32 arithmetic done element by
element, the AllGather/ReduceScatter transposition identity, and torch's own bf16 cast.
"""
import itertools

import numpy as np
import pytest
import torch

from golden_io import sections
from oracle import collectives as C
from oracle.bf16 import bf16_bits_to_f32, f32_to_bf16_bits


# ------------------------------------------------------------------------------------ bf16
@pytest.mark.parametrize("value,bits", [
    (1.0, 0x3F80), (-2.5, 0xC020), (0.0, 0x0000), (-0.0, 0x8000),
    (1.0 + 2.0 ** -8, 0x3F80),                  # exact tie, kept part even -> stays
    (1.0 + 3 * 2.0 ** -8, 0x3F82),              # exact tie, kept part odd -> rounds up to even
    (1.0 + 2.0 ** -8 + 2.0 ** -20, 0x3F81),     # just above the tie -> up
    (1.0 + 2.0 ** -8 - 2.0 ** -20, 0x3F80),     # just below the tie -> down
    (float(np.finfo(np.float32).max), 0x7F80),  # overflows to +inf
    (float("inf"), 0x7F80), (float("-inf"), 0xFF80),
])
def test_bf16_rounding_hand_values(value, bits):
    assert int(f32_to_bf16_bits(np.float32(value)).reshape(-1)[0]) == bits


def test_bf16_nan_stays_nan():
    out = f32_to_bf16_bits(np.array([np.nan], dtype=np.float32))
    assert np.isnan(bf16_bits_to_f32(out))[0]


def test_bf16_rounding_matches_torch_cast():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(200_000, generator=g) * torch.exp(torch.randn(200_000, generator=g) * 8)
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(f32_to_bf16_bits(x.numpy()), ref)


# ------------------------------------------------------------------------------------ ring order
@pytest.mark.parametrize("t", range(1, 9))
def test_ring_rs_order_follows_send_right_ring(t):
    # Device i sends to i+1, accumulating at every step, and device r ends with chunk r: chunk c's
    # copies are therefore added starting from shard c+1 and ending with shard c itself.
    prov = C.ring_sum_provenance(t)
    for c in range(t):
        assert prov[c] == [(c + k) % t for k in range(1, t + 1)]


def test_reduce_scatter_example_placement():
    # Device d's chunk c is 2**(4d + c): every sum is exact and each bit names its origin.
    ex = sections("collective_examples_n4.txt")["reduce_scatter"]
    t = 4
    bufs = [np.array([2.0 ** (4 * d + c) for c in range(t)], dtype=np.float32).reshape(t, 1) for d in range(t)]
    out = C.reduce_scatter(bufs, axis=0)
    for dev, expr in ex:
        terms = expr.split("+")
        expect = sum(2.0 ** (4 * (ord(term[0]) - ord("a")) + int(term[1:])) for term in terms)
        assert float(out[int(dev)][0, 0]) == expect


def test_all_to_all_example():
    ex = sections("collective_examples_n4.txt")["all_to_all"]
    t = 4
    names = [[f"{chr(ord('A') + d)}{c}" for c in range(t)] for d in range(t)]
    bufs = [np.array(n, dtype=object).reshape(t, 1) for n in names]
    out = C.all_to_all(bufs, split_axis=0, concat_axis=0)
    for dev, expr in ex:
        assert list(out[int(dev)][:, 0]) == expr.split(",")


def _parse_table(rows):
    return {int(k): [list(cell.strip()) for cell in v.split("|")] for k, v in rows}


@pytest.mark.parametrize("kind", ["unidirectional", "bidirectional"])
def test_all_gather_step_tables(kind):
    table = _parse_table(sections("ring_allgather_n4.txt")[kind])
    steps, final = C.all_gather_steps(list("ABCD"), bidirectional=(kind == "bidirectional"))
    last = max(table)
    assert len(steps) == last
    assert table[0] == [[x] for x in "ABCD"]
    for s in range(1, last):
        assert steps[s - 1] == table[s], f"step {s}"
    assert final == table[last]
    # and the final holdings are the same set as the gathered buffer (arrival order aside)
    for i in range(4):
        assert sorted(steps[-1][i]) == table[last][i]


@pytest.mark.parametrize("t", [1, 2, 3, 4, 5, 8])
def test_all_gather_every_shard_once(t):
    labels = [str(i) for i in range(t)]
    for bidir in (False, True):
        steps, final = C.all_gather_steps(labels, bidirectional=bidir)
        assert len(steps) == ((t // 2) if bidir else (t - 1))
        assert all(f == labels for f in final)


# ------------------------------------------------------------------------------------ numerics
def _elementwise_ring_sum(bufs32, t, axis):
    """Brute force: per element, add the shards' copies one binary32 add at a time in ring order."""
    rows, cols = bufs32[0].shape
    outs = []
    for c in range(t):
        if axis == 0:
            rr, cc = range(c * rows // t, (c + 1) * rows // t), range(cols)
        else:
            rr, cc = range(rows), range(c * cols // t, (c + 1) * cols // t)
        o = np.empty((len(rr), len(cc)), dtype=np.float32)
        for a, r in enumerate(rr):
            for b, col in enumerate(cc):
                acc = np.float32(bufs32[(c + 1) % t][r, col])
                for k in range(2, t + 1):
                    acc = np.float32(acc + np.float32(bufs32[(c + k) % t][r, col]))
                o[a, b] = acc
        outs.append(o)
    return outs


@pytest.mark.parametrize("t,axis", [(1, 0), (2, 0), (3, 1), (4, 0), (4, 1), (8, 0)])
def test_reduce_scatter_brute_force_f32(t, axis):
    g = np.random.default_rng(t * 10 + axis)
    bufs = [g.standard_normal((24, 24)).astype(np.float32) * 1e3 for _ in range(t)]
    got = C.reduce_scatter(bufs, axis=axis)
    ref = _elementwise_ring_sum(bufs, t, axis)
    for a, b in zip(got, ref):
        assert a.dtype == np.float32 and np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_reduce_scatter_order_is_visible_in_fp32():
    # (1e8 + 1) - 1e8 differs from 1e8 + (1 - 1e8) in binary32: the order is not a no-op.
    t = 3
    vals = [np.float32(1.0), np.float32(1e8), np.float32(-1e8)]   # shards 0, 1, 2
    bufs = [np.full((3, 1), v, dtype=np.float32) for v in vals]
    out = C.reduce_scatter(bufs, axis=0)
    # chunk 0: (U1 + U2) + U0 = 0 + 1 = 1; chunk 1: (U2 + U0) + U1 = (-1e8 + 1) + 1e8 = 0 in fp32
    assert float(out[0][0, 0]) == 1.0
    assert float(out[1][0, 0]) == 0.0


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_reduce_scatter_close_to_exact_sum(t):
    g = np.random.default_rng(100 + t)
    bufs = [g.uniform(-1, 1, (16, 8)).astype(np.float32) for _ in range(t)]
    got = np.concatenate(C.reduce_scatter(bufs, axis=0), axis=0).astype(np.float64)
    exact = sum(b.astype(np.float64) for b in bufs)
    # t-1 binary32 adds of values below t in magnitude
    assert np.max(np.abs(got - exact)) <= (t - 1) * t * 2.0 ** -24 + 1e-30


def test_reduce_scatter_bf16_rounds_once_at_the_end():
    g = np.random.default_rng(7)
    t = 4
    f = [g.standard_normal((8, 8)).astype(np.float32) for _ in range(t)]
    bits = [f32_to_bf16_bits(x) for x in f]
    got = C.reduce_scatter(bits, axis=0, dtype="bf16")
    widened = [bf16_bits_to_f32(b) for b in bits]
    ref = [f32_to_bf16_bits(o) for o in _elementwise_ring_sum(widened, t, 0)]
    for a, b in zip(got, ref):
        assert a.dtype == np.uint16 and np.array_equal(a, b)


@pytest.mark.parametrize("t,axis", [(2, 0), (4, 1), (3, 0)])
def test_all_gather_concatenates_in_shard_order(t, axis):
    g = np.random.default_rng(t)
    shards = [g.standard_normal((2, 3)).astype(np.float32) for _ in range(t)]
    out = C.all_gather(shards, axis=axis)
    ref = np.concatenate(shards, axis=axis)
    assert all(np.array_equal(o, ref) for o in out)


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_all_reduce_is_rs_then_ag_and_replicas_agree(t):
    g = np.random.default_rng(200 + t)
    bufs = [g.standard_normal((8, 4)).astype(np.float32) for _ in range(t)]
    ar = C.all_reduce(bufs)
    rs = np.concatenate(C.reduce_scatter(bufs, axis=0), axis=0)
    for o in ar:
        assert np.array_equal(o.view(np.uint32), ar[0].view(np.uint32))
        assert np.array_equal(o.view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("t,axis", [(2, 0), (4, 0), (4, 1), (3, 1)])
def test_allgather_reducescatter_transpose_identity(t, axis):
    # <AG x, y> = <x, RS y>: AllGather = broadcast (x) I and ReduceScatter = reduce (x) I are transposes.
    # Small integers keep every sum exact in fp64.
    g = np.random.default_rng(300 + t + axis)
    rows, cols = 4 * t, 2 * t
    xs = [g.integers(-9, 10, (rows // t, cols) if axis == 0 else (rows, cols // t)).astype(np.float64) for _ in range(t)]
    ys = [g.integers(-9, 10, (rows, cols)).astype(np.float64) for _ in range(t)]
    ag = C.all_gather(xs, axis=axis)
    rs = C.reduce_scatter_f64(ys, axis=axis)
    lhs = sum(float(np.sum(a * y)) for a, y in zip(ag, ys))
    rhs = sum(float(np.sum(x * r)) for x, r in zip(xs, rs))
    assert lhs == rhs


def test_reduce_scatter_axis1_is_axis0_on_the_transpose():
    g = np.random.default_rng(11)
    t = 4
    bufs = [g.standard_normal((6, 8)).astype(np.float32) for _ in range(t)]
    a1 = C.reduce_scatter(bufs, axis=1)
    a0 = C.reduce_scatter([b.T.copy() for b in bufs], axis=0)
    for x, y in zip(a1, a0):
        assert np.array_equal(x.T.view(np.uint32), y.view(np.uint32))


def test_t1_is_identity():
    x = np.arange(12, dtype=np.float32).reshape(3, 4)
    assert np.array_equal(C.reduce_scatter([x])[0], x)
    assert np.array_equal(C.all_gather([x])[0], x)
    assert np.array_equal(C.all_reduce([x])[0], x)


def test_indivisible_split_is_rejected():
    with pytest.raises(ValueError):
        C.reduce_scatter([np.zeros((3, 2), np.float32)] * 2, axis=0)


@pytest.mark.parametrize("t", [2, 3, 4])
def test_every_chunk_gets_every_shard_exactly_once(t):
    prov = C.ring_sum_provenance(t)
    for c, order in enumerate(prov):
        assert sorted(order) == list(range(t)) and order[-1] == c
    assert list(itertools.chain.from_iterable(prov)).count(0) == t


# ------------------------------------------------------------------------------------ per-hop bf16 mode
def test_per_hop_bf16_hand_example():
    # t = 3, chunk 0 is summed in the ring order U[1], U[2], U[0]. With U[1] = 1 and U[2] = U[0] = 2^-8:
    #   rounding once at the end: 1 + 2^-8 + 2^-8 = 1 + 2^-7, exactly a bf16 value (0x3F81);
    #   rounding after every hop: 1 + 2^-8 is a tie between 1 and 1 + 2^-7 and goes to the even 1
    #   (0x3F80), and so does the second hop.
    one, small = 0x3F80, 0x3B80          # bf16 bits of 1.0 and 2^-8
    assert float(bf16_bits_to_f32(np.uint16(small))) == 2.0 ** -8
    bufs = [np.array([[v], [0], [0]], dtype=np.uint16) for v in (small, one, small)]
    end = C.reduce_scatter(bufs, axis=0, dtype="bf16")
    hop = C.reduce_scatter(bufs, axis=0, dtype="bf16", rounding="hop")
    assert int(end[0][0, 0]) == 0x3F81
    assert int(hop[0][0, 0]) == 0x3F80


@pytest.mark.parametrize("t", [2, 3, 4, 8])
def test_per_hop_bf16_equals_sequential_bf16_adds(t):
    # A ring whose links carry bf16 adds one bf16 value at a time and keeps a bf16 partial: exactly
    # torch's bf16 tensor addition (binary32 add, round to nearest-even) applied in the ring order.
    g = torch.Generator().manual_seed(40 + t)
    xs = [torch.randn(t * 16, 24, generator=g).mul(torch.exp(torch.randn(1, generator=g))).to(torch.bfloat16)
          for _ in range(t)]
    bits = [x.view(torch.int16).numpy().view(np.uint16) for x in xs]
    hop = C.reduce_scatter(bits, axis=0, dtype="bf16", rounding="hop")
    rows = 16
    for c in range(t):
        acc = xs[(c + 1) % t][c * rows:(c + 1) * rows]
        for k in range(2, t + 1):
            acc = acc + xs[(c + k) % t][c * rows:(c + 1) * rows]
        ref = acc.view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(hop[c], ref), c
    # and the default mode differs somewhere on this data (a single rounding at the end)
    if t >= 3:
        end = C.reduce_scatter(bits, axis=0, dtype="bf16")
        assert any(not np.array_equal(a, b) for a, b in zip(hop, end))


def test_per_hop_mode_is_bf16_only():
    with pytest.raises(ValueError):
        C.reduce_scatter([np.zeros((2, 2), np.float32)] * 2, dtype="f32", rounding="hop")


@pytest.mark.parametrize("t,axis", [(2, 1), (3, 1), (4, 0), (4, 1)])
def test_all_reduce_along_either_axis_brute_force(t, axis):
    # AllReduce = ReduceScatter + AllGather along one axis: element (r, c) of every replica is the
    # ring sum of the chunk that holds it (rows for axis 0, columns for axis 1), added one binary32
    # add at a time starting at shard chunk+1 -- checked element by element by brute force.
    g = np.random.default_rng(60 + 10 * t + axis)
    rows, cols = 3 * t, 2 * t
    bufs = [(g.standard_normal((rows, cols)) * np.exp(g.standard_normal((rows, cols)) * 3)).astype(np.float32)
            for _ in range(t)]
    got = C.all_reduce(bufs, axis=axis)
    ref = np.concatenate(_elementwise_ring_sum(bufs, t, axis), axis=axis)
    for r in range(t):
        assert np.array_equal(got[r].view(np.uint32), ref.view(np.uint32))
    # the two axes order the adds differently (visible in binary32 on this data)
    if t >= 3:
        other = C.all_reduce(bufs, axis=1 - axis)
        assert not np.array_equal(got[0].view(np.uint32), other[0].view(np.uint32))
