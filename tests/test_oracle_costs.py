"""Pins of the oracle's closed-form sizes and costs against the numbers the pages print (CPU only)."""
import pytest

from golden_io import numbers
from oracle import costs

P = numbers()
MiB, GiB = costs.MiB, costs.GiB


def test_memory_example():
    # int8[128, 2048], A[I_XY, J] on {X:2, Y:8, Z:2}: replicated over Z
    mesh = {"X": 2, "Y": 8, "Z": 2}
    split = (("X", "Y"), ())
    assert costs.local_shape((128, 2048), split, mesh) == (P["memory.local_rows"], 2048)
    assert costs.per_device_bytes((128, 2048), split, mesh, 1) == P["memory.local_bytes"]
    assert costs.total_bytes((128, 2048), split, mesh, 1) == P["memory.total_bytes"] == 512 * 1024


def test_mesh_axis_used_twice_is_illegal():
    with pytest.raises(ValueError):
        costs.local_shape((8, 8), (("X",), ("X",)), {"X": 2})


def test_replication_ratio_problem1():
    # A[I_X, J, K, ...] on {X:4, Y:8, Z:2}: replicated over Y and Z
    assert costs.replication_ratio((("X",), (), ()), {"X": 4, "Y": 8, "Z": 2}) == 16


def test_case3_roofline_thresholds():
    C, W = P["roofline.flops"], P["roofline.ici_bw"]
    assert int(costs.case3_compute_bound_D(4, C, W)) == P["roofline.case3_D_N4"]
    assert int(costs.case3_compute_bound_D(2, C, W)) == P["roofline.case3_D_N2"]


def test_ring_bytes_per_rank():
    assert costs.ring_bytes_per_rank("all_gather", 8, 4) == 6
    assert costs.ring_bytes_per_rank("reduce_scatter", 8, 4) == 6
    assert costs.ring_bytes_per_rank("all_reduce", 8, 4) == 12
    assert costs.ring_bytes_per_rank("all_reduce", 8, 1) == 0


def test_llama70b_comm_example():
    c = costs.tp_layer_comm(b=1, s=4096, h=8192, t=8, layers=80)
    assert c["M"] == P["comm70b.M_MiB"] * MiB
    assert c["per_allreduce"] == P["comm70b.allreduce_MiB"] * MiB
    assert c["per_layer"] == P["comm70b.layer_MiB"] * MiB
    assert c["model"] == P["comm70b.model_GiB"] * GiB
    assert round(c["per_layer"] / 450e9 * 1e3, 2) == P["comm70b.layer_ms_at_450GBps"]


def test_llama70b_params_and_flops():
    per_layer = costs.params_per_layer(8192, 64, 8, 128, 28672)
    per_shard = costs.params_per_shard(8192, 64, 8, 128, 28672, 8)
    assert per_layer == 855_638_016 and round(per_layer / 1e8, 2) == P["params70b.per_layer"] / 1e8
    assert per_shard * 8 == per_layer and round(per_shard / 1e8, 2) == P["params70b.per_shard"] / 1e8
    f = costs.layer_forward_flops(1, 4096, per_layer, 8192)
    assert round(f["matmul"] / 1e12, 1) == P["comm70b.fwd_matmul_TFLOP"]
    assert round(f["attention"] / 1e12, 2) == P["comm70b.attention_TFLOP"]
    assert round(f["total"] / 1e12, 1) == P["comm70b.fwd_TFLOP"]
    per_card = 3 * f["total"] / 8
    assert round(per_card / 1e12, 2) == P["comm70b.per_card_TFLOP"]
    assert round(per_card / 990e12 * 1e3, 2) == P["comm70b.per_card_ms_at_990TFLOPs"]
    comm_ms = costs.tp_layer_comm(1, 4096, 8192, 8, 80)["per_layer"] / 450e9 * 1e3
    assert round(comm_ms / (per_card / 990e12 * 1e3), 2) == P["comm70b.comm_over_compute"]


def test_llama70b_shard_shapes():
    s = costs.llama_layer_shapes(8192, 64, 8, 128, 28672, 8)
    assert s == {"qkv": (8192, 1280), "o": (1024, 8192), "gate_up": (8192, 7168), "down": (3584, 8192)}


def test_overlap_ratio_and_tp_bounds():
    assert round(costs.allgather_overlap_ratio(8, 8192, 990e12, 450e9), 1) == P["overlap.ratio"]
    cw = P["tpbound.C_over_W"]
    assert round(990e12 / 450e9) == cw
    assert round(costs.tp_upper_bound(28672, cw)) == P["tpbound.llama70b"]
    assert round(costs.tp_upper_bound(14336, cw), 1) == P["tpbound.llama8b"]


def test_unidirectional_ring_traffic():
    # AllGather V(N-1)/N, AllToAll V(N-1)/(2N): AllToAll is half of AllGather on a one-way ring
    for N in (2, 4, 8, 16):
        ag = costs.unidirectional_link_traffic("all_gather", 1.0, N)
        a2a = costs.unidirectional_link_traffic("all_to_all", 1.0, N)
        assert ag == pytest.approx((N - 1) / N)
        assert a2a == pytest.approx((N - 1) / (2 * N))
        assert a2a / ag == pytest.approx(0.5)
