"""Oracle for the tensor-parallel MLP, the ring collectives and the four sharded-matmul cases.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, single-threaded-by-design CPU restatement of
what the pages compute, written from them in fp64 (GEMMs, activations) and in IEEE fp32 where the
ring's own summation order is emulated bit for bit. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s ``cpu_baseline`` / ``--impl reference`` legs may import it. The library in
``tensor_sharded_matmul_b200`` never imports, calls or links anything here, and nothing here imports
the library: the two share no code. Inputs come from ``synthetic`` (random draws only).

Sources (cited in each function by page title and section):
  * "Scaling Book 入门第 6 章：分片矩阵乘法 — 分布式计算的核心" (r00kie-liu.github.io, scaling-infra-ch06):
    sharding notation (§6.1), the four cases (§6.2), AllGather/ReduceScatter/AllReduce semantics and
    their transposition (§6.4), roofline (§6.5), Megatron column/row linear (§6.7), worked problems (§6.9).
  * "Scaling Book 入门第 5 章：Sharded Matrices 上篇 — 集合通信原语" (scaling-infra-ch05):
    the ring algorithm and its N=4 AllGather step tables (§5.2), the primitives' before/after
    examples and AllReduce = ReduceScatter + AllGather (§5.3).
  * "张量并行与序列并行" (hs-black.github.io, scaling-tensor-parallel): column/row parallel linear
    (§矩阵乘法的两种切法), the MLP and SwiGLU (§MLP：先列后行，只通信一次), fused QKV and GQA
    (§注意力：按头切 / §GQA), per-rank ring bytes (§预备), communication volume (§精确的通信量).
  * pufanyi.com "ml-revisit-infra", §Tensor Parallel: column/row identities and the MLP split.

Pins: every function is checked by ``tests/test_oracle_*.py`` against values the pages print,
closed forms, invariants or brute force. The one exception is stated where it applies:
exact GEMM outputs of full-size workloads beyond the stated bf16 tolerance are parity unpinned
(the pages print no values for them); the tolerance check itself is pinned through brute force
on tiny shapes and the block-matrix identity.
"""
