"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and the benchmark.

This module only draws random numbers and stores them in the input formats the library takes
(bf16 weights/activations, fp32 or bf16 collective payloads). It holds none of the arithmetic of
the tensor-parallel MLP, the ring collectives or the sharded matmuls, so that the oracle and the
CUDA path can both be fed from it without sharing any of the method.

Recipe (every workload): one ``torch.Generator`` seeded with the workload's seed draws the
tensors in the listed order as fp32 ``randn``/``rand`` values, scaled to the stated standard
deviation or range, then rounded once to bf16 (torch's round-to-nearest-even cast) where the
tensor is bf16. "~N(0, 0.02)" means standard deviation 0.02. Generating on a CUDA device gives a
different (but equally seeded) stream than on the CPU; parity tests compare the two sides on the
same bytes, whichever device drew them.
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "Draw", "bf16_bits", "bits_to_bf16", "to_f64",
    "tiny_mlp", "tiny_collectives", "collective_sweep_seed", "collective_payload",
    "llama8b_mlp", "case_operands", "llama70b_layer",
]


class Draw:
    """Sequential seeded draws: each call takes the next tensor from one generator."""

    def __init__(self, seed: int, device: str | torch.device = "cpu"):
        self.device = torch.device(device)
        self.gen = torch.Generator(device=self.device)
        self.gen.manual_seed(int(seed))

    def normal(self, shape, std: float = 1.0, dtype=torch.bfloat16) -> torch.Tensor:
        x = torch.randn(tuple(shape), generator=self.gen, device=self.device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        return x.to(dtype)

    def uniform(self, shape, lo: float = -1.0, hi: float = 1.0, dtype=torch.float32) -> torch.Tensor:
        x = torch.rand(tuple(shape), generator=self.gen, device=self.device, dtype=torch.float32)
        x.mul_(hi - lo).add_(lo)
        return x.to(dtype)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw uint16 storage of a bf16 tensor (copied to the host)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_bf16(bits: np.ndarray) -> torch.Tensor:
    """A CPU bf16 tensor whose storage is the given uint16 bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(torch.bfloat16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16/fp32 tensor to a float64 numpy array on the host."""
    return t.detach().cpu().to(torch.float64).numpy()


# --------------------------------------------------------------------------------------------
# Workload recipes (shapes of the pages' workloads; see each docstring for the draw order)
# --------------------------------------------------------------------------------------------

def tiny_mlp(seed: int = 0, device="cpu", N=64, h=256, F=1024):
    """Tiny GeLU MLP: X[N,h] ~N(0,1), A[h,F] ~N(0,0.02), B[F,h] ~N(0,0.02), all bf16, drawn in that order."""
    d = Draw(seed, device)
    X = d.normal((N, h), 1.0)
    A = d.normal((h, F), 0.02)
    B = d.normal((F, h), 0.02)
    return X, A, B


def tiny_collectives(seed: int = 0, device="cpu", t=4, chunk=256):
    """Four fp32 shards ~U(-1,1): first the AllGather inputs t x [chunk], then the ReduceScatter
    inputs t x [t*chunk] (each shard's full-size unreduced buffer)."""
    d = Draw(seed, device)
    ag_in = [d.uniform((chunk,)) for _ in range(t)]
    rs_in = [d.uniform((t * chunk,)) for _ in range(t)]
    return ag_in, rs_in


def collective_sweep_seed(t: int, dtype: str, mib: int) -> int:
    """Seed of one point of the collective sweep (t shards, payload dtype, payload MiB)."""
    return 1_000_003 * int(t) + 7 * int(mib) + (1 if dtype == "bf16" else 0)


def collective_payload(t: int, rows: int, cols: int, dtype: str, seed: int, device="cpu"):
    """t shard buffers [rows, cols] ~N(0,1) in fp32 or bf16."""
    d = Draw(seed, device)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return [d.normal((rows, cols), 1.0, dtype=tdt) for _ in range(t)]


def llama8b_mlp(seed: int = 0, device="cpu", N=4096, h=4096, F=14336):
    """Llama-3-8B-shaped SwiGLU MLP: X[N,h] ~N(0,1); fused W_gu[h, 2F] = [W_gate | W_up] ~N(0,0.02);
    W_down[F, h] ~N(0,0.02); bf16, drawn in that order."""
    d = Draw(seed, device)
    X = d.normal((N, h), 1.0)
    W_gu = d.normal((h, 2 * F), 0.02)
    W_down = d.normal((F, h), 0.02)
    return X, W_gu, W_down


def case_operands(seed: int = 0, device="cpu", B=8192, D=8192, F=28672):
    """Sharded-matmul operands: X[B,D] ~N(0,1), W[D,F] ~N(0,0.02), bf16, in that order."""
    d = Draw(seed, device)
    X = d.normal((B, D), 1.0)
    W = d.normal((D, F), 0.02)
    return X, W


def llama70b_layer(seed: int = 0, device="cpu", N=2048, h=8192, n_h=64, n_kv=8, d_h=128, F=28672):
    """Llama-3-70B-shaped layer with the attention core left out.

    Draw order: X[N,h] ~N(0,1); O[N, n_h*d_h] ~N(0,1) (stand-in attention output, shard i holds
    its own heads' columns); W_q[h, n_h*d_h], W_k[h, n_kv*d_h], W_v[h, n_kv*d_h], W_o[n_h*d_h, h],
    W_gate[h,F], W_up[h,F], W_down[F,h], all ~N(0,0.02); bf16."""
    d = Draw(seed, device)
    X = d.normal((N, h), 1.0)
    O = d.normal((N, n_h * d_h), 1.0)
    Wq = d.normal((h, n_h * d_h), 0.02)
    Wk = d.normal((h, n_kv * d_h), 0.02)
    Wv = d.normal((h, n_kv * d_h), 0.02)
    Wo = d.normal((n_h * d_h, h), 0.02)
    Wg = d.normal((h, F), 0.02)
    Wu = d.normal((h, F), 0.02)
    Wd = d.normal((F, h), 0.02)
    return dict(X=X, O=O, Wq=Wq, Wk=Wk, Wv=Wv, Wo=Wo, Wg=Wg, Wu=Wu, Wd=Wd)
