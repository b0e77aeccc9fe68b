"""One Llama-style tensor-parallel layer without its attention core, in fp64 (test infrastructure).

Source: "张量并行与序列并行", §注意力：按头切，以及 GQA 的约束 (Q/K/V column-split on head boundaries,
W_O row-split, one AllReduce after it; the layer has 2 AllReduces forward: attention output and MLP)
and §MLP：先列后行 (SwiGLU MLP, one AllReduce). The attention core (softmax(QK^T)V) is not part of this
path: the per-shard attention outputs O_i are inputs.

Reading: no norms (none are on the path); residual adds in fp32-or-wider; the MLP input is the
residual stream h1 rounded to bf16 (activations are bf16 on the pages).
"""
from __future__ import annotations

import numpy as np

from .bf16 import round_to_bf16_f64
from .mlp import activate, matmul


def layer_forward(X, O_shards, Wqkv_shards, Wo_shards, Wgu_shards, Wdown_shards, rows=None):
    """Returns the per-shard QKV projections, the attention-output sum, h1 = X + attn, the MLP sum
    and y = h1 + mlp, for all token rows or only ``rows`` (every quantity is row-local)."""
    sel = (lambda a: np.asarray(a)[rows]) if rows is not None else (lambda a: np.asarray(a))
    Xr = sel(X).astype(np.float64)
    qkv = [matmul(Xr, W) for W in Wqkv_shards]                      # column-parallel, no comm
    attn = sum(matmul(sel(O), W) for O, W in zip(O_shards, Wo_shards))   # row-parallel partials + AllReduce
    h1 = Xr + attn
    h1_in = round_to_bf16_f64(h1)                                    # bf16 activation into the MLP
    mlp = sum(matmul(activate(matmul(h1_in, Wgu), "swiglu"), Wd) for Wgu, Wd in zip(Wgu_shards, Wdown_shards))
    y = h1 + mlp
    return {"qkv": qkv, "attn": attn, "h1": h1, "mlp": mlp, "y": y}
