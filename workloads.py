"""Seeded synthetic inputs for the five attention workloads.

This module only draws random numbers and rounds them to the storage type. It
holds none of the attention arithmetic, so both the fp64 oracle (in tests) and
the CUDA path (tests, ``bench.py``, ``smoke()``) can take their inputs from it
without sharing any of the method's code.

Layout of every tensor: contiguous ``(B, H, N, D)``, head dimension innermost,
as in the ``naive_attention`` listing of "Flash Attention principles: making
Transformers faster" (ijyty.com), section "memory bottleneck".

Recipe (all draws on the CPU, ``torch.Generator().manual_seed(seed)``, in the
order Q, K, V, dO, as float32 from N(0, 1)):

* the values are multiplied by the workload's ``qkv_std`` (Q, K, V only;
  dO keeps std 1), then
* rounded to bfloat16 (round-to-nearest-even) unless the workload is fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    D: int
    causal: bool
    dtype: str            # "bf16", "fp16" or "fp32": the storage/input type
    backward: bool        # does the workload include the backward pass
    seed: int
    qkv_std: float = 1.0
    scale: float = field(default=0.0)
    note: str = ""

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale else 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}[self.dtype]

    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: 4*B*H*N^2*D, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.D
        return f / 2 if self.causal else f

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "N": self.N,
                "D": self.D, "causal": self.causal, "dtype": self.dtype,
                "scale": self.softmax_scale, "backward": self.backward}


# The five workloads.  Where a workload states no scale, 1/sqrt(D) is used, the
# scale printed in the ijyty.com listings (section "memory bottleneck").
WORKLOADS = {
    "c1_fp32_fwd": Workload("c1_fp32_fwd", 1, 2, 256, 64, False, "fp32", False,
                            seed=1001, scale=1.0 / 8.0,
                            note="forward only, fp32, B1 H2 N256 D64"),
    "c2_bf16_fwd": Workload("c2_bf16_fwd", 1, 12, 2048, 64, False, "bf16", False,
                            seed=1002, scale=1.0 / 8.0,
                            note="forward only, bf16, B1 H12 N2048 D64"),
    "c3_bf16_fwdbwd": Workload("c3_bf16_fwdbwd", 4, 16, 4096, 64, False, "bf16", True,
                               seed=1003,
                               note="forward+backward, bf16, B4 H16 N4096 D64"),
    "c4_gpt2_causal": Workload("c4_gpt2_causal", 8, 12, 1024, 64, True, "bf16", True,
                               seed=1004, qkv_std=0.5,
                               note="GPT-2-style causal fwd+bwd, bf16, B8 H12 N1024 D64, QKV std 0.5"),
    "c5_long_causal": Workload("c5_long_causal", 1, 8, 65536, 128, True, "bf16", True,
                               seed=1005, scale=1.0 / math.sqrt(128.0),
                               note="long-context causal fwd+bwd, bf16, B1 H8 N65536 D128"),
}


def custom(name: str, B: int, H: int, N: int, D: int, causal: bool, dtype: str = "bf16",
           seed: int = 7, qkv_std: float = 1.0, scale: float = 0.0,
           backward: bool = True) -> Workload:
    """A workload of arbitrary shape with the same recipe (used for edge cases)."""
    return Workload(name, B, H, N, D, causal, dtype, backward, seed, qkv_std, scale)


def make_inputs(w: Workload, with_grad_out: bool | None = None):
    """Return (q, k, v, do) CPU tensors of w's storage type; do is None when unused.

    The draws are made in float32 in the fixed order Q, K, V, dO from one
    generator seeded with ``w.seed``, so a workload always yields the same bits.
    """
    if with_grad_out is None:
        with_grad_out = w.backward
    g = torch.Generator().manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.D)
    out = []
    for i in range(4 if with_grad_out else 3):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if i < 3 and w.qkv_std != 1.0:
            x = x * w.qkv_std
        out.append(x.to(w.torch_dtype).contiguous())
    if not with_grad_out:
        out.append(None)
    return tuple(out)


def sample_rows(w: Workload, h: int, count: int = 64, seed_base: int = 2000):
    """Seeded sample of row indices for one head: rows 0 and N-1 plus (count-2)
    distinct random rows, sorted.  Used where the oracle is evaluated on a
    sample of rows instead of the whole head."""
    g = torch.Generator().manual_seed(seed_base + h)
    if w.N <= count:
        return torch.arange(w.N)
    perm = torch.randperm(w.N - 2, generator=g)[: count - 2] + 1
    rows = torch.cat([torch.tensor([0, w.N - 1]), perm])
    return torch.sort(rows).values
