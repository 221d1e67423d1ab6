"""Seeded synthetic inputs for FLCE: the one module both the GPU path's tests
and the CPU oracle's tests draw their inputs from.

It holds no loss arithmetic: only random draws, dtype rounding and the
workload shapes.  The shapes follow the workloads the pages name:

* the llm.c GPT-2 LM head of PyTorch PR #126348 (B=32, T=1024, C=768,
  V=50257, a bias-free bf16 ``nn.Linear(C, V)``),
* the Llama-3 and Gemma2 training shapes of Liger-Kernel issue #227
  (H=4096, V=128256; Gemma2 with a logit softcap), and
* that issue's ragged-BT sweep (BT = 2**12, then 80 draws of
  randint(2**12, 2**15+1) + randint(0, 1001), then 2**15).

No dataset, tokenizer or trained weights are involved: X and W are normal
draws at the stated scales, labels are uniform in [0, V), and an exact
fraction of rows (chosen by a seeded permutation) is set to ignore_index.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

IGNORE_INDEX = -100


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    BT: int
    H: int
    V: int
    dtype: str          # "bf16" or "fp32"
    x_std: float
    w_std: float
    ignore_frac: float
    softcap: float      # 0.0 = off
    seed: int

    @property
    def flops(self) -> float:
        """Credited fwd+bwd work: 2*BT*H*V per GEMM, three GEMMs."""
        return 6.0 * self.BT * self.H * self.V


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 64, 64, 512, "fp32", 0.02, 0.02, 0.10, 0.0, 1),
    "gpt2_small": Workload("gpt2_small", 32768, 768, 50257, "bf16", 1.0, 0.02, 0.0, 0.0, 2),
    "llama3_8b": Workload("llama3_8b", 8192, 4096, 128256, "bf16", 1.0, 0.02, 0.05, 0.0, 3),
    "gemma2_softcap": Workload("gemma2_softcap", 8192, 3584, 256000, "bf16", 1.0, 0.03, 0.05,
                               30.0, 4),
}


@dataclasses.dataclass(frozen=True)
class CEWorkload:
    """Logits a caller already holds, for the cross-entropy-only path."""
    name: str
    BT: int
    V: int
    dtype: str
    std: float          # logits ~ N(0, std^2), rounded to dtype
    ignore_frac: float
    softcap: float
    seed: int

    @property
    def bytes_per_step(self) -> float:
        """Algorithmic HBM bytes of forward + backward: the logits read twice
        and the gradient written once (labels and lse are negligible)."""
        return 3.0 * self.BT * self.V * (2 if self.dtype == "bf16" else 4)


# PyTorch PR #126348's llm.c tensor: batch 32, sequence 1024, vocabulary
# 50257, bf16.  The logits' scale is that of the GPT-2 LM head above: with
# X ~ N(0, 1) and W ~ N(0, 0.02^2) over H = 768, X W^T has standard deviation
# 0.02 * sqrt(768).
CE_WORKLOADS = {
    "ce_llmc": CEWorkload("ce_llmc", 32 * 1024, 50257, "bf16", 0.02 * 768 ** 0.5, 0.0, 0.0, 21),
}


def make_ce_workload(w: CEWorkload, device="cpu"):
    """Return (logits [BT, V], labels int64 [BT]) of a CE workload: normal
    draws times std rounded (RNE) to dtype, labels uniform in [0, V), an
    exact fraction of rows ignored (seeded permutation)."""
    g = torch.Generator(device=device)
    g.manual_seed(int(w.seed))
    Z = (torch.randn(w.BT, w.V, generator=g, device=device, dtype=torch.float32)
         * w.std).to(torch_dtype(w.dtype))
    labels = torch.randint(0, w.V, (w.BT,), generator=g, device=device, dtype=torch.int64)
    n_ignore = int(round(w.ignore_frac * w.BT))
    if n_ignore:
        labels[torch.randperm(w.BT, generator=g, device=device)[:n_ignore]] = IGNORE_INDEX
    return Z, labels


def ragged_bt_list() -> list[int]:
    """The 82 BT values of the ragged sweep, drawn with numpy's legacy seed 0
    (the issue gives the formula but no seed)."""
    rs = np.random.RandomState(0)
    mid = rs.randint(2 ** 12, 2 ** 15 + 1, 80) + rs.randint(0, 1001, 80)
    return [2 ** 12] + [int(v) for v in mid] + [2 ** 15]


def ragged_workload(index: int, BT: int) -> Workload:
    """Call `index` of the ragged sweep: Llama-3 shape and value scales."""
    base = WORKLOADS["llama3_8b"]
    return dataclasses.replace(base, name="ragged_%d" % index, BT=BT, seed=1000 + index)


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def make_inputs(BT: int, H: int, V: int, dtype: str = "bf16", x_std: float = 1.0,
                w_std: float = 0.02, ignore_frac: float = 0.0, seed: int = 0,
                device: str | torch.device = "cpu", ignore_index: int = IGNORE_INDEX):
    """Return (X [BT,H], W [V,H], labels int64 [BT]) on `device`.

    X and W are fp32 normal draws times the std, rounded (RNE) to `dtype`.
    Exactly round(ignore_frac * BT) rows, picked by a seeded permutation,
    carry ignore_index.  The same seed and device give the same tensors.
    """
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    dt = torch_dtype(dtype)
    X = (torch.randn(BT, H, generator=g, device=device, dtype=torch.float32) * x_std).to(dt)
    W = (torch.randn(V, H, generator=g, device=device, dtype=torch.float32) * w_std).to(dt)
    labels = torch.randint(0, V, (BT,), generator=g, device=device, dtype=torch.int64)
    n_ignore = int(round(ignore_frac * BT))
    if n_ignore:
        idx = torch.randperm(BT, generator=g, device=device)[:n_ignore]
        labels[idx] = ignore_index
    return X.contiguous(), W.contiguous(), labels.contiguous()


def make_workload(w: Workload, device="cpu", BT: int | None = None):
    """Inputs of a named workload (optionally with a different BT)."""
    return make_inputs(w.BT if BT is None else BT, w.H, w.V, w.dtype, w.x_std, w.w_std,
                       w.ignore_frac, w.seed, device=device)


def sample_rows(BT: int, k: int, seed: int = 0) -> list[int]:
    """k distinct row indices: the first and last rows, rows on both sides of
    128-row boundaries, and seeded random rows."""
    fixed = [0, BT - 1, 127, 128, 255, 256, BT // 2, BT - 129]
    rows = [r for r in dict.fromkeys(fixed) if 0 <= r < BT]
    rs = np.random.RandomState(seed)
    while len(rows) < min(k, BT):
        r = int(rs.randint(0, BT))
        if r not in rows:
            rows.append(r)
    return sorted(rows[:k])


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a CPU bf16 tensor as uint16 (for the oracle)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_view(t: torch.Tensor):
    """(array, dtype-tag) for the oracle: bf16 bits or fp32 values."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return bf16_bits(t), "bf16"
    return t.numpy(), None
