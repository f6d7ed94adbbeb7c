"""Seeded synthetic inputs shaped like the pages' attention workloads.

This module only draws random numbers and names shapes; it holds none of the
attention arithmetic, so the CUDA path and the CPU oracle can both take their
inputs from it without sharing any of the method.

Recipe: a CPU ``torch.Generator`` seeded per workload draws float32 N(0, 1)
samples for Q, then K, then V (Q and K multiplied by ``qk_mult`` before the
cast), which are rounded to the workload's 16-bit type with round-to-nearest-
even. Key-padding lengths, when the workload has them, are drawn last as
int32, uniform on [lo, hi].
"""

from dataclasses import dataclass, replace
from typing import Optional, Tuple

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hk: int
    N: int
    d: int
    dtype: str            # "fp16" or "bf16"
    causal: bool
    key_pad: Optional[Tuple[int, int]] = None   # uniform range of valid key counts
    qk_mult: float = 1.0
    seed: int = 0

    @property
    def scale(self) -> float:
        return float(self.d) ** -0.5

    @property
    def torch_dtype(self):
        return torch.float16 if self.dtype == "fp16" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads, plus the MQA variant of the GQA decoder shape.
WORKLOADS = {
    "single_head_128": Workload("single_head_128", 1, 1, 1, 128, 64, "fp16", False, seed=1000),
    "llama7b_4k_causal": Workload("llama7b_4k_causal", 1, 32, 32, 4096, 128, "fp16", True, seed=1001),
    "bert_large_512_keypad": Workload("bert_large_512_keypad", 32, 16, 16, 512, 64, "bf16", False,
                                      key_pad=(128, 512), seed=1002),
    "gqa_8k_causal": Workload("gqa_8k_causal", 4, 32, 8, 8192, 128, "bf16", True, seed=1003),
    "mqa_8k_causal": Workload("mqa_8k_causal", 4, 32, 1, 8192, 128, "bf16", True, seed=1004),
    "long_32k_causal": Workload("long_32k_causal", 1, 32, 8, 32768, 128, "bf16", True,
                                qk_mult=3.0, seed=1005),
}


def make_inputs(w: Workload, seed: Optional[int] = None, batch_offset: int = 0):
    """Return dict(q, k, v, key_pad_lens) as CPU tensors for workload ``w``.

    q: [B, Hq, N, d], k and v: [B, Hk, N, d] in the workload's 16-bit dtype,
    contiguous. key_pad_lens: int32 [B] or None. ``seed`` overrides the
    workload's seed; ``batch_offset`` shifts it (one shard per rank).
    """
    g = torch.Generator().manual_seed((w.seed if seed is None else seed) + batch_offset)
    dt = w.torch_dtype
    q = torch.randn((w.B, w.Hq, w.N, w.d), generator=g, dtype=torch.float32)
    if w.qk_mult != 1.0:
        q.mul_(w.qk_mult)
    q = q.to(dt)
    k = torch.randn((w.B, w.Hk, w.N, w.d), generator=g, dtype=torch.float32)
    if w.qk_mult != 1.0:
        k.mul_(w.qk_mult)
    k = k.to(dt)
    v = torch.randn((w.B, w.Hk, w.N, w.d), generator=g, dtype=torch.float32).to(dt)
    lens = None
    if w.key_pad is not None:
        lo, hi = w.key_pad
        lens = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int32)
    return {"q": q, "k": k, "v": v, "key_pad_lens": lens}



def make_bias(w: Workload, bias_B: int, bias_H: int, std: float = 2.0, seed: Optional[int] = None,
              device: str = "cpu"):
    """A seeded additive bias [bias_B, bias_H, N, N] in the workload's 16-bit dtype:
    N(0, std²) samples rounded to the dtype (the workloads' pages fix no bias
    distribution; this one moves row maxima by a few units). Drawn on
    ``device`` with its own generator so large planes need no host copy."""
    g = torch.Generator(device=device).manual_seed(
        (w.seed if seed is None else seed) + 7919)
    b = torch.randn((bias_B, bias_H, w.N, w.N), generator=g, dtype=torch.float32, device=device)
    return b.mul_(std).to(w.torch_dtype)
