"""Seeded synthetic inputs and the named workload shapes.

This module holds no attention arithmetic: it only draws random tensors.  Both
the CUDA path (through the tests and the bench) and the fp64 oracle receive the
same tensors from here.

Recipe: a CPU ``torch.Generator`` seeded with the workload's seed draws Q, K, V
and then dO, in that order, as float32 i.i.d. N(0, 1) of shape [B, H, N, d];
each is multiplied by ``input_scale`` (a power of two, so exact) and rounded to
the workload's 16-bit dtype with round-to-nearest-even.  The shapes and dtypes
are those of the pages' examples: the fp16 (B, H, N, d) sequence-length sweep
at B=4, H=32, d=128 of page "Flash Attention 落地评估" section 3, and the causal
fp16 call of page "Llama-Factory 支持 Flash Attention 了吗".
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str          # "fp16" | "bf16"
    causal: bool
    backward: bool
    seed: int
    input_scale: float = 1.0

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float16 if self.dtype == "fp16" else torch.bfloat16

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def fwd_flops(self) -> float:
        """Algorithmic forward flops: 4*B*H*Nq*Nk*d, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Algorithmic backward flops: 2.5x the forward count."""
        return 2.5 * self.fwd_flops()

    def label(self) -> str:
        mask = "causal" if self.causal else "noncausal"
        passes = "fwd+bwd" if self.backward else "fwd"
        return (f"{self.name}: {passes} {mask} {self.dtype} B{self.B} H{self.H} "
                f"N{self.N} d{self.d}")


# The five named workloads (the third is a sweep over N).
TINY = Workload("tiny", 1, 2, 128, 64, "fp16", False, False, 1001)
LAYER_7B = Workload("layer7b", 4, 32, 2048, 128, "bf16", True, False, 1002)
SWEEP = {n: Workload(f"sweep{n}", 4, 32, n, 128, "fp16", False, False, 1003)
         for n in (512, 1024, 2048, 4096, 8192)}
TRAIN_D64 = Workload("train_d64", 2, 16, 4096, 64, "fp16", True, True, 1004)
LONG_CTX = Workload("long_ctx", 1, 16, 16384, 128, "bf16", True, True, 1005, 0.5)
# Head dimension 256: the long-context shape at d = 256, forward only and
# forward + backward.
FWD_D256 = Workload("fwd_d256", 1, 16, 16384, 256, "bf16", True, False, 1006, 0.5)
LONG_CTX_D256 = Workload("long_ctx_d256", 1, 16, 16384, 256, "bf16", True, True, 1010, 0.5)
# The long sweep points run causal in bf16: the causal 16-bit forward at
# N >= 4096, d = 128 on the sweep's batch shape.
CAUSAL_SWEEP = {n: Workload(f"causal{n}", 4, 32, n, 128, "bf16", True, False, 1008) for n in (4096, 8192)}

ALL = [TINY, LAYER_7B, *SWEEP.values(), TRAIN_D64, LONG_CTX, FWD_D256, LONG_CTX_D256, *CAUSAL_SWEEP.values()]


def by_name(name: str) -> Workload:
    for w in ALL:
        if w.name == name:
            return w
    raise KeyError(name)


def make_inputs(w: Workload, with_grad: bool | None = None, device: str = "cpu"):
    """Draw (q, k, v[, do]) for workload ``w`` per the recipe above."""
    with_grad = w.backward if with_grad is None else with_grad
    return draw(w.B, w.H, w.N, w.N, w.d, w.torch_dtype, w.seed, w.input_scale,
                with_grad, device)


def draw(B, H, Nq, Nk, d, dtype, seed, input_scale=1.0, with_grad=False, device="cpu"):
    """Seeded draw of Q [B,H,Nq,d], K and V [B,H,Nk,d] and optionally dO [B,H,Nq,d]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shapes = [(B, H, Nq, d), (B, H, Nk, d), (B, H, Nk, d)]
    if with_grad:
        shapes.append((B, H, Nq, d))
    out = []
    for shp in shapes:
        t = torch.randn(shp, generator=g, dtype=torch.float32)
        if input_scale != 1.0:
            t.mul_(input_scale)
        out.append(t.to(dtype).to(device))
    return tuple(out)


# FP8 inputs: the long-context shape (H16 N16384 d128, causal) at B = 2, so
# that the E4M3 Q, K and V (64 MB each) exceed the 126 MB L2, with one
# descale factor per tensor; forward only.
FWD_FP8 = dict(name="fwd_fp8", B=2, H=16, N=16384, d=128, causal=True, seed=1009)

E4M3_MAX = 448.0  # largest finite E4M3 value


def draw_fp8(B, H, Nq, Nk, d, seed, device="cpu"):
    """Seeded E4M3 inputs with per-tensor descale factors.

    Q [B,H,Nq,d], K and V [B,H,Nk,d] are drawn as fp32 i.i.d. N(0, 1) from a
    CPU generator seeded with ``seed``; each tensor gets descale =
    max|x| / 448 (1 for an all-zero or empty tensor) and is stored as
    torch.float8_e4m3fn(x / descale), torch's round-to-nearest-even
    conversion.  Returns (q8, k8, v8, descale_q, descale_k, descale_v).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    codes, descales = [], []
    for n in (Nq, Nk, Nk):
        t = torch.randn((B, H, n, d), generator=g, dtype=torch.float32)
        amax = float(t.abs().max()) if t.numel() else 0.0
        descale = amax / E4M3_MAX if amax > 0 else 1.0
        codes.append((t / descale).to(torch.float8_e4m3fn).to(device))
        descales.append(descale)
    return (*codes, *descales)


# Packed variable-length batch: a seeded mix of causal self-attention
# sequences (lengths uniform in [1024, 16384], the last one cut so that the
# batch holds 65536 tokens), H = 16, d = 128, bf16, inputs scaled by 0.5.
VARLEN_MIX = dict(name="varlen_mix", H=16, d=128, dtype="bf16", causal=True, seed=1007, total=65536, lo=1024,
                  hi=16384, input_scale=0.5)


def varlen_lengths(seed: int, total: int, lo: int, hi: int) -> list[int]:
    """Seeded sequence lengths, uniform in [lo, hi], summing to total."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    lens: list[int] = []
    while sum(lens) < total:
        n = int(torch.randint(lo, hi + 1, (1,), generator=g))
        lens.append(min(n, total - sum(lens)))
    return lens


def make_varlen_inputs(lengths, H: int, d: int, dtype: torch.dtype, seed: int, input_scale: float = 1.0):
    """Packed head-major Q, K, V, dO [H, total, d] (self-attention: every
    sequence has as many keys as queries) and the int32 offsets [B + 1]."""
    total = sum(lengths)
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    out = []
    for _ in range(4):
        t = torch.randn((H, total, d), generator=g, dtype=torch.float32)
        if input_scale != 1.0:
            t.mul_(input_scale)
        out.append(t.to(dtype))
    cu = torch.tensor([0] + torch.tensor(lengths).cumsum(0).tolist(), dtype=torch.int32)
    return (*out, cu)
