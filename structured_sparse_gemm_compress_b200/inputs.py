"""Seeded synthetic inputs and workload shapes for the N:M sparse GEMM path.

This module holds no part of the method's arithmetic: it only draws seeded
random tensors on the CPU and lists the layer shapes of the workloads.  The CPU
oracle and the CUDA library both consume what it produces, so they see
identical bytes.

The shapes stand in for the models measured in "Realizable N:M Sparse
Transformer Inference via Search-Kernel Co-Design" (section 2.1: the Q/K/V
projection, the attention output projection and the two FFN linears dominate
ViT inference time).  No dataset or trained weight is used: ImageNet-1K and the
trained ViT/Swin checkpoints are replaced by the value distributions below.
"""
from __future__ import annotations

import random
from dataclasses import dataclass

import torch

INT8, FP16, BF16 = "int8", "fp16", "bf16"
PATTERNS = {"1:4": (1, 4), "2:4": (2, 4), "2:8": (2, 8), "4:8": (4, 8)}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def int8_uniform(shape, lo: int, hi: int, seed: int) -> torch.Tensor:
    """int8 tensor, uniform on the integers [lo, hi]."""
    return torch.randint(lo, hi + 1, tuple(shape), generator=_gen(seed), dtype=torch.int16).to(torch.int8)


def float_normal(shape, std: float, seed: int, dtype: str) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 and rounded to fp16 or bf16."""
    t = torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32) * std
    return t.to(torch.float16 if dtype == FP16 else torch.bfloat16)


def normal_f32(shape, std: float, seed: int) -> torch.Tensor:
    """fp32 N(0, std^2) (per-channel biases of the fused output stage)."""
    return torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32) * std


def scale_uniform(n: int, lo: float, hi: float, seed: int) -> torch.Tensor:
    """Per-output-channel fp32 scale, uniform on [lo, hi)."""
    return torch.rand((n,), generator=_gen(seed), dtype=torch.float32) * (hi - lo) + lo


@dataclass(frozen=True)
class Layer:
    name: str
    T: int          # tokens (rows of X and Y)
    K: int          # in-features
    n_out: int      # out-features
    dtype: str
    N: int
    M: int
    scaled: bool    # per-output-channel fp32 scale
    seed: int

    @property
    def nm(self) -> str:
        return "dense" if self.N == self.M else f"{self.N}:{self.M}"

    def weight(self) -> torch.Tensor:
        if self.dtype == INT8:
            return int8_uniform((self.n_out, self.K), -127, 127, self.seed)
        return float_normal((self.n_out, self.K), 0.02, self.seed, self.dtype)

    def activation(self, T: int | None = None) -> torch.Tensor:
        T = self.T if T is None else T
        if self.dtype == INT8:
            return int8_uniform((T, self.K), -128, 127, self.seed + 1)
        return float_normal((T, self.K), 1.0, self.seed + 1, self.dtype)

    def scale(self) -> torch.Tensor | None:
        if not self.scaled:
            return None
        return scale_uniform(self.n_out, 0.001, 0.01, self.seed + 2)

    def dense_ops(self) -> int:
        """Dense-equivalent operation count 2*T*K*n_out."""
        return 2 * self.T * self.K * self.n_out

    def kept_ops(self) -> int:
        """Useful operations: 2 per kept weight and token, (N/M) x the dense-equivalent count."""
        return 2 * self.T * (self.K // self.M) * self.N * self.n_out


def _vit_block(d: int, hidden: int):
    return [("qkv", d, 3 * d), ("proj", d, d), ("fc1", d, hidden), ("fc2", hidden, d)]


def single_layer() -> list[Layer]:
    """One ViT-B linear, INT8 2:4, T=197, 768->768, int32 output, seed 0."""
    return [Layer("vitb.single", 197, 768, 768, INT8, 2, 4, False, 0)]


def vit_b_int8(T: int = 12608, patterns=("1:4", "2:4", "2:8", "4:8")) -> list[Layer]:
    """ViT-B/16 linears at batch 64 (T=12608), INT8 with per-channel scale."""
    out = []
    for j, nm in enumerate(patterns):
        N, M = PATTERNS[nm]
        for i, (name, k, n) in enumerate(_vit_block(768, 3072)):
            out.append(Layer(f"vitb.{name}", T, k, n, INT8, N, M, True, 2000 + 16 * i))
    return out


def vit_l_fp16(T: int = 6304, patterns=("1:4", "2:4", "2:8"), dtype: str = FP16) -> list[Layer]:
    """ViT-L/16 linears at batch 32 (T=6304), FP16 weights N(0,0.02), X N(0,1)."""
    out = []
    for nm in patterns:
        N, M = PATTERNS[nm]
        for i, (name, k, n) in enumerate(_vit_block(1024, 4096)):
            out.append(Layer(f"vitl.{name}", T, k, n, dtype, N, M, False, 3000 + 16 * i))
    return out


SWIN_T_STAGES = ((96, 3136), (192, 784), (384, 196), (768, 49))


def swin_t_int8(batch: int = 128, patterns=("2:4", "2:8")) -> list[Layer]:
    """Swin-T window-attention and MLP linears at batch 128, per stage."""
    out = []
    for nm in patterns:
        N, M = PATTERNS[nm]
        for s, (d, tok) in enumerate(SWIN_T_STAGES):
            for i, (name, k, n) in enumerate(_vit_block(d, 4 * d)):
                out.append(Layer(f"swint.s{s}.{name}", batch * tok, k, n, INT8, N, M, True,
                                 4000 + 100 * s + 16 * i))
    return out


MIXED_CHOICES = ("dense", "4:8", "2:4", "2:8", "1:4")


def vit_b_mixed(T: int, seed: int = 5) -> list[Layer]:
    """All 48 linears of ViT-B/16, each layer's N:M drawn from MIXED_CHOICES."""
    rng = random.Random(seed)
    out = []
    for blk in range(12):
        for i, (name, k, n) in enumerate(_vit_block(768, 3072)):
            choice = rng.choice(MIXED_CHOICES)
            N, M = (4, 4) if choice == "dense" else PATTERNS[choice]
            out.append(Layer(f"vitb.b{blk}.{name}", T, k, n, INT8, N, M, True,
                             5000 + 16 * (4 * blk + i)))
    return out
