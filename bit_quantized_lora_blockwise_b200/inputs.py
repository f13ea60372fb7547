"""Seeded synthetic inputs and the workload shapes.

This module holds no arithmetic of the method (no quantization, no GEMM):
only seeded random tensors and the layer shapes of the workloads, so that
the CUDA path and the CPU oracle are fed byte-identical inputs.

Shapes follow the LLaMA-style decoder linears the workloads name:
adapters on every linear of the block (q, k, v, o, gate, up, down), as the
QLoRA pages' "LoRA placement" section (promptingindex.com) recommends.
A weight is stored [N, K] = (out_features, in_features), row-major.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BASE_SEED = 20261202


@dataclass(frozen=True)
class Linear:
    name: str
    N: int  # out features
    K: int  # in features


def decoder_linears(d: int, ffn: int) -> list[Linear]:
    """The seven linears of one decoder block: q, k, v, o (d x d),
    gate and up (d -> ffn) and down (ffn -> d)."""
    return [Linear("q", d, d), Linear("k", d, d), Linear("v", d, d), Linear("o", d, d),
            Linear("gate", ffn, d), Linear("up", ffn, d), Linear("down", d, ffn)]


@dataclass(frozen=True)
class Workload:
    key: str
    description: str
    linears: tuple
    M: tuple  # token counts
    r: int
    alpha: float
    w_std: float
    outlier_frac: float = 0.0
    outlier_sigma: float = 10.0
    layers: int = 1
    index: int = 0
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "single_1024": Workload(
        "single_1024", "single QLoRA linear 1024x1024, M=16, r=8, alpha=16",
        (Linear("single", 1024, 1024),), (16,), 8, 16.0, 0.02, index=1),
    "llama7b_set": Workload(
        "llama7b_set", "7B-shaped linear set (d=4096, ffn=11008), M=4x512=2048, r=64, alpha=16, "
        "0.1% outliers at +-10 sigma",
        tuple(decoder_linears(4096, 11008)), (2048,), 64, 16.0, 0.02, 0.001, 10.0, index=2),
    "llama13b_quant_sweep": Workload(
        "llama13b_quant_sweep", "quantize + double-quant + dequant over 40 layers x 7 linears "
        "(d=5120, ffn=13824)",
        tuple(decoder_linears(5120, 13824)), (), 0, 0.0, 0.02, layers=40, index=3),
    "llama65b_fwd": Workload(
        "llama65b_fwd", "65B-shaped linears (d=8192, ffn=22016), M in {1,4,16,4096}, r=64, alpha=16",
        tuple(decoder_linears(8192, 22016)), (1, 4, 16, 4096), 64, 16.0, 0.015, index=4),
    "llama33b_block": Workload(
        "llama33b_block", "33B-shaped decoder block (d=6656, ffn=17920), M=1x2048, r=64, alpha=16, "
        "fwd + recompute-dequant bwd",
        tuple(decoder_linears(6656, 17920)), (2048,), 64, 16.0, 0.02, index=5),
}


def seed_for(workload_index: int, linear_index: int, tensor_id: int, layer: int = 0) -> int:
    """seed = 20261202 + 1000*workload + 10*linear + tensor (+ 100000*layer)."""
    return BASE_SEED + 1000 * workload_index + 10 * linear_index + tensor_id + 100000 * layer


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) samples drawn in fp32 and rounded to bf16."""
    g = _gen(seed, device)
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def normal_f16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) samples drawn in fp32 and rounded to fp16."""
    g = _gen(seed, device)
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.float16)


def weight_bf16(N: int, K: int, std: float, seed: int, outlier_frac: float = 0.0,
                outlier_sigma: float = 10.0, device="cpu") -> torch.Tensor:
    """Frozen base weight [N, K]: N(0, std^2), with a fraction of entries at
    seeded uniform positions replaced by +-outlier_sigma*std (random sign)."""
    g = _gen(seed, device)
    w = torch.randn(N * K, generator=g, device=device, dtype=torch.float32)
    w.mul_(std)
    n_out = int(round(outlier_frac * N * K))
    if n_out > 0:
        pos = torch.randint(0, N * K, (n_out,), generator=g, device=device)
        sign = torch.randint(0, 2, (n_out,), generator=g, device=device).to(torch.float32) * 2 - 1
        w[pos] = sign * (outlier_sigma * std)
    return w.view(N, K).to(torch.bfloat16)


def layer_inputs(wl: Workload, li: int, M: int, device="cpu", layer: int = 0,
                 need_grad_inputs: bool = True) -> dict:
    """Every input of one linear of a workload: W, X, A, B, dY (bf16)."""
    lin = wl.linears[li]
    out = {"W": weight_bf16(lin.N, lin.K, wl.w_std, seed_for(wl.index, li, 0, layer),
                            wl.outlier_frac, wl.outlier_sigma, device)}
    if M > 0:
        out["X"] = normal_bf16((M, lin.K), 1.0, seed_for(wl.index, li, 1, layer), device)
        out["A"] = normal_bf16((lin.K, wl.r), 0.01, seed_for(wl.index, li, 2, layer), device)
        out["B"] = normal_bf16((wl.r, lin.N), 0.01, seed_for(wl.index, li, 3, layer), device)
        if need_grad_inputs:
            out["dY"] = normal_bf16((M, lin.N), 1.0, seed_for(wl.index, li, 4, layer), device)
    return out


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor's bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def f16_bits(t: torch.Tensor):
    """uint16 numpy view of an fp16 tensor's bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
