"""Seeded synthetic inputs for the NVFP4 linear layer.

This module holds no quantization arithmetic: it only draws bf16 tensors with the shapes and
value distributions of the pretraining workloads the Quartet II pages describe (LLM linear
layers: activations X [M,K], weights W [N,K] in PyTorch ``Linear`` layout, output gradients
dY [M,N]).  Both the CUDA path's tests and the oracle's tests draw their inputs here, so the
two sides see the same bytes.

Recipes (seed s; X, W and dY use sub-seeds s, s+1, s+2):
  tiny       X, W, dY 256x256, N(0,1); W scaled by 0.02.
  llm1p9b    M=16384, K=2048, N=8192.  X = t_3/sqrt(3) with a seeded 4 of every 1024
             channels (columns) scaled by 20; W ~ N(0, 0.02^2); dY ~ N(0, (1e-4)^2).
  mlp8b_up   M=16384, K=4096, N=14336 (gate/up): X ~ N(0,1); W ~ N(0, 0.02^2);
             dY = N(0, (1e-4)^2) * exp(z_m) with z_m ~ N(0,1) per row.
  mlp8b_down M=16384, K=14336, N=4096: X = SiLU(a) * b with a, b ~ N(0,1); W, dY as above.
  sweep      a bf16 [rows, L] tensor ~ N(0,1), each element independently x50 with p=0.001.
"""
from __future__ import annotations

import torch

SHAPES = {
    "tiny": (256, 256, 256),
    "llm1p9b": (16384, 2048, 8192),
    "mlp8b_up": (16384, 4096, 14336),
    "mlp8b_down": (16384, 14336, 4096),
    "stack1p1b_qkv": (32768, 2048, 6144),
    "stack1p1b_down": (32768, 5632, 2048),
}

# Workloads made of several linear layers: (name, M, K, N, x kind, dY kind, name of the linear
# whose input X this one shares or None).  A shared X is the same tensor (gate and up read the
# block's normalised hidden state).
#   mlp8b      the Llama-3-8B MLP at 16384 tokens: gate and up 4096 -> 14336 on one X ~ N(0,1),
#              down 14336 -> 4096 on X = SiLU(a) * b; dY rows log-normal (many tiny groups).
#   stack1p1b  the linears of one 1.1B-class block (d_model 2048, 16 heads, FFN 5632) at 32768
#              tokens: QKV 2048 -> 6144, O 2048 -> 2048, gate and up 2048 -> 5632 (shared X),
#              down 5632 -> 2048 (SiLU-gated X); other inputs as llm1p9b.
STACKS = {
    "mlp8b": [("gate", 16384, 4096, 14336, "gauss", "lognormal_rows", None),
              ("up", 16384, 4096, 14336, "gauss", "lognormal_rows", "gate"),
              ("down", 16384, 14336, 4096, "silu_gated", "lognormal_rows", None)],
    "stack1p1b": [("qkv", 32768, 2048, 6144, "t3_outlier_channels", "gauss_1e-4", None),
                  ("o", 32768, 2048, 2048, "t3_outlier_channels", "gauss_1e-4", None),
                  ("gate", 32768, 2048, 5632, "t3_outlier_channels", "gauss_1e-4", None),
                  ("up", 32768, 2048, 5632, "t3_outlier_channels", "gauss_1e-4", "gate"),
                  ("down", 32768, 5632, 2048, "silu_gated", "gauss_1e-4", None)],
}
_SINGLE_KINDS = {"tiny": ("gauss", "gauss1"), "llm1p9b": ("t3_outlier_channels", "gauss_1e-4"),
                 "mlp8b_up": ("gauss", "lognormal_rows"), "mlp8b_down": ("silu_gated", "lognormal_rows"),
                 "stack1p1b_qkv": ("t3_outlier_channels", "gauss_1e-4"),
                 "stack1p1b_down": ("silu_gated", "gauss_1e-4")}


def stack_linears(cfg: str):
    """The linears of a workload as (name, M, K, N, x kind, dY kind, shared-X source)."""
    if cfg in STACKS:
        return list(STACKS[cfg])
    M, K, N = SHAPES[cfg]
    xk, dk = _SINGLE_KINDS[cfg]
    return [(cfg, M, K, N, xk, dk, None)]


def stack_inputs(cfg: str, seed: int = 0, device="cpu", only: str | None = None):
    """{name: (X, W, dY)} for every linear of a workload (a single-linear config gives exactly
    linear_inputs(cfg, seed)); linear i draws from sub-seeds seed + 10 i + {0, 1, 2}.  With
    `only`, just that linear (and the one whose X it shares) is drawn."""
    if cfg not in STACKS:
        return {cfg: linear_inputs(cfg, seed, device)}
    need = None
    if only is not None:
        src = {n: sh for n, *_, sh in STACKS[cfg]}
        need = {only, src[only]}
    out = {}
    for i, (name, M, K, N, xk, dk, shared) in enumerate(STACKS[cfg]):
        if need is not None and name not in need:
            continue
        s = seed + 10 * i
        x = out[shared][0] if shared else make_x(M, K, xk, s, device)
        out[name] = (x, make_w(N, K, s + 1, device=device), make_dy(M, N, dk, s + 2, device))
    return out


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def student_t3_unit(shape, g, device) -> torch.Tensor:
    """Student-t with 3 degrees of freedom divided by sqrt(3) (unit variance):
    Z / sqrt(chi2_3 / 3) / sqrt(3) = Z / sqrt(chi2_3)."""
    z = _randn(shape, g, device)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(3):
        chi2 += _randn(shape, g, device) ** 2
    return z / torch.sqrt(chi2)


def make_x(M: int, K: int, kind: str, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(device, seed)
    if kind == "gauss":
        x = _randn((M, K), g, device)
    elif kind == "t3_outlier_channels":
        x = student_t3_unit((M, K), g, device)
        n_out = max(1, (4 * K) // 1024)
        perm = torch.randperm(K, generator=g, device=device)[:n_out]
        x[:, perm] *= 20.0
    elif kind == "silu_gated":
        a = _randn((M, K), g, device)
        b = _randn((M, K), g, device)
        x = torch.nn.functional.silu(a) * b
    else:
        raise ValueError(kind)
    return x.to(torch.bfloat16)


def make_w(N: int, K: int, seed: int, std: float = 0.02, device="cpu") -> torch.Tensor:
    g = _gen(device, seed)
    return (_randn((N, K), g, device) * std).to(torch.bfloat16)


def make_dy(M: int, N: int, kind: str, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(device, seed)
    if kind == "gauss1":
        y = _randn((M, N), g, device)
    elif kind == "gauss_1e-4":
        y = _randn((M, N), g, device) * 1e-4
    elif kind == "lognormal_rows":
        y = _randn((M, N), g, device) * 1e-4
        z = _randn((M, 1), g, device)
        y = y * torch.exp(z)
    else:
        raise ValueError(kind)
    return y.to(torch.bfloat16)


def linear_inputs(cfg: str, seed: int = 0, device="cpu"):
    """(X [M,K], W [N,K], dY [M,N]) bf16 for a named linear-layer workload: X and dY of the
    workload's kinds from sub-seeds seed and seed + 2, W ~ N(0, 0.02) from seed + 1."""
    if cfg not in SHAPES:
        raise ValueError(cfg)
    M, K, N = SHAPES[cfg]
    xk, dk = _SINGLE_KINDS[cfg]
    x = make_x(M, K, xk, seed, device)
    w = make_w(N, K, seed + 1, device=device)
    dy = make_dy(M, N, dk, seed + 2, device)
    return x, w, dy


def custom_linear_inputs(M: int, K: int, N: int, seed: int = 0, device="cpu", x_kind="t3_outlier_channels",
                         dy_kind="lognormal_rows"):
    """Inputs of an arbitrary shape with the llm1p9b-style distributions (used for ragged and
    multi-tile parity cases)."""
    return (make_x(M, K, x_kind, seed, device), make_w(N, K, seed + 1, device=device),
            make_dy(M, N, dy_kind, seed + 2, device))


def sweep_tensor(numel_log2: int, L: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """Quantizer-sweep input: 2^p elements as rows of length L (rows rounded to a multiple of
    128, at least 128), N(0,1) with 0.1% of elements x50."""
    rows = max(128, int(round((2 ** numel_log2) / L / 128.0)) * 128)
    g = _gen(device, seed)
    x = _randn((rows, L), g, device)
    mask = torch.rand((rows, L), generator=g, device=device) < 1e-3
    x = torch.where(mask, x * 50.0, x)
    return x.to(torch.bfloat16)


def sweep_rows(numel_log2: int, L: int) -> int:
    return max(128, int(round((2 ** numel_log2) / L / 128.0)) * 128)

