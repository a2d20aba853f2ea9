"""Seeded synthetic workloads for the fused linear diffusion cross-entropy.

This module only draws random inputs. It holds none of the loss arithmetic,
so both the float64 oracle (through the tests) and the CUDA path can take
their inputs from it and see bit-identical tensors.

The workloads follow the shapes of a masked / block-diffusion LM head:
hidden states ``H[N, D] ~ N(0, 1)``, an LM-head weight ``W[V, D] ~
N(0, sigma_w^2)``, and a masking probability ``t`` drawn per sequence (or
per block of tokens).  Each token is masked with probability ``t``; a
masked token gets a uniform target in ``[0, V)`` and ``p_mask = t``, an
unmasked token gets ``ignore_index`` (its ``p_mask`` is still ``t``, and
the loss never reads it).  This is the noising recipe that produces the
``p_mask`` consumed by ``FusedLinearDiffusionCrossEntropyLoss.forward`` on
the page "fused_linear_diffusion_cross_entropy.py".

Every draw uses one ``torch.Generator`` on the CPU, seeded per case, in a
fixed order: H, W, (large only) the peaky rows, t, the mask, the targets.
H and W are rounded once to the run dtype (bf16 round-to-nearest-even via
torch, or kept fp32) and that exact tensor is what every consumer sees.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

IGNORE_INDEX = -100


@dataclasses.dataclass
class Workload:
    """One synthetic problem: inputs plus the scalar options of the loss."""

    name: str
    H: torch.Tensor            # [N, D] bf16 or fp32, CPU
    W: torch.Tensor            # [V, D] bf16 or fp32, CPU
    target: torch.Tensor       # [N] int64, CPU
    p_mask: torch.Tensor       # [N] fp32, CPU
    logit_scale: float = 1.0
    label_smoothing: float = 0.0
    ignore_index: int = IGNORE_INDEX
    total: float = 0.0         # > 0: explicit; <= 0: count of non-ignored tokens
    grad_out: float = 1.0
    chunk_n: int = 0           # 0: the library picks the token-chunk size
    peaky_rows: Optional[torch.Tensor] = None   # W rows drawn x peaky_mult (sorted), or None

    @property
    def N(self) -> int:
        return int(self.H.shape[0])

    @property
    def D(self) -> int:
        return int(self.H.shape[1])

    @property
    def V(self) -> int:
        return int(self.W.shape[0])

    @property
    def dtype_name(self) -> str:
        return "bf16" if self.H.dtype == torch.bfloat16 else "fp32"

    def n_valid(self) -> int:
        t = self.target
        return int(((t != self.ignore_index) & (t >= 0) & (t < self.V)).sum())


@dataclasses.dataclass(frozen=True)
class Recipe:
    """Shape and distribution of one workload family."""

    name: str
    batch: int
    seq: int
    D: int
    V: int
    dtype: torch.dtype
    sigma_w: float
    t_lo: float
    t_block: int = 0             # 0: one t per sequence; k: one t per k tokens
    logit_scale: float = 1.0
    label_smoothing: float = 0.0
    total_is_count: bool = False
    peaky_frac: float = 0.0      # fraction of W rows multiplied by peaky_mult
    peaky_mult: float = 8.0
    chunk_n: int = 0

    @property
    def N(self) -> int:
        return self.batch * self.seq

    def flops(self) -> float:
        """Credited work of one fwd+bwd call: 6·N·D·V."""
        return 6.0 * self.N * self.D * self.V


# The five workloads the method is exercised on.  Sizes, distributions and
# options are the stated ones; seed 0 everywhere.
RECIPES = {
    "tiny": Recipe("tiny", 2, 32, 64, 512, torch.float32, 0.02, 0.05),
    "mid": Recipe("mid", 4, 1024, 2048, 32000, torch.bfloat16, 0.02, 1e-3),
    "headline": Recipe("headline", 2, 4096, 2560, 151936, torch.bfloat16, 0.02, 1e-3,
                       t_block=4),
    "ragged": Recipe("ragged", 8, 2048, 4096, 128257, torch.bfloat16, 0.015, 1e-3,
                     logit_scale=0.5, label_smoothing=0.1, total_is_count=True),
    "large": Recipe("large", 8, 4096, 4096, 256000, torch.bfloat16, 0.015, 1e-3,
                    peaky_frac=0.01),
}


def make(recipe: Recipe | str, seed: int = 0, *, batch: Optional[int] = None,
         seq: Optional[int] = None, D: Optional[int] = None, V: Optional[int] = None,
         dtype: Optional[torch.dtype] = None, **overrides) -> Workload:
    """Draw one workload.

    ``batch``/``seq``/``D``/``V``/``dtype`` override the recipe's shape so the
    same distribution can be drawn at sizes small enough for the oracle;
    any other keyword overrides a field of the returned workload
    (``label_smoothing``, ``grad_out``, ``total`` ...).
    """
    if isinstance(recipe, str):
        recipe = RECIPES[recipe]
    B = recipe.batch if batch is None else batch
    T = recipe.seq if seq is None else seq
    D_ = recipe.D if D is None else D
    V_ = recipe.V if V is None else V
    dt = recipe.dtype if dtype is None else dtype
    N = B * T

    g = torch.Generator().manual_seed(seed)
    H = torch.randn(N, D_, generator=g).to(dt)
    W = (recipe.sigma_w * torch.randn(V_, D_, generator=g)).to(dt)
    peaky = None
    if recipe.peaky_frac > 0.0:
        rows = torch.randperm(V_, generator=g)[: max(1, int(V_ * recipe.peaky_frac))]
        W[rows] *= recipe.peaky_mult          # a power of two: exact in bf16
        peaky = torch.sort(rows).values
    if recipe.t_block > 0:
        n_blocks = -(-N // recipe.t_block)
        t_unit = recipe.t_lo + (1.0 - recipe.t_lo) * torch.rand(n_blocks, generator=g)
        t = t_unit.repeat_interleave(recipe.t_block)[:N]
    else:
        t_seq = recipe.t_lo + (1.0 - recipe.t_lo) * torch.rand(B, generator=g)
        t = t_seq.repeat_interleave(T)
    masked = torch.rand(N, generator=g) < t
    target = torch.randint(0, V_, (N,), generator=g, dtype=torch.int64)
    target[~masked] = IGNORE_INDEX
    p_mask = t.to(torch.float32).contiguous()

    wl = Workload(
        name=recipe.name, H=H.contiguous(), W=W.contiguous(), target=target,
        p_mask=p_mask, logit_scale=recipe.logit_scale,
        label_smoothing=recipe.label_smoothing,
        total=0.0 if recipe.total_is_count else float(N),
        chunk_n=recipe.chunk_n, peaky_rows=peaky,
    )
    for k, v in overrides.items():
        if not hasattr(wl, k):
            raise TypeError(f"unknown workload field {k!r}")
        setattr(wl, k, v)
    return wl


def sample_rows(n: int, k: int, seed: int, must: tuple = ()) -> torch.Tensor:
    """``k`` distinct row indices in ``[0, n)`` (sorted), always including ``must``."""
    g = torch.Generator().manual_seed(10_000 + seed)
    k = min(k, n)
    idx = set(int(i) for i in must if 0 <= int(i) < n)
    perm = torch.randperm(n, generator=g).tolist()
    for i in perm:
        if len(idx) >= k:
            break
        idx.add(i)
    return torch.tensor(sorted(idx), dtype=torch.int64)
