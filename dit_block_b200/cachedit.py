"""Cache-DiT reuse decision on top of ``sol_gated_residual_cache_diff``.

The SGLang write-up ("8xH200 上的 MiniMax-H3", xhh.club, Q&A on Cache-DiT) describes the
policy: after warm-up steps, the boundary blocks' normalised residual change is compared
with the cached state; if it is below a threshold and the consecutive-cache limit
allows, the middle blocks reuse the cached result, otherwise they recompute and refresh
the cache.  Video and audio tokens share one packed stack, so a sample takes one joint
decision for both streams ("SGLang acelera video do MiniMax-H3", "Resultado principal").

Readings (the pages give no formula): the change of sample s is
sum|r - cache| / sum|cache| over all of its elements (the two sums the fused kernel
returns); a batch reuses only if every sample may (its middle blocks run for the whole
batch); a sample without cached mass (sum|cache| == 0) always recomputes.
"""
from __future__ import annotations

import dataclasses

import torch


def relative_change(sums: torch.Tensor) -> torch.Tensor:
    """Per-sample change sum|r - cache| / sum|cache| from the [n_samples, 2] sums
    (inf where the cache holds no mass)."""
    s = sums.detach().to("cpu", torch.float64)
    ref = s[:, 1]
    return torch.where(ref > 0, s[:, 0] / torch.where(ref > 0, ref, torch.ones_like(ref)),
                       torch.full_like(ref, float("inf")))


@dataclasses.dataclass
class CacheDiTPolicy:
    threshold: float
    warmup_steps: int
    max_consecutive: int
    consecutive: int = 0

    def decide(self, step: int, change) -> bool:
        """True: reuse the cached middle blocks at this step; False: recompute them (the
        caller then refreshes the cache).  `change` is one value or one per sample."""
        values = [float(c) for c in (change if hasattr(change, "__iter__") else [change])]
        reuse = (step >= self.warmup_steps and all(c < self.threshold for c in values)
                 and self.consecutive < self.max_consecutive)
        self.consecutive = self.consecutive + 1 if reuse else 0
        return reuse
