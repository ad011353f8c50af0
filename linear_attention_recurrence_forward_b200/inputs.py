"""Seeded synthetic inputs for the KDA recurrence (shared by the CUDA path and the oracle).

This module only draws random numbers and shapes them; it holds none of the
recurrence's arithmetic.  Both the CUDA library and the CPU oracle consume the
exact bytes produced here (the oracle widens them losslessly to fp64).

Workload recipe (the pages publish no dataset for this path; everything is synthetic):

* q, k ~ N(0, 1) per element, then L2-normalised over the head dimension in fp32.
  The pages say nothing about query/key normalisation; it is done here, never
  inside the library.
* v ~ N(0, 1).
* beta = sigmoid(N(0, 1)), one scalar per (batch, token, head).
* g = -5 * sigmoid(z) per channel, z ~ N(mu_z, 1).  This is the bounded
  scaled-sigmoid log-decay with lower bound -5 that the Kimi K3 skill card's
  quick facts give for KDA (g in [-5, 0)).  mu_z = 0 by default, -2 for the
  slow-decay K3 workload.
* S0 = 0, or N(0, std) in fp32 when an initial state is requested.
* Everything except the state is then rounded once (round-to-nearest-even) to the
  compute dtype (bf16 or fp32).

Draw order is fixed: q, k, v, z_g, z_beta, then S0, from one torch.Generator
seeded with `seed`.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

__all__ = [
    "KdaConfig",
    "DecodeConfig",
    "PREFILL_CONFIGS",
    "DECODE_CONFIG",
    "make_prefill_inputs",
    "make_decode_inputs",
    "make_prefill_raw_inputs",
    "torch_dtype",
    "fingerprint",
]


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


@dataclass(frozen=True)
class KdaConfig:
    """One prefill workload: shapes, dtype and input distribution."""

    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str = "bf16"
    s0_std: float = 0.0          # 0 -> S0 = 0 (passed as NULL)
    zg_mean: float = 0.0          # mean of the decay logit z
    seed: int = 0
    note: str = ""

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H


@dataclass(frozen=True)
class DecodeConfig:
    """The batched single-token decode workload."""

    name: str
    batch: int
    H: int
    dk: int
    dv: int
    steps: int
    dtype: str = "bf16"
    seed: int = 0


# The five workloads the build is measured and checked on.  Sizes follow the Kimi K3
# description (96 heads; head dim 128; contexts up to 64K) on synthetic data.
PREFILL_CONFIGS = {
    "small_fp32": KdaConfig("small_fp32", B=1, T=256, H=2, dk=64, dv=64, dtype="fp32",
                            note="fp32, chunk 64, S0 = 0"),
    "h32_t4k": KdaConfig("h32_t4k", B=1, T=4096, H=32, dk=128, dv=128, dtype="bf16",
                         note="bf16 inputs, fp32 state, S0 = 0"),
    "k3_b4_t8k": KdaConfig("k3_b4_t8k", B=4, T=8192, H=96, dk=128, dv=128, dtype="bf16",
                           s0_std=0.02, zg_mean=-2.0,
                           note="K3 head count; S0 ~ N(0, 0.02^2); slow-decay regime z ~ N(-2, 1)"),
    "k3_t64k": KdaConfig("k3_t64k", B=1, T=65536, H=96, dk=128, dv=128, dtype="bf16",
                         note="long context, 1024 chunks of 64 carried sequentially"),
}

DECODE_CONFIG = DecodeConfig("decode_b256_h96", batch=256, H=96, dk=128, dv=128, steps=1000)


def _normal(shape, gen, device, mean=0.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if mean != 0.0:
        x.add_(mean)
    return x


def _l2_normalise_(x: torch.Tensor) -> torch.Tensor:
    # fp32 normalisation over the last (head) dimension, in place.
    x.div_(torch.linalg.vector_norm(x, dim=-1, keepdim=True).clamp_min(1e-12))
    return x


def make_prefill_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16",
                        seed: int = 0, s0_std: float = 0.0, zg_mean: float = 0.0,
                        device: str = "cpu", gen: Optional[torch.Generator] = None):
    """Draw (q, k, v, g, beta, S0) in the layouts the library takes.

    q, k, g: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H]; S0: [B, H, dk, dv] fp32 or
    None.  All tensors are contiguous and live on `device`.
    """
    if gen is None:
        gen = torch.Generator(device=device)
        gen.manual_seed(seed)
    dt = torch_dtype(dtype)
    q = _l2_normalise_(_normal((B, T, H, dk), gen, device)).to(dt)
    k = _l2_normalise_(_normal((B, T, H, dk), gen, device)).to(dt)
    v = _normal((B, T, H, dv), gen, device).to(dt)
    z_g = _normal((B, T, H, dk), gen, device, mean=zg_mean)
    g = (torch.sigmoid(z_g).mul_(-5.0)).to(dt)
    del z_g
    beta = torch.sigmoid(_normal((B, T, H), gen, device)).to(dt)
    S0 = None
    if s0_std > 0.0:
        S0 = _normal((B, H, dk, dv), gen, device).mul_(s0_std)
    return q, k, v, g, beta, S0


def make_prefill_raw_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16",
                            seed: int = 0, s0_std: float = 0.0, zg_mean: float = 0.0,
                            device: str = "cpu", gen: Optional[torch.Generator] = None):
    """The same draws as make_prefill_inputs before any transformation: (q_raw, k_raw, v, z_g,
    z_beta, S0) with q_raw, k_raw ~ N(0, 1) (not normalised), z_g ~ N(zg_mean, 1), z_beta ~ N(0, 1),
    all rounded to the dtype; for the prologue-fused prefill."""
    if gen is None:
        gen = torch.Generator(device=device)
        gen.manual_seed(seed)
    dt = torch_dtype(dtype)
    q = _normal((B, T, H, dk), gen, device).to(dt)
    k = _normal((B, T, H, dk), gen, device).to(dt)
    v = _normal((B, T, H, dv), gen, device).to(dt)
    z_g = _normal((B, T, H, dk), gen, device, mean=zg_mean).to(dt)
    z_beta = _normal((B, T, H), gen, device).to(dt)
    S0 = None
    if s0_std > 0.0:
        S0 = _normal((B, H, dk, dv), gen, device).mul_(s0_std)
    return q, k, v, z_g, z_beta, S0


def make_config_inputs(cfg: KdaConfig, device: str = "cpu"):
    return make_prefill_inputs(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.dtype, seed=cfg.seed,
                               s0_std=cfg.s0_std, zg_mean=cfg.zg_mean, device=device)


def make_decode_inputs(batch: int, H: int, dk: int, dv: int, dtype: str = "bf16",
                       gen: Optional[torch.Generator] = None, seed: int = 0, device: str = "cpu"):
    """One decode step's fresh token: q, k, g [batch, H, dk]; v [batch, H, dv]; beta [batch, H].

    Same distributions as the prefill recipe (z_g ~ N(0, 1)).  Successive calls with the
    same generator continue its stream, so step s of a run is reproducible.
    """
    if gen is None:
        gen = torch.Generator(device=device)
        gen.manual_seed(seed)
    q, k, v, g, beta, _ = make_prefill_inputs(batch, 1, H, dk, dv, dtype, gen=gen, device=device)
    return (q.view(batch, H, dk), k.view(batch, H, dk), v.view(batch, H, dv),
            g.view(batch, H, dk), beta.view(batch, H))


def fingerprint(*tensors) -> str:
    """SHA-256 (hex) of the exact bytes of the given tensors (None entries skipped), each preceded by
    its dtype and shape, in the order given: the identity of a run's inputs, whichever side (the
    library or the oracle) consumes them.  Device tensors are copied to the host in 256 MiB pieces."""
    import hashlib

    h = hashlib.sha256()
    for t in tensors:
        if t is None:
            continue
        t = t.contiguous()
        h.update(f"{t.dtype}:{tuple(t.shape)};".encode())
        flat = t.view(-1).view(torch.uint8) if t.numel() else t.new_empty(0, dtype=torch.uint8)
        step = 256 << 20
        for i in range(0, flat.numel(), step):
            h.update(flat[i:i + step].cpu().numpy().tobytes())
    return h.hexdigest()
