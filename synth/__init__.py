"""Seeded synthetic inputs for the HAD attention forward pass.

This module holds no arithmetic of the method itself: it only draws the
inputs (Q, K, V and the per-head standardization coefficients sigma) that
both the CUDA path and the CPU oracle consume.  Everything is generated on
the CPU with ``torch.Generator`` so the same seed gives the same tensors on
any machine.

The five workloads are shaped like the settings the pages evaluate (the
pith.science review of arXiv 2502.01770, "Referee Report" summary and the
free-parameter notes: BERT on GLUE, DeiT/ViT on ImageNet, T5 on QuALITY with
N scaled linearly with the context length).  No dataset item is used; the
tensors only share the shapes and value structure of those settings.

  tiny   B1  H2  n128   d64  N16   fp32  Q,K,V iid N(0,1)
  bert   B32 H12 n512   d64  N64   bf16  Q,K = rank-16 shared signal + 0.5 noise
  vit    B64 H12 n197   d64  N32   bf16  Q,K,V iid N(0,1) + 0.3 offset
  long   B4  H16 n4096  d64  N512  bf16  Q,K = rank-32 shared signal + unit noise
  vlong  B1  H32 n16384 d128 N2048 bf16  as long, d = 128

sigma_h is the population standard deviation, over (B, n, d), of head h of
the tensor after the cast to its storage dtype, computed in fp64 and stored
as fp32 (the calibration of Eq. 12 needs training data, so the harness
estimates it from the synthetic tensor itself).  tau = 1/sqrt(d).
"""
from dataclasses import dataclass, field
import math

import torch


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    H: int
    n: int
    d: int
    N: int
    dtype: str          # "f32" or "bf16": storage dtype of Q, K, V
    gen: str            # "iid", "iid_offset", "lowrank"
    seed: int
    rank: int = 0
    noise: float = 1.0
    offset: float = 0.0

    @property
    def tau(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def rows(self) -> int:
        return self.B * self.H * self.n

    @property
    def tokens(self) -> int:
        """Query positions per call (each covers all H heads)."""
        return self.B * self.n

    def describe(self) -> str:
        return (f"{self.name}: B={self.B} H={self.H} n={self.n} d={self.d} "
                f"N={self.N} {self.dtype} {self.gen}")


CONFIGS = {
    "tiny": Config("tiny", 1, 2, 128, 64, 16, "f32", "iid", 1001),
    "bert": Config("bert", 32, 12, 512, 64, 64, "bf16", "lowrank", 1002,
                   rank=16, noise=0.5),
    "vit": Config("vit", 64, 12, 197, 64, 32, "bf16", "iid_offset", 1003,
                  offset=0.3),
    "long": Config("long", 4, 16, 4096, 64, 512, "bf16", "lowrank", 1004,
                   rank=32, noise=1.0),
    "vlong": Config("vlong", 1, 32, 16384, 128, 2048, "bf16", "lowrank", 1005,
                    rank=32, noise=1.0),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _randn(shape, seed):
    return torch.randn(shape, generator=_gen(seed), dtype=torch.float32)


def per_head_sigma(x: torch.Tensor) -> torch.Tensor:
    """Population std over (B, n, d) of each head of x [B,H,n,d] (fp64 -> fp32)."""
    x64 = x.to(torch.float64).transpose(0, 1).reshape(x.shape[1], -1)
    return x64.std(dim=1, unbiased=False).to(torch.float32)


def make_inputs(cfg: Config, B: int = None):
    """Draw (Q, K, V, sigma_q, sigma_k) for a workload, on the CPU.

    ``B`` overrides the batch size (used to give each rank of a multi-GPU
    run its own share); batch element b of a larger draw is not the same
    tensor as element b of a smaller one, so overrides are their own inputs.
    """
    B = cfg.B if B is None else B
    H, n, d = cfg.H, cfg.n, cfg.d
    s = cfg.seed * 16
    if cfg.gen == "iid":
        q = _randn((B, H, n, d), s + 1)
        k = _randn((B, H, n, d), s + 2)
    elif cfg.gen == "iid_offset":
        q = _randn((B, H, n, d), s + 1) + cfg.offset
        k = _randn((B, H, n, d), s + 2) + cfg.offset
    elif cfg.gen == "lowrank":
        r = cfg.rank
        u = _randn((B, H, n, r), s + 3)
        w = _randn((H, r, d), s + 4)
        sig = torch.einsum("bhnr,hrd->bhnd", u, w) / math.sqrt(r)
        q = sig + cfg.noise * _randn((B, H, n, d), s + 1)
        k = sig + cfg.noise * _randn((B, H, n, d), s + 2)
        del u, w, sig
    else:
        raise ValueError(cfg.gen)
    v = _randn((B, H, n, d), s + 5)
    if cfg.gen == "iid_offset":
        v = v + cfg.offset
    dt = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    q, k, v = q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous()
    return q, k, v, per_head_sigma(q), per_head_sigma(k)


def to_oracle_array(x: torch.Tensor):
    """numpy view the oracle accepts: float32, or the raw bits of bf16."""
    if x.dtype == torch.bfloat16:
        return x.contiguous().view(torch.int16).numpy().view("uint16")
    if x.dtype == torch.float32:
        return x.contiguous().numpy()
    raise TypeError(x.dtype)


def sample_rows(cfg: Config, count: int, seed: int = 7, B: int = None):
    """Seeded sample of flat query-row ids, always including both ends."""
    B = cfg.B if B is None else B
    total = B * cfg.H * cfg.n
    g = _gen(seed)
    pick = torch.randint(0, total, (max(count - 2, 0),), generator=g)
    ids = torch.cat([torch.tensor([0, total - 1]), pick]).unique()
    return ids.numpy()
