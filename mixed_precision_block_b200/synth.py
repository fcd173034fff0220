"""Seeded synthetic Q/K/V shaped like latent video attention inputs.

This module holds the input recipe only: the workload table and the
blob + noise + outlier generator.  It contains none of the attention method's
arithmetic, so both the CUDA path (tests, bench) and the CPU oracle draw their
inputs from here.

Recipe (per tensor Q, K, V and per (batch, head)):

* 4 Gaussian blobs over the (t, y, x) latent grid: centres uniform over the
  grid extent, per-axis width ``sigma_frac * extent`` (0.25; the long
  few-step workload uses sharper blobs, 0.125), amplitude vectors with
  i.i.d. N(0, 1) entries, one per blob;
* plus i.i.d. N(0, 0.5^2) noise on every element;
* then 2 channels (chosen per tensor and head) multiplied by 8 — the outlier
  channels that make per-block quantisation non-trivial;
* computed in fp32 and rounded once to bf16.

Draw order is fixed (tensor Q, K, V; within a tensor: centres, amplitudes,
outlier ranks, noise), so a seed fixes the tensors on a given device type.
CPU and CUDA generators produce different streams; parity tests always feed
the oracle the exact bf16 tensors the GPU consumed.
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, region size, draft weight, budget.

    ``budget`` is (skip, 4-bit, 8-bit, 16-bit) in percent — the reading
    note's 0/4/8/16 "Bit" column order.
    """

    name: str
    B: int
    H: int
    T: int
    Hh: int
    Ww: int
    d: int
    lam: float
    budget: tuple
    rh: int = 8
    rw: int = 8
    sigma_frac: float = 0.25
    seed: int = 0

    @property
    def N(self) -> int:
        return self.T * self.Hh * self.Ww

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny sanity case, a mid-size case, the 118,800-token
# 24-head video shape under two budgets, and a long few-step shape.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 4, 16, 16, 64, 0.5, (25.0, 25.0, 25.0, 25.0)),
    "mid": Workload("mid", 1, 12, 16, 32, 32, 128, 0.5, (50.0, 25.0, 15.0, 10.0)),
    "video": Workload("video", 1, 24, 33, 45, 80, 128, 0.5, (85.0, 0.0, 7.5, 7.5)),
    "video4bit": Workload("video4bit", 1, 24, 33, 45, 80, 128, 0.5,
                          (80.7, 14.4, 4.8, 0.0)),
    "long": Workload("long", 1, 24, 91, 48, 84, 128, 0.5, (70.0, 20.0, 8.0, 2.0),
                     sigma_frac=0.125),
}
WORKLOAD_ORDER = ["tiny", "mid", "video", "video4bit", "long"]


def _blob_field(gen, B, H, T, Hh, Ww, d, sigma_frac, device):
    """Returns blob field [B, H, N, d] fp32 and outlier mask [B, H, d]."""
    ext = torch.tensor([T, Hh, Ww], dtype=torch.float32, device=device)
    centres = torch.rand((B, H, 4, 3), generator=gen, device=device) * ext
    amps = torch.randn((B, H, 4, d), generator=gen, device=device)
    ranks = torch.rand((B, H, d), generator=gen, device=device)
    sig = ext * sigma_frac
    tt = torch.arange(T, device=device, dtype=torch.float32)
    yy = torch.arange(Hh, device=device, dtype=torch.float32)
    xx = torch.arange(Ww, device=device, dtype=torch.float32)
    coords = torch.stack(torch.meshgrid(tt, yy, xx, indexing="ij"), -1).reshape(-1, 3)
    field = torch.empty((B, H, T * Hh * Ww, d), dtype=torch.float32, device=device)
    for b in range(B):
        for h in range(H):
            z = (coords[None, :, :] - centres[b, h][:, None, :]) / sig  # [4, N, 3]
            g = torch.exp(-0.5 * (z * z).sum(-1))  # [4, N]
            field[b, h] = g.t() @ amps[b, h]
    # the two highest-ranked channels become outliers
    top2 = torch.topk(ranks, 2, dim=-1).indices
    outlier = torch.zeros((B, H, d), dtype=torch.bool, device=device)
    outlier.scatter_(-1, top2, True)
    return field, outlier


def make_tensor(gen, wl: Workload, device) -> torch.Tensor:
    field, outlier = _blob_field(gen, wl.B, wl.H, wl.T, wl.Hh, wl.Ww, wl.d,
                                 wl.sigma_frac, device)
    noise = torch.randn(field.shape, generator=gen, device=device, dtype=torch.float32)
    field.add_(noise, alpha=0.5)
    scale = torch.where(outlier, 8.0, 1.0)[:, :, None, :]
    field.mul_(scale)
    return field.to(torch.bfloat16)


def make_qkv(wl: Workload, device="cpu", seed=None):
    """Q, K, V bf16 [B, H, N, d], contiguous, on ``device``."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed if seed is None else seed)
    q = make_tensor(gen, wl, device)
    k = make_tensor(gen, wl, device)
    v = make_tensor(gen, wl, device)
    return q, k, v


def dense_flops(wl: Workload) -> float:
    """Dense-equivalent attention FLOPs over real tokens: 4 * N^2 * d * B * H."""
    return 4.0 * float(wl.N) ** 2 * wl.d * wl.B * wl.H


def region_counts(wl: Workload):
    nry = math.ceil(wl.Hh / wl.rh)
    nrx = math.ceil(wl.Ww / wl.rw)
    return nry, nrx, wl.T * nry * nrx
