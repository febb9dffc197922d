"""Seeded synthetic inputs for the MonarchAttention forward pass.

This module only draws random numbers and places positional features; it holds
none of the method's arithmetic, so both the float64 oracle (through the tests)
and the CUDA path consume exactly the same tensors.

Workloads (the pages' ViT-B / video-DiT activations are not available, these
stand in for them with the same shapes):

* ``iid``   : Q, K, V drawn i.i.d. N(0, 1) in fp32, in that order, from a CPU
  ``torch.Generator`` seeded with ``seed``, then cast to the requested dtype.
* ``video`` : a (f, h, w) video latent flattened row-major.  Q = Z_q + P and
  K = Z_k + P where Z ~ N(0, 1) and P holds per-axis periodic features
  alpha * [cos(2 pi r x_a / n_a), sin(2 pi r x_a / n_a)], r = 1..4, in disjoint
  channels (f: 0-7, h: 8-15, w: 16-23), alpha^2 = gamma * sqrt(d) / 4 with
  gamma = 2.  Each axis then adds (gamma / 4) * sum_r cos(2 pi r dx_a / n_a) to
  the scaled logit, i.e. the separable positional term D of the MonarchRT
  structure model A = D + S + eps (MonarchRT summary, "Key claims" and
  "Method" (1)).  V ~ N(0, 1).  With ``noise=False`` Z = 0 and the logits are
  a pure separable sum of per-axis terms.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

GAMMA = 2.0
HARMONICS = 4


@dataclass(frozen=True)
class Workload:
    """One synthetic configuration of the forward pass."""

    name: str
    B: int
    H: int
    b1: int
    b2: int
    d: int
    T: int
    c1: int = 1
    c2: int = 1
    dtype: torch.dtype = torch.bfloat16
    kind: str = "iid"          # "iid" or "video"
    latent: tuple | None = None  # (f, h, w) for video workloads
    seed: int = 0

    @property
    def N(self) -> int:
        return self.b1 * self.b2

    @property
    def heads(self) -> int:
        return self.B * self.H


def _cast(x: torch.Tensor, dtype: torch.dtype) -> torch.Tensor:
    return x.to(dtype).contiguous()


def iid_qkv(B, H, N, d, dtype=torch.bfloat16, seed=0):
    """Q, K, V ~ N(0, 1) i.i.d., drawn in fp32 in the order Q, K, V."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    k = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    return _cast(q, dtype), _cast(k, dtype), _cast(v, dtype)


def positional_features(f, h, w, d, gamma=GAMMA):
    """(f*h*w, d) fp32 matrix of per-axis periodic features, zero elsewhere."""
    if d < 6 * HARMONICS:
        raise ValueError("video features need d >= 24 channels")
    alpha = math.sqrt(gamma * math.sqrt(d) / 4.0)
    P = torch.zeros(f, h, w, d, dtype=torch.float64)
    axes = [(f, 0), (h, 1), (w, 2)]
    for n_a, a in axes:
        x = torch.arange(n_a, dtype=torch.float64)
        base = 2 * HARMONICS * a
        for r in range(1, HARMONICS + 1):
            ang = 2 * math.pi * r * x / n_a
            shape = [1, 1, 1]
            shape[a] = n_a
            P[..., base + 2 * (r - 1)] += alpha * torch.cos(ang).view(*shape)
            P[..., base + 2 * (r - 1) + 1] += alpha * torch.sin(ang).view(*shape)
    return P.reshape(f * h * w, d).to(torch.float32)


def video_qkv(B, H, latent, d, dtype=torch.bfloat16, seed=0, noise=True):
    """Video-latent Q/K with a separable periodic logit term, V ~ N(0, 1)."""
    f, h, w = latent
    N = f * h * w
    g = torch.Generator(device="cpu").manual_seed(seed)
    zq = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    zk = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    if not noise:
        zq.zero_()
        zk.zero_()
    P = positional_features(f, h, w, d)
    q = zq + P
    k = zk + P
    return _cast(q, dtype), _cast(k, dtype), _cast(v, dtype)


def make_inputs(wl: Workload, noise: bool = True):
    """Q, K, V (B, H, N, d) for a workload, on the CPU."""
    if wl.kind == "iid":
        return iid_qkv(wl.B, wl.H, wl.N, wl.d, wl.dtype, wl.seed)
    if wl.kind == "video":
        f, h, w = wl.latent
        if f * h * w != wl.N:
            raise ValueError("latent does not match b1*b2")
        return video_qkv(wl.B, wl.H, wl.latent, wl.d, wl.dtype, wl.seed, noise)
    raise ValueError(wl.kind)


# The five synthetic configurations the forward pass is measured and checked on.
TINY_F32 = Workload("tiny-f32 N=256 (16x16) d=64 T=1", 1, 1, 16, 16, 64, 1,
                    dtype=torch.float32, seed=0)
VIT_B = Workload("vit-b B=32 H=12 N=196 (14x14) d=64 T=3", 32, 12, 14, 14, 64, 3,
                 seed=1)
SWEEP = [Workload(f"sweep N={s*s} ({s}x{s}) H=12 d=64 T=1", 1, 12, s, s, 64, 1,
                  seed=2) for s in (16, 32, 64, 128)]
VIDEO_480P = Workload("video-480p f=3 h=30 w=52 N=4680 (fh,w)=(90,52) H=12 d=128 T=1",
                      1, 12, 90, 52, 128, 1, kind="video", latent=(3, 30, 52), seed=3)
VIDEO_720P = Workload("video-720p f=21 h=45 w=80 N=75600 (fh,w)=(945,80) c=2x2 H=12 d=128 T=1",
                      1, 12, 945, 80, 128, 1, c1=2, c2=2, kind="video",
                      latent=(21, 45, 80), seed=4)

WORKLOADS = {
    "tiny": TINY_F32,
    "vit": VIT_B,
    "sweep256": SWEEP[0],
    "sweep1k": SWEEP[1],
    "sweep4k": SWEEP[2],
    "sweep16k": SWEEP[3],
    "480p": VIDEO_480P,
    "720p": VIDEO_720P,
}
