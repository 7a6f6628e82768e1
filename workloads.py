"""Seeded synthetic attention inputs shaped like video-DiT workloads.

This module is shared by the tests, the bench and the oracle's callers.  It
holds only the input recipe (shapes, distributions, seeds) and none of the
attention or quantisation arithmetic.

Recipe (identical for every caller):
  * one ``torch.Generator('cpu')`` per (batch, head), seeded with
    ``seed * 1_000_003 + b * H + h``; per head it draws in float32, in order,
    q [N, d], k [N, d], the k bias [d], v [N, d] and the outlier mask [N, d],
    then casts to the workload dtype, so the device and the oracle see the same
    stored tensors and any single head can be regenerated on its own.
  * Q, V ~ N(0, 1).
  * K ~ N(0, 1) + b[c], b ~ N(0, 3^2) drawn once per (batch, head) and shared
    by all tokens: the per-channel offset that K smoothing removes.
  * Optionally a fraction of Q entries (uniform random positions) multiplied
    by a factor (0.1 % x 20 on the N=4096 and N=32760 workloads).
  * sm_scale = 1/sqrt(d).
Token counts follow the video latent grids 21x30x52 = 32760 and
21x45x80 = 75600 (frames x height x width after patchify).
"""

from dataclasses import dataclass
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str = "bf16"            # "bf16" | "fp16"
    causal: bool = False
    seed: int = 0
    q_outlier_frac: float = 0.0
    q_outlier_mult: float = 20.0
    modes: tuple = ("i8f8", "nvfp4")

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    @property
    def sm_scale(self):
        return 1.0 / math.sqrt(self.d)

    def ops(self):
        """Metric operations 4*B*H*N^2*d (QK^T and PV, 2 ops per MAC)."""
        return 4.0 * self.B * self.H * self.N * self.N * self.d


SMALL = Workload("small-fp16-B1H2N256d64", 1, 2, 256, 64, "fp16", seed=0, modes=("i8f8",))
MID = Workload("mid-B1H12N4096d128", 1, 12, 4096, 128, "bf16", seed=1, q_outlier_frac=1e-3)
VIDEO_32760 = Workload("video-21x30x52-B1H12N32760d128", 1, 12, 32760, 128, "bf16", seed=2,
                       q_outlier_frac=1e-3)
VIDEO_75600 = Workload("video-21x45x80-B1H40N75600d128", 1, 40, 75600, 128, "bf16", seed=3)

WORKLOADS = {w.name: w for w in (SMALL, MID, VIDEO_32760, VIDEO_75600)}


def sweep(d, N, causal):
    """One point of the B=4, H=32 sweep (d in {64,128}, N in 1024..32768)."""
    return Workload(f"sweep-B4H32N{N}d{d}{'-causal' if causal else ''}", 4, 32, N, d,
                    "bf16", causal=causal, seed=4)


SWEEP_POINTS = [(d, n, c) for d in (64, 128) for n in (1024, 2048, 4096, 8192, 16384, 32768)
                for c in (False, True)]


def make_head(w: Workload, b: int, h: int):
    """Return (q, k, v) of one (batch, head): [N, d] in the workload dtype."""
    g = torch.Generator("cpu").manual_seed(w.seed * 1_000_003 + b * w.H + h)
    shape = (w.N, w.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    k += torch.randn((1, w.d), generator=g, dtype=torch.float32) * 3.0
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if w.q_outlier_frac > 0:
        mask = torch.rand(shape, generator=g, dtype=torch.float32) < w.q_outlier_frac
        q = torch.where(mask, q * w.q_outlier_mult, q)
    dt = w.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt)


def make_inputs(w: Workload, device="cpu"):
    """Return (q, k, v) with shape [B, H, N, d] in the workload dtype."""
    dt = w.torch_dtype
    q = torch.empty((w.B, w.H, w.N, w.d), dtype=dt, device=device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    for b in range(w.B):
        for h in range(w.H):
            hq, hk, hv = make_head(w, b, h)
            q[b, h].copy_(hq)
            k[b, h].copy_(hk)
            v[b, h].copy_(hv)
    return q, k, v


def make_heads_f32(w: Workload, heads):
    """float32 numpy arrays [1, len(heads), N, d] of the selected (b, h) pairs."""
    import numpy as np
    qs, ks, vs = [], [], []
    for (b, h) in heads:
        hq, hk, hv = make_head(w, b, h)
        qs.append(hq.float().numpy())
        ks.append(hk.float().numpy())
        vs.append(hv.float().numpy())
    return (np.stack(qs)[None], np.stack(ks)[None], np.stack(vs)[None])


def custom(B, H, N, d, dtype="bf16", causal=False, seed=0, q_outlier_frac=0.0):
    """Workload of arbitrary shape with the same recipe (tests: ragged, edge cases)."""
    return Workload(f"custom-B{B}H{H}N{N}d{d}", B, H, N, d, dtype, causal=causal, seed=seed,
                    q_outlier_frac=q_outlier_frac)


def make_inputs_device(w: Workload, device):
    """The same distributions as ``make_inputs``, drawn on ``device`` with one
    device generator seeded by the workload seed (a different random stream:
    for timing large workloads, not for comparison with the CPU oracle)."""
    g = torch.Generator(device=device).manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.d)
    q = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    k += torch.randn((w.B, w.H, 1, w.d), generator=g, device=device, dtype=torch.float32) * 3.0
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if w.q_outlier_frac > 0:
        mask = torch.rand(shape, generator=g, device=device, dtype=torch.float32) < w.q_outlier_frac
        q = torch.where(mask, q * w.q_outlier_mult, q)
    dt = w.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt)
