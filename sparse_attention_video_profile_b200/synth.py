"""Seeded synthetic inputs for spatial/temporal sparse 3D attention.

This module builds inputs only: the workload table, Q/K/V tensors and the
sampled query rows. It holds none of the method's arithmetic (no masks, no
softmax, no profiling), so both the fp64 oracle and the CUDA path can be fed
from it without sharing any computation.

Token layout follows "Sparse Video-Gen" (paperhub.cn, Weakness 1 answer): a
video of N frames with F tokens per frame, token (i, j) flattened to
x = i*F + j, tensors laid out [B, H, L=N*F, d].

Head construction: every head has a frame embedding table E_f[N, d] and a
position embedding table E_p[F, d], shared by Q, K and V of that head, and
    X[i*F + j] = w_f * E_f[i] + w_p * E_p[j] + noise * eps,   eps ~ N(0, 1)
with separate eps draws for Q, K and V.  A head meant to be spatial gets a
large frame weight (w_f = W, w_p = 1); a temporal head the reverse.  The
embeddings are drawn as N(0, 1) * emb_std with emb_std = d**-0.25 by default:
with score scale 1/sqrt(d) the in-band logit boost is then about W**2, which
concentrates the softmax mass in the intended band.  (With emb_std = d**-0.5,
the literal reading, the boost is only about W**2/sqrt(d) and the intended
labels do not hold; that reading is still available through ``emb_std``.)
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

SPATIAL = 0
TEMPORAL = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention-call shape plus its synthetic-head recipe."""

    name: str
    B: int
    H: int
    N: int          # frames
    F: int          # tokens per frame
    d: int          # head dim
    dtype: str      # "bf16" or "fp32"
    a1: int         # spatial band: keep |i1 - i2| < a1
    a2: int         # temporal band: keep |j1 - j2| < a2
    S: int          # sampled query rows for online profiling
    kinds: str      # "fixed01" (head0 spatial, head1 temporal), "half" or "coin"
    weight: tuple   # ("const", W) or ("uniform", lo, hi)
    noise: float = 0.1

    @property
    def L(self) -> int:
        return self.N * self.F

    def with_bands(self, a1: int, a2: int, name: Optional[str] = None) -> "Workload":
        return dataclasses.replace(self, a1=a1, a2=a2, name=name or f"{self.name}-a1{a1}-a2{a2}")


# The workload table.  Band widths for the two video-model shapes are the
# integers whose mask density is nearest the stated target (closed-form
# densities are checked in the tests).
WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=2, N=4, F=64, d=64, dtype="fp32", a1=1, a2=4, S=32,
                     kinds="fixed01", weight=("const", 3.0)),
    "small": Workload("small", B=1, H=8, N=8, F=256, d=64, dtype="bf16", a1=2, a2=16, S=64,
                      kinds="half", weight=("const", 3.0)),
    "cogvideox": Workload("cogvideox", B=1, H=48, N=13, F=1350, d=64, dtype="bf16", a1=3, a2=181,
                          S=64, kinds="coin", weight=("uniform", 1.0, 4.0)),
    "hunyuan": Workload("hunyuan", B=1, H=24, N=33, F=3600, d=128, dtype="bf16", a1=3, a2=281,
                        S=128, kinds="coin", weight=("uniform", 1.0, 4.0)),
}

# Mixed sparse-pattern workload (per-head modes instead of spatial/temporal
# labels): diagonal band of width 2F, multi-diagonal of stride F and width 64
# (half-width 32), vertical stripe over the first 512 keys.
WORKLOADS["mixed"] = Workload("mixed", B=1, H=24, N=21, F=1560, d=128, dtype="bf16", a1=3, a2=33, S=128,
                              kinds="coin", weight=("uniform", 1.0, 4.0))
MIXED_PARAMS = {"window": 1560, "md_half": 32, "stripe": 512}
# SVG2-style semantic-aware attention on the HunyuanVideo shape: query / key
# cluster counts, Lloyd rounds from the deterministic start, keep threshold.
SVG2_PARAMS = {"Cq": 128, "Ck": 512, "iters": 8, "p": 0.9}
WORKLOADS["svg2"] = Workload("svg2", B=1, H=24, N=33, F=3600, d=128, dtype="bf16", a1=3, a2=281, S=128,
                             kinds="coin", weight=("uniform", 1.0, 4.0))
# Mode shares for heads after the first five (which take modes 0..4 in order
# so every mode is present): full, skip, diagonal, multi-diagonal, stripe.
MIXED_MODE_P = (0.10, 0.05, 0.35, 0.30, 0.20)

# HunyuanVideo-shaped density sweep: target density -> (a1, a2).
HUNYUAN_SWEEP = {0.05: (1, 92), 0.10: (2, 185), 0.15: (3, 281), 0.20: (4, 381),
                 0.30: (6, 589), 0.40: (8, 812), 0.50: (10, 1055)}


def head_kinds(wl: Workload, seed: int) -> np.ndarray:
    """Constructed kind of every (b, h) head: 0 spatial, 1 temporal. Shape [B, H] int8."""
    rng = np.random.default_rng(seed)
    n = wl.B * wl.H
    if wl.kinds == "fixed01":
        kinds = np.array([h % 2 for h in range(n)])
    elif wl.kinds == "half":
        kinds = rng.permutation(np.arange(n) % 2)
    elif wl.kinds == "coin":
        kinds = (rng.random(n) < 0.5).astype(np.int64)
    else:
        raise ValueError(wl.kinds)
    return kinds.reshape(wl.B, wl.H).astype(np.int8)


def head_weights(wl: Workload, seed: int) -> np.ndarray:
    """Dominant weight W of every head, shape [B, H] float64."""
    rng = np.random.default_rng(seed + 7919)
    n = wl.B * wl.H
    if wl.weight[0] == "const":
        w = np.full(n, float(wl.weight[1]))
    else:
        w = rng.uniform(wl.weight[1], wl.weight[2], n)
    return w.reshape(wl.B, wl.H)


def head_modes(B: int, H: int, seed: int) -> np.ndarray:
    """Mixed-pattern mode of every head, [B, H] int8 (0 full, 1 skip,
    2 diagonal, 3 multi-diagonal, 4 vertical stripe)."""
    rng = np.random.default_rng(seed + 15485863)
    n = B * H
    modes = rng.choice(5, size=n, p=MIXED_MODE_P)
    modes[:min(5, n)] = np.arange(min(5, n))
    return modes.reshape(B, H).astype(np.int8)


def torch_dtype(wl: Workload) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[wl.dtype]


def make_qkv(wl: Workload, seed: int = 0, device="cpu", emb_std: Optional[float] = None):
    """Q, K, V of shape [B, H, L, d] in the workload dtype, on ``device``.

    Draw order (torch generator seeded with ``seed`` on ``device``): E_f for
    all heads, E_p for all heads, then eps_Q, eps_K, eps_V.  Values are formed
    in fp32 and rounded once to the workload dtype.
    """
    if emb_std is None:
        emb_std = wl.d ** -0.25
    B, H, N, F, d = wl.B, wl.H, wl.N, wl.F, wl.d
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    kinds = torch.from_numpy(head_kinds(wl, seed).astype(np.float32)).to(device)
    W = torch.from_numpy(head_weights(wl, seed).astype(np.float32)).to(device)
    w_f = torch.where(kinds == SPATIAL, W, torch.ones_like(W)).view(B, H, 1, 1, 1)
    w_p = torch.where(kinds == TEMPORAL, W, torch.ones_like(W)).view(B, H, 1, 1, 1)
    E_f = torch.randn(B, H, N, 1, d, generator=gen, device=device) * emb_std
    E_p = torch.randn(B, H, 1, F, d, generator=gen, device=device) * emb_std
    base = w_f * E_f + w_p * E_p                      # [B, H, N, F, d]
    out = []
    for _ in range(3):
        eps = torch.randn(B, H, N, F, d, generator=gen, device=device)
        x = base + wl.noise * eps
        out.append(x.reshape(B, H, N * F, d).to(torch_dtype(wl)).contiguous())
        del eps, x
    return tuple(out)


def sample_rows(L: int, S: int, seed: int = 0) -> np.ndarray:
    """Profiling query rows: S distinct positions in [0, L), sorted, int32.

    The same rows serve every head; they are passed explicitly to both sides.
    """
    if not 0 < S <= L:
        raise ValueError("need 0 < S <= L")
    rng = np.random.default_rng(seed + 104729)
    return np.sort(rng.choice(L, size=S, replace=False)).astype(np.int32)


def round_bf16_to_f64(x: torch.Tensor) -> np.ndarray:
    """Exact fp64 copy of a (bf16 or fp32) tensor for the oracle."""
    return x.detach().to("cpu", torch.float64).numpy()

