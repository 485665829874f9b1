"""Seeded synthetic inputs for the causal long convolution.

This module only draws random numbers and shapes them into the workloads the
pages' method is exercised on; it holds none of the convolution's arithmetic.
Both the CUDA path (through tests and bench.py) and the CPU oracle consume the
arrays it returns, so it imports neither of them.

Recipe (numpy ``default_rng(seed)``, PCG64; float32 normals; draw order u, v,
w, alpha, kernel normals, D):

* ``hyena_b8_h768_n4096`` etc. follow the five named workloads: the decaying
  filters k[h,t] = N(0,1) exp(-alpha t) imitate the smooth long filters that
  "Simple Hardware-Efficient Long Convolutions for Sequence Modeling"
  (abstract) finds necessary; bf16 tensors are drawn as fp32 normals and then
  rounded to nearest-even bf16, so every consumer sees the same bf16 values.
* The 2-D kernel is a Gaussian-windowed normal field anchored at (0,0).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to nearest-even bf16, returned as exactly-equal fp32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    # round-to-nearest-even on the low 16 bits; NaN/Inf are not produced here
    lsb = (bits >> 16) & 1
    bits = (bits + 0x7FFF + lsb) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32)


@dataclass
class Workload1D:
    name: str
    B: int
    H: int
    N: int
    dtype: str
    gated: bool
    u: np.ndarray                      # [B,H,N] float32 holding dtype values
    k: np.ndarray                      # [H,L] float32
    D: Optional[np.ndarray] = None     # [H] float32 or None
    v: Optional[np.ndarray] = None     # [B,H,N] (gated)
    w: Optional[np.ndarray] = None     # [B,H,N] (gated)
    seed: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def L(self) -> int:
        return int(self.k.shape[1])

    def io_bytes(self) -> int:
        """Bytes of u, v, w and y (the algorithmic traffic of one forward)."""
        esz = 4 if self.dtype == F32 else 2
        n_in = 3 if self.gated else 1
        return (n_in + 1) * self.B * self.H * self.N * esz


@dataclass
class Workload2D:
    name: str
    B: int
    C: int
    Hs: int
    Ws: int
    dtype: str
    u: np.ndarray                      # [B,C,Hs,Ws] float32 holding dtype values
    k: np.ndarray                      # [C,Kh,Kw] float32
    seed: int = 0
    meta: dict = field(default_factory=dict)

    def io_bytes(self) -> int:
        esz = 4 if self.dtype == F32 else 2
        return 2 * self.B * self.C * self.Hs * self.Ws * esz


def _normals(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def make_1d(B, H, N, dtype=F32, gated=False, seed=0, L=None, kernel="decay",
            alpha=None, with_D=True, name=None) -> Workload1D:
    """Draw one 1-D workload.

    kernel: "decay" -> k[h,t] = N(0,1) exp(-alpha_h t), alpha_h ~ U(1e-4, 1e-2)
            unless ``alpha`` fixes it; "pr1" -> N(0,1) exp(-0.005 t)/sqrt(N);
            "normal" -> plain N(0,1).
    """
    L = N if L is None else L
    rng = np.random.default_rng(seed)
    u = _normals(rng, (B, H, N))
    v = w = None
    if gated:
        v = _normals(rng, (B, H, N))
        w = _normals(rng, (B, H, N))
    t = np.arange(L, dtype=np.float64)
    if kernel == "decay":
        if alpha is None:
            a = rng.uniform(1e-4, 1e-2, size=H)
        else:
            a = np.full(H, float(alpha))
        kn = _normals(rng, (H, L)).astype(np.float64)
        k = kn * np.exp(-a[:, None] * t[None, :])
    elif kernel == "pr1":
        kn = _normals(rng, (H, L)).astype(np.float64)
        k = kn * np.exp(-0.005 * t)[None, :] / np.sqrt(N)
    elif kernel == "normal":
        k = _normals(rng, (H, L)).astype(np.float64)
    else:
        raise ValueError(f"unknown kernel recipe {kernel!r}")
    k = k.astype(np.float32)
    D = _normals(rng, (H,)) if with_D else None
    if dtype == BF16:
        u = round_bf16(u)
        if gated:
            v = round_bf16(v)
            w = round_bf16(w)
    elif dtype != F32:
        raise ValueError(dtype)
    name = name or f"conv1d_b{B}_h{H}_n{N}_{dtype}{'_gated' if gated else ''}"
    return Workload1D(name, B, H, N, dtype, gated, u, k, D, v, w, seed)


def make_2d(B, C, Hs, Ws, dtype=BF16, seed=0, Kh=None, Kw=None, sigma=64.0,
            name=None) -> Workload2D:
    """Draw one 2-D workload: u ~ N(0,1); k[c,p,q] = N(0,1) exp(-(p^2+q^2)/(2 sigma^2))."""
    Kh = Hs if Kh is None else Kh
    Kw = Ws if Kw is None else Kw
    rng = np.random.default_rng(seed)
    u = _normals(rng, (B, C, Hs, Ws))
    p = np.arange(Kh, dtype=np.float64)[:, None]
    q = np.arange(Kw, dtype=np.float64)[None, :]
    win = np.exp(-(p * p + q * q) / (2.0 * sigma * sigma))
    k = (_normals(rng, (C, Kh, Kw)).astype(np.float64) * win[None]).astype(np.float32)
    if dtype == BF16:
        u = round_bf16(u)
    elif dtype != F32:
        raise ValueError(dtype)
    name = name or f"conv2d_b{B}_c{C}_{Hs}x{Ws}_{dtype}"
    return Workload2D(name, B, C, Hs, Ws, dtype, u, k, seed)


# The five named workloads.  Seeds: the first is given as 0; the others take
# their position in the list.
CONFIGS = {
    "pr1_b1_h4_n1024_f32": dict(kind="1d", B=1, H=4, N=1024, dtype=F32, gated=False,
                                kernel="pr1", with_D=True, seed=0),
    "hyena_b8_h768_n4096_bf16": dict(kind="1d", B=8, H=768, N=4096, dtype=BF16, gated=False,
                                     kernel="decay", with_D=True, seed=1),
    "gated_b4_h1024_n16384_bf16": dict(kind="1d", B=4, H=1024, N=16384, dtype=BF16, gated=True,
                                       kernel="decay", with_D=False, seed=2),
    "long_b2_h64_n1048576_f32": dict(kind="1d", B=2, H=64, N=1 << 20, dtype=F32, gated=False,
                                     kernel="decay", alpha=1e-5, with_D=True, seed=3),
    "conv2d_b4_c256_256x256_bf16": dict(kind="2d", B=4, C=256, Hs=256, Ws=256, dtype=BF16,
                                        sigma=64.0, seed=4),
}
CONFIG_ORDER = list(CONFIGS)


def make_config(name: str):
    """Draw one of the named workloads (full size)."""
    c = dict(CONFIGS[name])
    kind = c.pop("kind")
    if kind == "1d":
        return make_1d(name=name, **c)
    return make_2d(name=name, **c)


def sample_points_1d(B, H, N, n_per_row, seed=0):
    """Seeded output positions for sampled parity: every row, the edge times
    {0, 1, N/2-1, N/2, N-1} and the powers of two below N, plus n_per_row
    uniform draws on top of that fixed set."""
    rng = np.random.default_rng(1_000_003 + seed)
    fixed = sorted({0, 1, max(N // 2 - 1, 0), N // 2, N - 1} |
                   {1 << i for i in range(N.bit_length()) if (1 << i) < N})
    fixed = [t for t in fixed if 0 <= t < N]
    bs, hs, ts = [], [], []
    for b in range(B):
        for h in range(H):
            extra = rng.integers(0, N, size=max(int(n_per_row), 0))
            tt = np.concatenate([np.asarray(fixed, dtype=np.int64), extra.astype(np.int64)])
            bs.append(np.full(tt.size, b, np.int64))
            hs.append(np.full(tt.size, h, np.int64))
            ts.append(tt)
    return np.concatenate(bs), np.concatenate(hs), np.concatenate(ts)


def sample_points_2d(B, C, Hs, Ws, n, seed=0):
    """Seeded pixel sample: the four corners of every (b,c) image the draw
    touches, the far corner, plus uniform draws, n in total (at least 5)."""
    rng = np.random.default_rng(2_000_003 + seed)
    corners = [(0, 0), (0, Ws - 1), (Hs - 1, 0), (Hs - 1, Ws - 1), (Hs // 2, Ws // 2)]
    m = max(n - len(corners), 0)
    b = rng.integers(0, B, size=n)
    c = rng.integers(0, C, size=n)
    i = np.concatenate([np.array([p for p, _ in corners]), rng.integers(0, Hs, size=m)])[:n]
    j = np.concatenate([np.array([q for _, q in corners]), rng.integers(0, Ws, size=m)])[:n]
    return (b.astype(np.int64), c.astype(np.int64), i.astype(np.int64), j.astype(np.int64))
