"""Seeded synthetic inputs for the XAttention prefill path.

This module only draws random tensors and plants structure in them. It holds
none of the method's arithmetic, so both the CUDA path and the CPU oracle can
read the same inputs from it.

The paper's workloads are real models on RULER / LongBench / Video-MME / VBench
("XAttention: Block Sparse Attention with Antidiagonal Scoring", §3.1). We
have neither the weights nor the datasets. These generators stand in for them
with tensors of the models' attention shapes:

* ``tiny``: 1 head, L=1024, d=64, fp32. Vertical lines come from sink keys
  {0,1,2,3,517}, and a slash comes from keys that copy queries 64 tokens later.
* ``llama``: Llama-3.1-8B attention (32 query heads, 8 KV heads, d=128), bf16.
  Each KV group has sink keys (the first 4 tokens, key norm about x4) and
  smooth "slash bands" that make q_i . k_j large when i - j is near an offset.
* ``video``: a video-DiT layer (24 heads, MHA, d=128, 30 frames x 2560
  tokens), bf16, non-causal. Each token adds a per-frame component and a
  per-spatial-position component shared across frames.

All draws come from one ``torch.Generator`` on the CPU, in a fixed order.
Tensors are made in fp32, then rounded to the problem dtype. They are laid out
[batch, heads, L, d], contiguous.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = ["Problem", "CONFIGS", "make_problem", "SLASH_GAMMA"]

# Amplitude of the slash-band process (a free constant of the recipe). It is
# picked once, on the 256K Llama-shaped layer, to give a block density near the
# ~7 % that the paper reports at 256K. The same value is used at every length.
SLASH_GAMMA = 0.755


@dataclass
class Problem:
    """One attention layer's inputs plus the XAttention parameters."""

    name: str
    batch: int
    hq: int
    hkv: int
    L: int
    d: int
    B: int
    S: int
    causal: bool
    dtype: str            # "f32" or "bf16"
    tau: np.ndarray       # float32 [hq], per-head threshold
    Q: torch.Tensor = field(repr=False)
    K: torch.Tensor = field(repr=False)
    V: torch.Tensor = field(repr=False)
    recipe: dict = field(default_factory=dict)

    @property
    def NB(self) -> int:
        return -(-self.L // self.B)   # the last block is shorter when B does not divide L


# The five workloads. "S" is a list for the stride sweep of the video layer.
CONFIGS = {
    "c0": dict(kind="tiny", batch=1, hq=1, hkv=1, L=1024, d=64, dtype="f32",
               causal=True, B=64, S=8, tau=0.9, seed=0),
    "c1": dict(kind="llama", batch=1, hq=32, hkv=8, L=32768, d=128, dtype="bf16",
               causal=True, B=128, S=8, tau=0.9, seed=1, bands=1, band_offsets="zero"),
    "c2": dict(kind="llama", batch=1, hq=32, hkv=8, L=131072, d=128, dtype="bf16",
               causal=True, B=128, S=16, tau="choice", seed=2, bands=3,
               band_offsets="random"),
    "c3": dict(kind="llama", batch=1, hq=32, hkv=8, L=262144, d=128, dtype="bf16",
               causal=True, B=128, S=8, tau=0.9, seed=3, bands=1, band_offsets="zero"),
    "c4": dict(kind="video", batch=1, hq=24, hkv=24, L=76800, d=128, dtype="bf16",
               causal=False, B=128, S=[4, 8, 16, 64], tau=0.95, seed=4,
               frames=30, frame_tokens=2560),
}

TAU_CHOICES = (0.8, 0.85, 0.9, 0.95)


def _unit(g: torch.Generator, d: int) -> torch.Tensor:
    u = torch.randn(d, generator=g, dtype=torch.float32)
    return u / u.norm()


def _cast(x: torch.Tensor, dtype: str) -> torch.Tensor:
    return x.to(torch.float32 if dtype == "f32" else torch.bfloat16)


def _band_process(g: torch.Generator, length: int, d: int, w: int) -> torch.Tensor:
    """A smooth random process s(t), t in [0, length).

    Independent N(0, I_d) anchors sit every w/2 tokens, and s is linearly
    interpolated between them. s(i) . s(j) is large when |i - j| is well
    under w/2.
    """
    half = w // 2
    n_anchor = length // half + 2
    anchors = torch.randn(n_anchor, d, generator=g, dtype=torch.float32)
    t = torch.arange(length)
    k = t // half
    f = ((t % half).to(torch.float32) / half).unsqueeze(1)
    return anchors[k] * (1.0 - f) + anchors[k + 1] * f


def _tiny(cfg: dict, L: int, seed: int) -> tuple:
    g = torch.Generator().manual_seed(seed)
    d = cfg["d"]
    Q = torch.randn(1, 1, L, d, generator=g, dtype=torch.float32)
    K = torch.randn(1, 1, L, d, generator=g, dtype=torch.float32)
    V = torch.randn(1, 1, L, d, generator=g, dtype=torch.float32)
    u = _unit(g, d)
    # Vertical lines: sink keys share a direction with every query. The sinks
    # go in first, then the slash reads the already-shifted queries.
    sinks = [j for j in (0, 1, 2, 3, 517) if j < L]
    K[0, 0, sinks, :] += 3.0 * u
    Q[0, 0] += 0.5 * u
    # Slash band: key j copies 0.8 x query j+64, so q_i . k_{i-64} is large.
    off = 64
    if L > off:
        K[0, 0, : L - off] += 0.8 * Q[0, 0, off:]
    recipe = dict(sinks=sinks, sink_gain=3.0, query_gain=0.5, slash_offset=off,
                  slash_gain=0.8)
    return Q, K, V, recipe


def _llama(cfg: dict, L: int, hq: int, hkv: int, seed: int, gamma: float) -> tuple:
    g = torch.Generator().manual_seed(seed)
    d, batch = cfg["d"], cfg["batch"]
    dt = cfg["dtype"]
    gsz = hq // hkv
    w = 512
    nb = cfg["bands"]
    beta = math.sqrt(15.0 * d)   # |k_sink| ~ sqrt(d + beta^2) = 4 sqrt(d)
    # Per KV group: sink direction and band offsets.
    u = [_unit(g, d) for _ in range(hkv)]
    if cfg["band_offsets"] == "zero":
        offsets = [[0] * nb for _ in range(hkv)]
    else:
        offsets = [torch.randint(0, max(L // 2, 1), (nb,), generator=g).tolist()
                   for _ in range(hkv)]
    Q = torch.empty(batch, hq, L, d, dtype=torch.float32 if dt == "f32" else torch.bfloat16)
    K = torch.empty(batch, hkv, L, d, dtype=Q.dtype)
    V = torch.empty(batch, hkv, L, d, dtype=Q.dtype)
    for b in range(batch):
        for kv in range(hkv):
            q_bias = torch.zeros(L, d)
            k_bias = torch.zeros(L, d)
            for band in range(nb):
                dl = offsets[kv][band]
                s = _band_process(g, L + dl, d, w)
                q_bias += gamma * s[:L]
                k_bias += gamma * s[dl: dl + L]
            q_bias += 0.5 * u[kv]
            kk = torch.randn(L, d, generator=g, dtype=torch.float32)
            kk += k_bias
            kk[0:4] += beta * u[kv]
            K[b, kv] = _cast(kk, dt)
            V[b, kv] = _cast(torch.randn(L, d, generator=g, dtype=torch.float32), dt)
            for hh in range(gsz):
                qq = torch.randn(L, d, generator=g, dtype=torch.float32)
                qq += q_bias
                Q[b, kv * gsz + hh] = _cast(qq, dt)
    recipe = dict(sink_tokens=4, sink_beta=beta, query_gain=0.5, band_width=w,
                  gamma=gamma, band_offsets=offsets)
    return Q, K, V, recipe


def _video(cfg: dict, frames: int, frame_tokens: int, hq: int, seed: int) -> tuple:
    g = torch.Generator().manual_seed(seed)
    d, batch, dt = cfg["d"], cfg["batch"], cfg["dtype"]
    L = frames * frame_tokens
    frame_of = torch.arange(L) // frame_tokens
    pos_of = torch.arange(L) % frame_tokens
    out = []
    for _ in ("Q", "K"):
        x = torch.empty(batch, hq, L, d, dtype=torch.float32 if dt == "f32" else torch.bfloat16)
        for b in range(batch):
            for h in range(hq):
                f = torch.randn(frames, d, generator=g, dtype=torch.float32)
                p = 0.7 * torch.randn(frame_tokens, d, generator=g, dtype=torch.float32)
                xx = torch.randn(L, d, generator=g, dtype=torch.float32)
                xx += f[frame_of] + p[pos_of]
                x[b, h] = _cast(xx, dt)
        out.append(x)
    V = torch.empty_like(out[0])
    for b in range(batch):
        for h in range(hq):
            V[b, h] = _cast(torch.randn(L, d, generator=g, dtype=torch.float32), dt)
    recipe = dict(frames=frames, frame_tokens=frame_tokens, frame_sigma=1.0, pos_sigma=0.7)
    return out[0], out[1], V, recipe


def make_problem(name: str, *, L: int | None = None, hq: int | None = None,
                 hkv: int | None = None, S: int | None = None, frames: int | None = None,
                 frame_tokens: int | None = None, seed: int | None = None,
                 tau: float | None = None, gamma: float | None = None,
                 batch: int | None = None) -> Problem:
    """Build one workload by name ("c0".."c4").

    The keyword overrides shrink a workload for tests: same recipe, fewer
    tokens or heads (or more sequences: ``batch``). For "c4", S picks one stride of the sweep (default 8),
    and ``frames`` and ``frame_tokens`` set L.
    """
    cfg = dict(CONFIGS[name])
    if batch is not None:
        if cfg["kind"] == "tiny" and batch != 1:
            raise ValueError("the tiny fp32 workload has one sequence")
        cfg["batch"] = int(batch)
    seed = cfg["seed"] if seed is None else seed
    hq = cfg["hq"] if hq is None else hq
    hkv = cfg["hkv"] if hkv is None else hkv
    if cfg["kind"] == "video":
        hkv = hq
    stride = cfg["S"] if S is None else S
    if isinstance(stride, list):
        stride = 8
    if cfg["kind"] == "tiny":
        L = cfg["L"] if L is None else L
        Q, K, V, recipe = _tiny(cfg, L, seed)
    elif cfg["kind"] == "llama":
        L = cfg["L"] if L is None else L
        Q, K, V, recipe = _llama(cfg, L, hq, hkv, seed,
                                 SLASH_GAMMA if gamma is None else gamma)
    else:
        fr = cfg["frames"] if frames is None else frames
        ft = cfg["frame_tokens"] if frame_tokens is None else frame_tokens
        if L is not None and frames is None and frame_tokens is None:
            ft = cfg["frame_tokens"]
            fr = max(L // ft, 1)
            if fr * ft != L:
                ft, fr = L, 1
        L = fr * ft
        Q, K, V, recipe = _video(cfg, fr, ft, hq, seed)
    if tau is not None:
        taus = np.full(hq, tau, dtype=np.float32)
    elif cfg["tau"] == "choice":
        g = torch.Generator().manual_seed(seed)
        pick = torch.randint(0, len(TAU_CHOICES), (hq,), generator=g)
        taus = np.array([TAU_CHOICES[i] for i in pick.tolist()], dtype=np.float32)
    else:
        taus = np.full(hq, cfg["tau"], dtype=np.float32)
    return Problem(name=name, batch=cfg["batch"], hq=hq, hkv=hkv, L=L, d=cfg["d"],
                   B=cfg["B"], S=stride, causal=cfg["causal"], dtype=cfg["dtype"],
                   tau=taus, Q=Q, K=K, V=V, recipe=recipe)
