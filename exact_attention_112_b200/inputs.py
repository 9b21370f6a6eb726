"""Seeded synthetic inputs for the attention workloads.

This module holds no attention arithmetic: it only draws random tensors, rounds
them to the 16-bit storage type and picks row samples.  Both the CUDA path and
the float64 oracle are fed from it, so the two always see identical values.

Workloads (Llama-3-8B layer shapes from the FlashAttention case-study slides,
nmj0.github.io, "The same computation at real size": d = 4096, h = 32,
d_k = 128, n = 8192; the 32k-context anecdote of the lastdictionary.com
"FlashAttention" entry sets the top of the sequence sweep):

  tiny    B=1  H=1  N=256   D=64  fp16  non-causal                 N(0,1)
  llama   B=1  H=32 N=8192  D=128 fp16 and bf16, causal            N(0,1)
  sweep   H=16 D=128 bf16, N in 512..32768, B = max(1, 16384 // N),
          causal and non-causal                                    N(0,1)
  stress  B=16 H=16 N=2048  D=64  bf16 non-causal, Q,K ~ N(0, 8^2),
          V ~ U(-1,1), -inf key bias on 205 (= round(0.1 * 2048)) seeded
          key columns per batch
  bwd     B=2  H=32 N=4096  D=128 bf16 causal, Q,K,V,dO ~ N(0,1)
  decode  B=1  H=8  Nq=256 Nk=65536 D=128 bf16 non-causal (split-KV)  N(0,1)

There is no public dataset behind these: i.i.d. activations of the named shapes
stand in for a real layer's Q/K/V (no trained weights are needed or used).
"""
from __future__ import annotations

import math

import numpy as np
import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn}

SWEEP_N = (512, 1024, 2048, 4096, 8192, 16384, 32768)


def workload(name: str, **over) -> dict:
    """Shape/distribution description of a named workload (plus overrides)."""
    base = {
        "tiny": dict(B=1, H=1, Nq=256, Nk=256, D=64, dtype="f16", causal=False,
                     qk_std=1.0, v_dist="normal", bias_frac=0.0, seed=1000),
        "llama": dict(B=1, H=32, Nq=8192, Nk=8192, D=128, dtype="bf16",
                      causal=True, qk_std=1.0, v_dist="normal", bias_frac=0.0,
                      seed=1001),
        "sweep": dict(B=2, H=16, Nq=8192, Nk=8192, D=128, dtype="bf16",
                      causal=True, qk_std=1.0, v_dist="normal", bias_frac=0.0,
                      seed=1002),
        "stress": dict(B=16, H=16, Nq=2048, Nk=2048, D=64, dtype="bf16",
                       causal=False, qk_std=8.0, v_dist="uniform", bias_frac=0.1,
                       seed=1003),
        "bwd": dict(B=2, H=32, Nq=4096, Nk=4096, D=128, dtype="bf16",
                    causal=True, qk_std=1.0, v_dist="normal", bias_frac=0.0,
                    seed=1004),
        # few queries against a long key sequence (the shape the split-KV
        # forward is for): 256 query rows of 8 heads over 65536 keys
        "decode": dict(B=1, H=8, Nq=256, Nk=65536, D=128, dtype="bf16",
                       causal=False, qk_std=1.0, v_dist="normal", bias_frac=0.0,
                       seed=1005),
    }[name]
    cfg = dict(base)
    cfg.update(over)
    if name == "sweep" and "N" in over:
        n = over["N"]
        cfg.update(Nq=n, Nk=n, B=max(1, 16384 // n))
        cfg.pop("N", None)
    cfg["name"] = name
    return cfg


def _randn(shape, gen, std):
    return torch.randn(shape, generator=gen, dtype=torch.float32) * std


def make_inputs(B, H, Nq, Nk, D, dtype="bf16", seed=0, qk_std=1.0,
                v_dist="normal", bias_frac=0.0, with_dO=False, **_ignored):
    """Draw Q, K, V (and dO) on the host, rounded to the storage dtype.

    Returns a dict of CPU tensors: q [B,H,Nq,D], k/v [B,H,Nk,D] (16-bit, or
    8-bit E4M3 for dtype "e4m3"), optional do [B,H,Nq,D] and key_bias [B,Nk]
    float32 (or None).  The rounding (round-to-nearest-even, torch's cast)
    happens here, once, so the oracle receives exactly the values the kernels
    read.  E4M3 draws are far inside its range (|x| <= 448), so the cast never
    saturates.
    """
    tdt = DTYPES[dtype]
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    q = _randn((B, H, Nq, D), gen, qk_std).to(tdt)
    k = _randn((B, H, Nk, D), gen, qk_std).to(tdt)
    if v_dist == "uniform":
        v = (torch.rand((B, H, Nk, D), generator=gen) * 2.0 - 1.0).to(tdt)
    else:
        v = _randn((B, H, Nk, D), gen, 1.0).to(tdt)
    out = {"q": q, "k": k, "v": v, "key_bias": None, "do": None}
    if with_dO:
        out["do"] = _randn((B, H, Nq, D), gen, 1.0).to(tdt)
    if bias_frac > 0:
        out["key_bias"] = make_key_bias(B, Nk, bias_frac, seed + 7919)
    return out


def make_key_bias(B, Nk, frac, seed):
    """Additive key bias [B, Nk] float32: -inf on round(frac * Nk) distinct,
    seeded key columns per batch (shared by all heads and queries), 0 elsewhere."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    n_masked = int(round(frac * Nk))
    bias = torch.zeros((B, Nk), dtype=torch.float32)
    for b in range(B):
        cols = torch.randperm(Nk, generator=gen)[:n_masked]
        bias[b, cols] = -math.inf
    return bias


def make_mask(kind, Nq, Nk, seed, planes=(1, 1), ldm=None):
    """General additive mask, float32 [Bm, Hm, Nq, ldm] (columns [Nk, ldm) are
    padding, filled with NaN so that reading them would show; the mask proper
    is the [..., :Nk] view, which is returned).  Kinds:
      random    -inf on a seeded 10% of entries, elsewhere N(0, 0.5^2) values;
                every row keeps its first visible key finite, so no row is
                fully hidden
      window    sliding window: key j visible to query i iff
                i' - 255 <= j <= i' with i' = i + Nk - Nq (bottom-right)
      document  packed documents of seeded lengths 1..max(1, Nk // 3):
                causal inside a document, hidden across documents (query
                rows are aligned to the keys bottom-right)
      rows      like random, and every 7th query row entirely -inf (rows
                that see no key: O = 0, LSE = -inf)
    """
    Bm, Hm = planes
    if ldm is None:
        ldm = max(4, (Nk + 3) // 4 * 4)
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    buf = torch.full((Bm, Hm, Nq, ldm), float("nan"), dtype=torch.float32)
    m = buf[..., :Nk]
    i = torch.arange(Nq).view(-1, 1) + (Nk - Nq)
    j = torch.arange(Nk).view(1, -1)
    if kind in ("random", "rows"):
        vals = torch.randn((Bm, Hm, Nq, Nk), generator=gen) * 0.5
        hide = torch.rand((Bm, Hm, Nq, Nk), generator=gen) < 0.1
        if Nk > 0:
            hide[..., 0] = False
        vals[hide] = -math.inf
        if kind == "rows":
            vals[:, :, ::7, :] = -math.inf
        m.copy_(vals)
    elif kind == "window":
        vis = (j <= i) & (j >= i - 255)
        m.copy_(torch.where(vis, 0.0, -math.inf).expand(Bm, Hm, Nq, Nk))
    elif kind == "document":
        doc = torch.empty(Nk, dtype=torch.long)
        start, d = 0, 0
        while start < Nk:
            ln = int(torch.randint(1, max(2, Nk // 3 + 1), (1,), generator=gen))
            doc[start:start + ln] = d
            start += ln
            d += 1
        qdoc = doc[torch.clamp(i.view(-1), 0, max(Nk - 1, 0))].view(-1, 1) if Nk > 0 else None
        vis = (j <= i) & (qdoc == doc.view(1, -1)) if Nk > 0 else torch.zeros((Nq, 0), dtype=torch.bool)
        m.copy_(torch.where(vis, 0.0, -math.inf).expand(Bm, Hm, Nq, Nk))
    else:
        raise ValueError(kind)
    return m


def sample_rows(N, n_random=512, tile=128, seed=0):
    """Query rows checked at full size: every tile-boundary row (0, 127, 128,
    255, ..., N-1) plus n_random seeded rows, sorted and unique."""
    rows = set()
    for t in range(0, N, tile):
        rows.add(t)
        rows.add(min(t + tile - 1, N - 1))
    rows.add(N - 1)
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, N, size=min(n_random, N)).tolist())
    return np.array(sorted(rows), dtype=np.int64)


def to_f64(t):
    """Host float64 copy of a (16-bit or float32) tensor, for the oracle."""
    if t is None:
        return None
    return t.detach().to("cpu", torch.float64).numpy()
