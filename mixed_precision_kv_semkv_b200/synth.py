"""Seeded synthetic inputs for the SemKV hot path.

This module is the only thing the CUDA path and the CPU oracle share.  It holds none of the
method's arithmetic: it draws K, V, queries and per-token importance scores with the shapes and
value distributions of the five workloads below, and nothing else.

Workloads (shapes as in the Llama-3.1-8B / Mistral-7B attention layers; head_dim 128):

  tiny         B1 H1 Hq4 T4096; K,V ~ N(0,1) fp16 with 4 K channels x8; scores ~ Zipf(1.1);
               G128, L 8/5, p 0.5
  llama8b_1L   B1 H8 Hq32 T32768 (one layer); K,V ~ N(0,1) * sigma_c, sigma_c ~ LogNormal(0,0.5)
               per (K|V, head, channel); scores = softmax mass of 64 N(0,1) queries against K;
               G64, L 8/5, p 0.25
  llama8b_32L  B1 32 layers H8 Hq32 T131072; per layer as llama8b_1L (seed = layer);
               G128, L 6/5, p 0.5
  gen          B16 32 layers H8 Hq32, 32768-token prefill then 256 generated tokens; data as
               llama8b_1L; G64, L 8/5, p 0.25
  mistral_sweep B8 32 layers H8 Hq32 T32768; K,V ~ Student-t(5) * LogNormal(0,0.7) per channel;
               scores ~ Zipf(1.0); (L_hi, L_lo) in {(6,5), (8,6), (16,8)}, p in {0,.25,.5,.75,1},
               G in {32,64,128}

Zipf(a) scores: a random permutation r_t of 1..T, score_t = r_t^-a normalised to sum 1 (no ties).
CPU draws use numpy's Philox generator; large GPU workloads use torch's CUDA Philox generator.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

D_HEAD = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Hq: int
    T: int
    G: int
    L_hi: int
    L_lo: int
    p: float
    layers: int = 1
    steps: int = 0          # generated tokens after the prefill (gen workload)
    kv_dist: str = "lognormal"  # "outlier" | "lognormal" | "student"
    sigma_c: float = 0.5
    score: str = "softmax"  # "zipf" | "softmax"
    zipf_a: float = 1.1
    D: int = D_HEAD


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 4, 4096, 128, 8, 5, 0.5, kv_dist="outlier", score="zipf", zipf_a=1.1),
    "llama8b_1L": Workload("llama8b_1L", 1, 8, 32, 32768, 64, 8, 5, 0.25),
    "llama8b_32L": Workload("llama8b_32L", 1, 8, 32, 131072, 128, 6, 5, 0.5, layers=32),
    "gen": Workload("gen", 16, 8, 32, 32768, 64, 8, 5, 0.25, layers=32, steps=256),
    "mistral_sweep": Workload("mistral_sweep", 8, 8, 32, 32768, 128, 6, 5, 0.5, layers=32,
                              kv_dist="student", sigma_c=0.7, score="zipf", zipf_a=1.0),
}

SWEEP_PAIRS = [(6, 5), (8, 6), (16, 8)]
SWEEP_P = [0.0, 0.25, 0.5, 0.75, 1.0]
SWEEP_G = [32, 64, 128]


def sm_scale(D: int = D_HEAD) -> float:
    return 1.0 / math.sqrt(D)


def _rng(seed: int, stream: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[seed & 0xFFFFFFFFFFFFFFFF, stream]))


# ---------------------------------------------------------------- CPU (numpy) draws

def kv_cpu(w: Workload, seed: int, layer: int = 0, T: int | None = None, B: int | None = None):
    """K, V as fp16 numpy arrays [B][H][T][D]."""
    T = w.T if T is None else T
    B = w.B if B is None else B
    r = _rng(seed * 1000 + layer, 1)
    shape = (B, w.H, T, w.D)
    if w.kv_dist == "outlier":
        K = r.standard_normal(shape)
        V = r.standard_normal(shape)
        ch = r.choice(w.D, size=4, replace=False)
        K[..., ch] *= 8.0
    elif w.kv_dist == "lognormal":
        sk = r.lognormal(0.0, w.sigma_c, size=(1, w.H, 1, w.D))
        sv = r.lognormal(0.0, w.sigma_c, size=(1, w.H, 1, w.D))
        K = r.standard_normal(shape) * sk
        V = r.standard_normal(shape) * sv
    elif w.kv_dist == "student":
        sk = r.lognormal(0.0, w.sigma_c, size=(1, w.H, 1, w.D))
        sv = r.lognormal(0.0, w.sigma_c, size=(1, w.H, 1, w.D))
        K = r.standard_t(5, size=shape) * sk
        V = r.standard_t(5, size=shape) * sv
    else:
        raise ValueError(w.kv_dist)
    return K.astype(np.float16), V.astype(np.float16)


def q_cpu(w: Workload, seed: int, layer: int = 0, B: int | None = None):
    """Decode queries fp16 [B][Hq][D]."""
    B = w.B if B is None else B
    r = _rng(seed * 1000 + layer, 2)
    return r.standard_normal((B, w.Hq, w.D)).astype(np.float16)


def zipf_scores_cpu(a: float, T: int, units: int, seed: int) -> np.ndarray:
    r = _rng(seed, 3)
    out = np.empty((units, T), np.float32)
    base = np.arange(1, T + 1, dtype=np.float64) ** (-a)
    for u in range(units):
        perm = r.permutation(T)
        s = base[perm]
        out[u] = (s / s.sum()).astype(np.float32)
    return out


def softmax_mass_scores_cpu(K16: np.ndarray, nq: int, seed: int, scale: float) -> np.ndarray:
    """scores[b,h,t] = sum over nq random N(0,1) queries of softmax_t(scale * q.k_t), in fp64."""
    B, H, T, D = K16.shape
    r = _rng(seed, 4)
    out = np.empty((B, H, T), np.float32)
    for b in range(B):
        for h in range(H):
            k = K16[b, h].astype(np.float64)
            q = r.standard_normal((nq, D))
            lg = scale * (q @ k.T)
            lg -= lg.max(axis=1, keepdims=True)
            e = np.exp(lg)
            e /= e.sum(axis=1, keepdims=True)
            out[b, h] = e.sum(axis=0).astype(np.float32)
    return out


def scores_cpu(w: Workload, K16: np.ndarray, seed: int, layer: int = 0) -> np.ndarray:
    """Per-token importance scores fp32 [B][H][T]."""
    B, H, T, _ = K16.shape
    if w.score == "zipf":
        return zipf_scores_cpu(w.zipf_a, T, B * H, seed * 1000 + layer).reshape(B, H, T)
    return softmax_mass_scores_cpu(K16, 64, seed * 1000 + layer, sm_scale(w.D))


def layer_cpu(w: Workload, seed: int, layer: int = 0, T: int | None = None, B: int | None = None):
    """One layer's inputs on the CPU: dict of K, V (fp16 [B][H][T][D]), scores, q."""
    K, V = kv_cpu(w, seed, layer, T=T, B=B)
    S = scores_cpu(w, K, seed, layer)
    q = q_cpu(w, seed, layer, B=K.shape[0])
    return {"K": K, "V": V, "scores": S, "q": q}


def gen_steps_cpu(w: Workload, K16: np.ndarray, seed: int, layer: int, steps: int):
    """Generated tokens: new k, v fp16 [steps][B][H][D], their scores fp32 [steps][B][H], and the
    decode queries fp16 [steps][B][Hq][D].

    A new token's score is its softmax mass against the same 64 queries that scored the prefill,
    normalised with the prefill's per-query max and sum, so that it is comparable with the prefill
    scores.
    """
    B, H, T, D = K16.shape
    r = _rng(seed * 1000 + layer, 5)
    shape = (steps, B, H, D)
    if w.kv_dist in ("lognormal", "student"):
        r1 = _rng(seed * 1000 + layer, 1)  # the prefill's per-channel scales, drawn again
        sk = r1.lognormal(0.0, w.sigma_c, size=(1, H, 1, D)).reshape(1, 1, H, D)
        sv = r1.lognormal(0.0, w.sigma_c, size=(1, H, 1, D)).reshape(1, 1, H, D)
        kn = r.standard_normal(shape) * sk
        vn = r.standard_normal(shape) * sv
    else:
        kn = r.standard_normal(shape)
        vn = r.standard_normal(shape)
    kn = kn.astype(np.float16)
    vn = vn.astype(np.float16)
    qs = r.standard_normal((steps, B, w.Hq, D)).astype(np.float16)
    sc = np.empty((steps, B, H), np.float32)
    r2 = _rng(seed * 1000 + layer, 4)  # the prefill's scoring queries
    scale = sm_scale(D)
    for b in range(B):
        for h in range(H):
            k = K16[b, h].astype(np.float64)
            q = r2.standard_normal((64, D))
            lg = scale * (q @ k.T)
            m = lg.max(axis=1)
            z = np.exp(lg - m[:, None]).sum(axis=1)
            ln = scale * (kn[:, b, h].astype(np.float64) @ q.T)  # [steps][64]
            sc[:, b, h] = (np.exp(ln - m[None, :]) / z[None, :]).sum(axis=1).astype(np.float32)
    return {"k": kn, "v": vn, "scores": sc, "q": qs}


# ---------------------------------------------------------------- GPU (torch) draws

def layer_gpu(w: Workload, seed: int, layer: int = 0, device: str = "cuda", T: int | None = None,
              B: int | None = None):
    """One layer's inputs drawn on the GPU with torch's Philox generator (large workloads)."""
    import torch

    T = w.T if T is None else T
    B = w.B if B is None else B
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + layer)
    shape = (B, w.H, T, w.D)
    if w.kv_dist == "student":
        sk = torch.empty((1, w.H, 1, w.D), device=device).log_normal_(0.0, w.sigma_c, generator=g)
        sv = torch.empty((1, w.H, 1, w.D), device=device).log_normal_(0.0, w.sigma_c, generator=g)

        def student5():
            chi2 = torch.zeros(shape, device=device)
            for _ in range(5):  # chi-square with 5 degrees of freedom
                chi2 += torch.randn(shape, device=device, generator=g) ** 2
            return torch.randn(shape, device=device, generator=g) / torch.sqrt(chi2 / 5.0)

        K = student5() * sk
        V = student5() * sv
    elif w.kv_dist == "lognormal":
        sk = torch.empty((1, w.H, 1, w.D), device=device).log_normal_(0.0, w.sigma_c, generator=g)
        sv = torch.empty((1, w.H, 1, w.D), device=device).log_normal_(0.0, w.sigma_c, generator=g)
        K = torch.randn(shape, device=device, generator=g) * sk
        V = torch.randn(shape, device=device, generator=g) * sv
    else:
        K = torch.randn(shape, device=device, generator=g)
        V = torch.randn(shape, device=device, generator=g)
        ch = torch.randperm(w.D, device=device, generator=g)[:4]
        K[..., ch] *= 8.0
    K = K.to(torch.float16)
    V = V.to(torch.float16)
    q = torch.randn((B, w.Hq, w.D), device=device, generator=g).to(torch.float16)
    if w.score == "zipf":
        base = torch.arange(1, T + 1, device=device, dtype=torch.float64) ** (-w.zipf_a)
        S = torch.empty((B, w.H, T), device=device, dtype=torch.float32)
        for u in range(B * w.H):
            perm = torch.randperm(T, device=device, generator=g)
            s = base[perm]
            S.view(-1, T)[u] = (s / s.sum()).to(torch.float32)
    else:
        S = torch.zeros((B, w.H, T), device=device, dtype=torch.float32)
        qs = torch.randn((B, w.H, 64, w.D), device=device, generator=g)
        for b in range(B):
            lg = torch.einsum("hqd,htd->hqt", qs[b], K[b].float()) * sm_scale(w.D)
            S[b] = torch.softmax(lg, dim=-1).sum(dim=1)
    return {"K": K, "V": V, "scores": S, "q": q}


def prefill_channel_scales_gpu(w: Workload, seed: int, layer: int = 0, device: str = "cuda"):
    """The per-channel scales (sigma_K, sigma_V), each [1][H][1][D], that layer_gpu draws first from
    the layer's generator (None, None for the outlier workload, which has none)."""
    import torch

    if w.kv_dist not in ("lognormal", "student"):
        return None, None
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + layer)
    sk = torch.empty((1, w.H, 1, w.D), device=device).log_normal_(0.0, w.sigma_c, generator=g)
    sv = torch.empty((1, w.H, 1, w.D), device=device).log_normal_(0.0, w.sigma_c, generator=g)
    return sk, sv


def gen_steps_gpu(w: Workload, K16, seed: int, layer: int, steps: int, device: str = "cuda"):
    """Generated tokens on the GPU: new k, v fp16 [steps][B][H][D] with the prefill's per-channel
    scales, their scores fp32 [steps][B][H] (softmax mass against 64 scoring queries, normalised by
    those queries' prefill max and sum), and decode queries fp16 [steps][B][Hq][D]."""
    import torch

    B, H, T, D = K16.shape
    sk, sv = prefill_channel_scales_gpu(w, seed, layer, device)
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + layer + 500000)
    if sk is None:
        kn = torch.randn((steps, B, H, D), device=device, generator=g).to(torch.float16)
        vn = torch.randn((steps, B, H, D), device=device, generator=g).to(torch.float16)
    else:
        sk = sk.reshape(1, 1, H, D)
        sv = sv.reshape(1, 1, H, D)
        kn = (torch.randn((steps, B, H, D), device=device, generator=g) * sk).to(torch.float16)
        vn = (torch.randn((steps, B, H, D), device=device, generator=g) * sv).to(torch.float16)
    qs = torch.randn((steps, B, w.Hq, D), device=device, generator=g).to(torch.float16)
    qsc = torch.randn((B, H, 64, D), device=device, generator=g)
    sc = torch.empty((steps, B, H), device=device, dtype=torch.float32)
    scale = sm_scale(D)
    for b in range(B):
        lg = torch.einsum("hqd,htd->hqt", qsc[b], K16[b].float()) * scale  # [H][64][T]
        m = lg.amax(dim=-1)                                                 # [H][64]
        z = torch.exp(lg - m[..., None]).sum(dim=-1)                        # [H][64]
        ln = torch.einsum("shd,hqd->shq", kn[:, b].float(), qsc[b]) * scale  # [steps][H][64]
        sc[:, b] = (torch.exp(ln - m[None]) / z[None]).sum(dim=-1)
    return {"k": kn, "v": vn, "scores": sc, "q": qs}
