"""Seeded synthetic inputs for the MoE-layer forward workloads.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark. It draws random numbers and rounds them to the storage precision of
each workload; it performs none of the layer's arithmetic (no projection, no
scoring, no selection, no balancing). Every array is returned as numpy float32
(values already representable in the storage dtype) or int32.

Workload shapes follow the five layer configurations studied on the pages:
  tiny       Switch layer, fp32          m=1024  d=64   n=8   k=1 softmax d_ff=256  capacity 160
  switch     Switch-Base-like, bf16      m=8192  d=768  n=128 k=1 softmax d_ff=3072 capacity 80
  lossfree   Loss-Free sigmoid top-6     m=16384 d=2048 n=64  k=6 sigmoid d_ff=1408 no drop
  qb         balanced assignment scores  m=65536 n=256 k=8 (routing only)
  global     global-batch top-2, bf16    16 x 4096 tokens d=4096 n=64 k=2 d_ff=4096 capacity 256/micro-batch

Draw order per workload (one numpy Generator seeded with `seed`):
  layer workloads: x, w_r, w1, b1, w2, b2 (the 'global' workload draws its
  cluster centres and memberships first); the Loss-Free bias b comes from a
  second stream seeded with [seed, 1], so router-only callers get the same b.
  qb: the N(0,1) score matrix, then the per-expert skew c_j.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); return float32."""
    a = np.array(a, dtype=np.float32, copy=True, order="C")
    if not np.isfinite(a).all():
        raise ValueError("round_to_bf16 expects finite values")
    bits = a.view(np.uint32)
    lsb = (bits >> np.uint32(16)) & np.uint32(1)
    bits += np.uint32(0x7FFF)
    bits += lsb
    bits &= np.uint32(0xFFFF0000)
    return a


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


@dataclass
class LayerConfig:
    name: str
    m: int
    d: int
    n: int
    k: int
    d_ff: int
    score_fn: str            # "softmax" or "sigmoid"
    dtype: str               # "fp32" or "bf16"
    capacity: int            # per expert per segment; >= seg_len*k means no drop
    seg_len: int             # tokens per micro-batch segment (== m for one segment)
    wr_std: float            # router weight standard deviation
    renorm_topk: int = 0     # k>=2 softmax: gate = softmax over the selected logits
    lossfree_bias: float = 0.0   # half-width of U(-w, w) ranking bias, 0 = none
    clusters: int = 0        # >0: tokens drawn from Gaussian clusters per segment
    alpha: float = 1e-2
    gamma: float = 1e-3
    residual: int = 0
    extra: dict = field(default_factory=dict)


def capacity_from_factor(cf: float, m_seg: int, k: int, n: int) -> int:
    """Expert capacity = (dispatched copies per segment / experts) x capacity factor, rounded up."""
    return int(math.ceil(cf * k * m_seg / n - 1e-9))


CONFIGS = {
    "tiny": LayerConfig("tiny", m=1024, d=64, n=8, k=1, d_ff=256, score_fn="softmax", dtype="fp32",
                        capacity=capacity_from_factor(1.25, 1024, 1, 8), seg_len=1024, wr_std=0.02),
    "switch": LayerConfig("switch", m=8192, d=768, n=128, k=1, d_ff=3072, score_fn="softmax", dtype="bf16",
                          capacity=capacity_from_factor(1.25, 8192, 1, 128), seg_len=8192,
                          wr_std=0.1 / math.sqrt(768)),
    "lossfree": LayerConfig("lossfree", m=16384, d=2048, n=64, k=6, d_ff=1408, score_fn="sigmoid", dtype="bf16",
                            capacity=16384 * 6, seg_len=16384, wr_std=1.0 / math.sqrt(2048),
                            lossfree_bias=0.05),
    "global": LayerConfig("global", m=65536, d=4096, n=64, k=2, d_ff=4096, score_fn="softmax", dtype="bf16",
                          capacity=capacity_from_factor(2.0, 4096, 2, 64), seg_len=4096,
                          wr_std=1.0 / math.sqrt(4096), renorm_topk=1, clusters=8),
}

QB_CONFIG = dict(m=65536, n=256, k=8, skew_std=1.5)


def scaled_config(base: str, **over) -> LayerConfig:
    """A copy of a named configuration with some fields replaced (smaller parity cases)."""
    c = CONFIGS[base]
    kw = dict(c.__dict__)
    kw.update(over)
    kw["extra"] = dict(c.extra)
    return LayerConfig(**kw)


def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    return round_to_bf16(a) if dtype == "bf16" else np.ascontiguousarray(a, dtype=np.float32)


def _draw_tokens(rng: np.random.Generator, cfg: LayerConfig) -> np.ndarray:
    """x [m,d]: N(0,1) tokens, or (clusters > 0) centre mu_q ~ N(0,I) plus N(0, 0.5^2 I) noise,
    where micro-batch s takes 90% of its tokens from cluster s mod q and 10% from a uniform cluster."""
    m, d = cfg.m, cfg.d
    if cfg.clusters:
        q = cfg.clusters
        centres = rng.standard_normal(size=(q, d), dtype=np.float32)
        member = np.empty(m, dtype=np.int64)
        for s in range(m // cfg.seg_len):
            u = rng.random(cfg.seg_len)
            other = rng.integers(0, q, size=cfg.seg_len)
            member[s * cfg.seg_len:(s + 1) * cfg.seg_len] = np.where(u < 0.9, s % q, other)
        x = centres[member] + _normal(rng, (m, d), 0.5)
    else:
        x = _normal(rng, (m, d), 1.0)
    return _store(x, cfg.dtype)


def _rank_bias(cfg: LayerConfig, seed: int):
    if cfg.lossfree_bias <= 0:
        return None
    w = cfg.lossfree_bias
    return np.random.default_rng([seed, 1]).uniform(-w, w, size=cfg.n).astype(np.float32)


def make_layer_inputs(cfg: LayerConfig, seed: int = 0, bias_std: float = 0.0) -> dict:
    """All inputs of one layer forward, as float32 arrays holding storage-dtype values.

    Shapes: x [m,d]; w_r [d,n] (fp32 always); w1 [n,d_ff,d] and w2 [n,d,d_ff]
    (each expert's matrices in the output-major layout of a linear layer);
    b1 [n,d_ff]; b2 [n,d]; rank_bias [n] or None.
    bias_std > 0 draws N(0, bias_std^2) FFN biases instead of zeros.
    """
    rng = np.random.default_rng(seed)
    m, d, n, d_ff = cfg.m, cfg.d, cfg.n, cfg.d_ff
    x = _draw_tokens(rng, cfg)
    w_r = _normal(rng, (d, n), cfg.wr_std)
    w1 = np.empty((n, d_ff, d), dtype=np.float32)
    for e in range(n):
        w1[e] = _store(_normal(rng, (d_ff, d), 1.0 / math.sqrt(d)), cfg.dtype)
    b1 = _store(_normal(rng, (n, d_ff), bias_std) if bias_std > 0 else np.zeros((n, d_ff), np.float32), cfg.dtype)
    w2 = np.empty((n, d, d_ff), dtype=np.float32)
    for e in range(n):
        w2[e] = _store(_normal(rng, (d, d_ff), 1.0 / math.sqrt(d_ff)), cfg.dtype)
    b2 = _store(_normal(rng, (n, d), bias_std) if bias_std > 0 else np.zeros((n, d), np.float32), cfg.dtype)
    return dict(x=x, w_r=w_r, w1=w1, b1=b1, w2=w2, b2=b2, rank_bias=_rank_bias(cfg, seed))


def make_router_inputs(cfg: LayerConfig, seed: int = 0) -> dict:
    """Only the router-side inputs (x, w_r, rank_bias) in the same draw order, no expert weights."""
    rng = np.random.default_rng(seed)
    m, d, n = cfg.m, cfg.d, cfg.n
    x = _draw_tokens(rng, cfg)
    w_r = _normal(rng, (d, n), cfg.wr_std)
    return dict(x=x, w_r=w_r, rank_bias=_rank_bias(cfg, seed))


def make_qb_scores(m: int = 65536, n: int = 256, seed: int = 0, skew_std: float = 1.5) -> np.ndarray:
    """Scores s_ij = N(0,1) + c_j with a per-expert skew c_j ~ N(0, skew_std^2), fp32 [m,n]."""
    rng = np.random.default_rng(seed)
    s = rng.standard_normal(size=(m, n), dtype=np.float32)
    c = rng.standard_normal(size=n, dtype=np.float32) * np.float32(skew_std)
    s += c[None, :]
    return s


def make_topk_idx(m: int, n: int, k: int, seed: int = 0, skew: float = 1.0) -> np.ndarray:
    """Random distinct expert choices per token, [m,k] int32, with a skewed expert popularity."""
    rng = np.random.default_rng(seed)
    pop = np.exp(skew * rng.standard_normal(n))
    keys = rng.gumbel(size=(m, n)) + np.log(pop)[None, :]
    idx = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    return np.ascontiguousarray(idx.astype(np.int32))


def make_uniform_probs(m: int, n: int) -> np.ndarray:
    """probs identically 1/n (the balanced case for the auxiliary loss)."""
    return np.full((m, n), 1.0 / n, dtype=np.float32)


def make_round_robin_idx(m: int, n: int, k: int) -> np.ndarray:
    """Token i picks experts (i*k + r) mod n, r < k: every expert gets exactly m*k/n picks when n | m*k."""
    i = np.arange(m, dtype=np.int64)[:, None] * k + np.arange(k, dtype=np.int64)[None, :]
    return np.ascontiguousarray((i % n).astype(np.int32))
