"""Seeded synthetic inputs for HSTU pointwise attention (numpy only).

This module holds input generation and nothing of the method's arithmetic; the
CUDA library, the CPU oracle, the tests and the benchmark all draw their
inputs from it.  The pages' own data (Yambda-5B per-user music timelines,
DLRMv4 article, section "Dataset") is not available here; these generators
stand in for it with the same structure: per-user time-ordered event
sequences, jagged lengths, timestamps in seconds, truncated to a fixed upper
length.

Recipe (shared by all workloads):
  * timestamps: start 1.7e9 s; gaps max(1, round(Exp(mean 600 s))), so every
    sequence is strictly increasing; M-FALCON candidates all take the last
    history timestamp plus one more such gap; prefix context tokens (when
    asked for) take the first event's timestamp.
  * rab tables: N(0, 0.02) float32, one scalar per bucket.
  * Q, K, V, dO, X: N(0, 1), rounded to the path's dtype (bf16 by
    round-to-nearest-even).
  * alpha = 1/sqrt(d_qk); silu_scale = 1/max_seq_len.
  * weights: Xavier-uniform; biases 0; LayerNorm gamma 1, beta 0.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

TS_START = 1_700_000_000
TS_MEAN_GAP = 600.0


def round_bf16(a: np.ndarray) -> np.ndarray:
    """float32 array of the bf16 values nearest to ``a`` (ties to even)."""
    x = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    x = (x + 0x7FFF + ((x >> 16) & 1)) >> 16 << 16
    return (x.astype(np.uint32)).view(np.float32)


def _cast(a: np.ndarray, dtype: str) -> np.ndarray:
    a = np.asarray(a, dtype=np.float32)
    return round_bf16(a) if dtype == "bf16" else a


def _timestamps(rng, lengths, num_candidates=None, num_prefix=0) -> np.ndarray:
    out = []
    for b, L in enumerate(lengths):
        nc = 0 if num_candidates is None else int(num_candidates[b])
        nh = int(L) - nc
        gaps = np.maximum(1, np.rint(rng.exponential(TS_MEAN_GAP, size=nh))).astype(np.int64)
        ts = TS_START + np.cumsum(gaps) - gaps[0] if nh > 0 else np.zeros(0, np.int64)
        # prefix context tokens carry the first event's timestamp
        npf = min(int(num_prefix), nh)
        if npf and nh > npf:
            ts[:npf] = ts[npf]
        if nc:
            last = ts[-1] if nh else TS_START
            gap = max(1, int(np.rint(rng.exponential(TS_MEAN_GAP))))
            ts = np.concatenate([ts, np.full(nc, last + gap, np.int64)])
        out.append(ts.astype(np.int64))
    return np.concatenate(out) if out else np.zeros(0, np.int64)


def _offsets(lengths) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(lengths, np.int64))]).astype(np.int64)


@dataclass
class AttnWorkload:
    """One jagged attention problem with its inputs (float32 arrays; bf16
    workloads hold bf16-representable values)."""
    name: str
    dtype: str                         # "f32" or "bf16"
    offsets: np.ndarray                # int64 [B+1]
    timestamps: np.ndarray             # int64 [T]
    num_heads: int
    d_qk: int
    d_v: int
    num_pos_buckets: int
    num_time_buckets: int
    time_bucket_sub_bits: int
    max_seq_len: int
    alpha: float
    silu_scale: float
    q: np.ndarray                      # [T, H, d_qk]
    k: np.ndarray
    v: np.ndarray                      # [T, H, d_v]
    rab_p: np.ndarray                  # [nb_p] or [H, nb_p]
    rab_t: np.ndarray
    dout: Optional[np.ndarray] = None  # [T, H, d_v]
    num_candidates: Optional[np.ndarray] = None   # int32 [B] (M-FALCON)
    rab_per_head: bool = False

    @property
    def batch(self) -> int:
        return len(self.offsets) - 1

    @property
    def total_tokens(self) -> int:
        return int(self.offsets[-1])

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.offsets)

    def visible_pairs(self) -> int:
        """Number of visible (query, key) pairs per head."""
        n = 0
        for b, L in enumerate(self.lengths.tolist()):
            nc = 0 if self.num_candidates is None else int(self.num_candidates[b])
            nh = L - nc
            n += nh * (nh + 1) // 2 + nc * (nh + 1)
        return n


def make_attention(name: str, lengths, num_heads: int, d: int, nb: int, sub_bits: int,
                   dtype: str, seed: int, max_seq_len: Optional[int] = None,
                   num_candidates=None, with_grad: bool = False, d_v: Optional[int] = None,
                   nb_t: Optional[int] = None, rab_per_head: bool = False,
                   time_gap_scale: float = 1.0, num_prefix: int = 0) -> AttnWorkload:
    """A seeded jagged attention problem.  num_prefix > 0 starts every
    sequence with that many context tokens (user id, slowly changing
    features) ahead of its events; they are ordinary tokens of the sequence
    (every later token sees them through the causal mask) and take the
    first event's timestamp."""
    rng = np.random.default_rng(seed)
    lengths = [int(l) for l in lengths]
    dv = d if d_v is None else d_v
    nbt = nb if nb_t is None else nb_t
    offsets = _offsets(lengths)
    T = int(offsets[-1])
    ts = _timestamps(rng, lengths, num_candidates, num_prefix)
    if time_gap_scale != 1.0:   # stretch the timeline (exercises wide time spans)
        ts = TS_START + ((ts - TS_START) * time_gap_scale).astype(np.int64)
    msl = max(lengths) if max_seq_len is None else max_seq_len
    tabs = num_heads if rab_per_head else 1
    rab_p = (rng.standard_normal((tabs, nb)) * 0.02).astype(np.float32)
    rab_t = (rng.standard_normal((tabs, nbt)) * 0.02).astype(np.float32)
    if not rab_per_head:
        rab_p, rab_t = rab_p[0], rab_t[0]
    q = _cast(rng.standard_normal((T, num_heads, d)), dtype)
    k = _cast(rng.standard_normal((T, num_heads, d)), dtype)
    v = _cast(rng.standard_normal((T, num_heads, dv)), dtype)
    dout = _cast(rng.standard_normal((T, num_heads, dv)), dtype) if with_grad else None
    nc = None if num_candidates is None else np.asarray(num_candidates, np.int32)
    return AttnWorkload(name=name, dtype=dtype, offsets=offsets, timestamps=ts,
                        num_heads=num_heads, d_qk=d, d_v=dv, num_pos_buckets=nb,
                        num_time_buckets=nbt, time_bucket_sub_bits=sub_bits, max_seq_len=msl,
                        alpha=1.0 / float(np.sqrt(d)), silu_scale=1.0 / float(msl), q=q, k=k,
                        v=v, rab_p=rab_p, rab_t=rab_t, dout=dout, num_candidates=nc,
                        rab_per_head=rab_per_head)


@dataclass
class LayerWeights:
    w1: np.ndarray      # [N1, d_model], rows U | V | Q | K
    b1: np.ndarray      # [N1]
    ln_gamma: np.ndarray
    ln_beta: np.ndarray
    w2: np.ndarray      # [d_model, H d_v]
    b2: np.ndarray      # [d_model]
    rab_p: np.ndarray
    rab_t: np.ndarray


@dataclass
class LayerWorkload:
    name: str
    attn: AttnWorkload       # shapes, offsets, timestamps (its q/k/v are unused)
    d_model: int
    x: np.ndarray            # [T, d_model]
    layers: List[LayerWeights] = field(default_factory=list)
    ln_eps: float = 1e-5
    residual: bool = True


def xavier_uniform(rng, fan_out: int, fan_in: int, dtype: str) -> np.ndarray:
    bound = float(np.sqrt(6.0 / (fan_in + fan_out)))
    return _cast(rng.uniform(-bound, bound, size=(fan_out, fan_in)), dtype)


def make_layer(name: str, lengths, num_heads: int, d: int, d_model: int, nb: int, sub_bits: int,
               seed: int, n_layers: int = 1, num_candidates=None,
               max_seq_len: Optional[int] = None) -> LayerWorkload:
    attn = make_attention(name, lengths, num_heads, d, nb, sub_bits, "bf16", seed,
                          max_seq_len=max_seq_len, num_candidates=num_candidates)
    rng = np.random.default_rng(seed + 1000)
    T = attn.total_tokens
    n1 = 4 * num_heads * d
    x = _cast(rng.standard_normal((T, d_model)), "bf16")
    layers = []
    for _ in range(n_layers):
        layers.append(LayerWeights(
            w1=xavier_uniform(rng, n1, d_model, "bf16"),
            b1=np.zeros(n1, np.float32),
            ln_gamma=np.ones(num_heads * d, np.float32),
            ln_beta=np.zeros(num_heads * d, np.float32),
            w2=xavier_uniform(rng, d_model, num_heads * d, "bf16"),
            b2=np.zeros(d_model, np.float32),
            rab_p=(rng.standard_normal(nb) * 0.02).astype(np.float32),
            rab_t=(rng.standard_normal(nb) * 0.02).astype(np.float32)))
    return LayerWorkload(name=name, attn=attn, d_model=d_model, x=x, layers=layers)


def zipf_lengths(rng, n: int, s: float, lo: int, hi: int) -> np.ndarray:
    """n lengths from P(L) proportional to L^-s on the integers [lo, hi]."""
    support = np.arange(lo, hi + 1, dtype=np.float64)
    pmf = support ** (-s)
    pmf /= pmf.sum()
    return rng.choice(np.arange(lo, hi + 1), size=n, p=pmf).astype(np.int64)


# ---------------------------------------------------------------------------
# The five reference workloads.
# ---------------------------------------------------------------------------

def tiny_f32_fwd() -> AttnWorkload:
    """2 sequences (37, 64), 2 heads, d=32, fp32; 64 position / 32 time buckets."""
    return make_attention("tiny_f32_fwd", [37, 64], 2, 32, 64, 0, "f32", seed=0,
                          nb_t=32, max_seq_len=64, with_grad=True)


def layer_bf16_fwd() -> LayerWorkload:
    """Batch 32, lengths U[64,1024], d_model 256, 4 heads, d 64, 128 buckets."""
    rng = np.random.default_rng(1)
    lengths = rng.integers(64, 1024, size=32, endpoint=True)
    return make_layer("layer_bf16_fwd", lengths, 4, 64, 256, 128, 2, seed=1, max_seq_len=1024)


def zipf_bf16_fwd_bwd() -> AttnWorkload:
    """Batch 16, Zipf(1.1) lengths on [16,4096], 8 heads, d 128, 128 buckets."""
    rng = np.random.default_rng(2)
    lengths = zipf_lengths(rng, 16, 1.1, 16, 4096)
    return make_attention("zipf_bf16_fwd_bwd", lengths, 8, 128, 128, 2, "bf16", seed=2,
                          max_seq_len=4096, with_grad=True)


def long_bf16_fwd_bwd() -> AttnWorkload:
    """Batch 4 x length 8192, 8 heads, d 128, causal, 256 buckets."""
    return make_attention("long_bf16_fwd_bwd", [8192] * 4, 8, 128, 256, 3, "bf16", seed=3,
                          max_seq_len=8192, with_grad=True)


def mfalcon_bf16_fwd(n_users: int = 8) -> LayerWorkload:
    """8 users x (4096 history + 1024 candidates), 8 heads, d 128, d_model 512,
    3 stacked layers, 128 buckets."""
    return make_layer("mfalcon_bf16_fwd", [4096 + 1024] * n_users, 8, 128, 512, 128, 2,
                      seed=4, n_layers=3, num_candidates=[1024] * n_users, max_seq_len=5120)


WORKLOADS = {
    "tiny_f32_fwd": tiny_f32_fwd,
    "layer_bf16_fwd": layer_bf16_fwd,
    "zipf_bf16_fwd_bwd": zipf_bf16_fwd_bwd,
    "long_bf16_fwd_bwd": long_bf16_fwd_bwd,
    "mfalcon_bf16_fwd": mfalcon_bf16_fwd,
}
