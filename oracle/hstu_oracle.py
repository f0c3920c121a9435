"""Python face of the CPU oracle (float64), plus the layer restated in numpy.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  It imports nothing from
the CUDA library's package and the CUDA library imports nothing from here.

The attention itself is computed by ``libhstu_oracle.so`` (``hstu_oracle.c``),
a direct float64 loop over (sequence, head, query, key).  The layer around it
follows the DLRMv4 article ("DLRMv4: MLPerf's recommendation-training benchmark
enters the sequence era", section "Model architecture: HSTU replaces the
feature-interaction stack"): one projection produces the layer's internal
representations, pointwise attention aggregates the sequence, and a gated
transformation takes the place of the cross network and feed-forward block.
Readings taken where that page is silent:
  R8   SiLU on all four projected blocks, column order U | V | Q | K.
  R9   LayerNorm over the H*d_v features of a token, biased variance.
  R10  residual connection around the layer (stacked layers).
  R11  biases b1, b2 on both projections.
Library primitives used as steps: numpy matmul for the two projections.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_oracle.c")
_HDR = os.path.join(_HERE, "hstu_oracle.h")
_LIB = os.path.join(_HERE, "libhstu_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP over sequences x heads)."""
    stale = (not os.path.exists(_LIB) or
             os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_heads", ctypes.c_int32),
        ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32),
        ("num_pos_buckets", ctypes.c_int32), ("num_time_buckets", ctypes.c_int32),
        ("time_bucket_sub_bits", ctypes.c_int32), ("rab_per_head", ctypes.c_int32),
        ("alpha", ctypes.c_double), ("silu_scale", ctypes.c_double),
        ("offsets", ctypes.c_void_p), ("num_candidates", ctypes.c_void_p),
        ("timestamps", ctypes.c_void_p),
    ]


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.POINTER(_Problem)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        _lib.hstu_oracle_time_bucket.argtypes = [i64, i32, i32]
        _lib.hstu_oracle_time_bucket.restype = i32
        _lib.hstu_oracle_pos_bucket.argtypes = [i64, i32]
        _lib.hstu_oracle_pos_bucket.restype = i32
        _lib.hstu_oracle_visible.argtypes = [i64, i64, i64]
        _lib.hstu_oracle_visible.restype = i32
        _lib.hstu_oracle_position.argtypes = [i64, i64]
        _lib.hstu_oracle_position.restype = i64
        _lib.hstu_oracle_buckets.argtypes = [P, vp, vp]
        _lib.hstu_oracle_attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, i64, vp]
        _lib.hstu_oracle_attn_bwd.argtypes = [P] + [vp] * 11
        _lib.hstu_oracle_attn_bwd_sampled.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, i64, vp,
                                                      vp, i64, vp, vp, i32, vp]
        _lib.hstu_oracle_attn_drab.argtypes = [P] + [vp] * 8
        _lib.hstu_oracle_num_threads.restype = ctypes.c_int
    return _lib


def num_threads() -> int:
    return int(lib().hstu_oracle_num_threads())


@dataclass
class Problem:
    """One jagged attention problem, in the oracle's terms."""
    offsets: np.ndarray                 # int64 [B+1]
    timestamps: np.ndarray              # int64 [T]
    num_heads: int
    d_qk: int
    d_v: int
    num_pos_buckets: int
    num_time_buckets: int
    time_bucket_sub_bits: int
    alpha: float
    silu_scale: float
    num_candidates: Optional[np.ndarray] = None   # int32 [B] (M-FALCON) or None
    rab_per_head: bool = False
    _keep: list = field(default_factory=list, repr=False)

    @property
    def batch(self) -> int:
        return len(self.offsets) - 1

    @property
    def total_tokens(self) -> int:
        return int(self.offsets[-1])

    def c(self) -> _Problem:
        off = np.ascontiguousarray(self.offsets, dtype=np.int64)
        ts = np.ascontiguousarray(self.timestamps, dtype=np.int64)
        nc = (None if self.num_candidates is None
              else np.ascontiguousarray(self.num_candidates, dtype=np.int32))
        self._keep = [off, ts, nc]
        return _Problem(self.batch, self.num_heads, self.d_qk, self.d_v, self.num_pos_buckets,
                        self.num_time_buckets, self.time_bucket_sub_bits, int(self.rab_per_head),
                        float(self.alpha), float(self.silu_scale), off.ctypes.data,
                        None if nc is None else nc.ctypes.data, ts.ctypes.data)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a) -> Optional[int]:
    return None if a is None else a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def time_bucket(dt: int, sub_bits: int, num_buckets: int) -> int:
    return int(lib().hstu_oracle_time_bucket(int(dt), int(sub_bits), int(num_buckets)))


def pos_bucket(dp: int, num_buckets: int) -> int:
    return int(lib().hstu_oracle_pos_bucket(int(dp), int(num_buckets)))


def visible(i: int, j: int, n_hist: int) -> bool:
    return bool(lib().hstu_oracle_visible(int(i), int(j), int(n_hist)))


def position(i: int, n_hist: int) -> int:
    return int(lib().hstu_oracle_position(int(i), int(n_hist)))


def buckets(p: Problem):
    """Per-sequence dense L x L (bp, bt) int32 blocks, -1 where not visible."""
    L = np.diff(p.offsets)
    n = int((L.astype(np.int64) ** 2).sum())
    bp = np.empty(max(n, 1), np.int32)
    bt = np.empty(max(n, 1), np.int32)
    _check(lib().hstu_oracle_buckets(ctypes.byref(p.c()), bp.ctypes.data, bt.ctypes.data),
           "buckets")
    out, base = [], 0
    for l in L:
        l = int(l)
        out.append((bp[base:base + l * l].reshape(l, l), bt[base:base + l * l].reshape(l, l)))
        base += l * l
    return out


def attn_fwd(p: Problem, q, k, v, rab_p, rab_t, rows=None) -> np.ndarray:
    """O [T or n_rows, H, d_v] in float64."""
    q, k, v, rab_p, rab_t = map(_f64, (q, k, v, rab_p, rab_t))
    T, H = p.total_tokens, p.num_heads
    rows_a = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = T if rows_a is None else len(rows_a)
    out = np.zeros((n, H, p.d_v), np.float64)
    _check(lib().hstu_oracle_attn_fwd(ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(rab_p), _ptr(rab_t), _ptr(rows_a),
                                      0 if rows_a is None else n, _ptr(out)), "attn_fwd")
    return out


def attn_bwd(p: Problem, q, k, v, rab_p, rab_t, dout):
    """(dq, dk, dv, drab_p, drab_t) in float64."""
    q, k, v, rab_p, rab_t, dout = map(_f64, (q, k, v, rab_p, rab_t, dout))
    T, H = p.total_tokens, p.num_heads
    dq = np.zeros((T, H, p.d_qk))
    dk = np.zeros((T, H, p.d_qk))
    dv = np.zeros((T, H, p.d_v))
    drp = np.zeros(rab_p.shape)
    drt = np.zeros(rab_t.shape)
    _check(lib().hstu_oracle_attn_bwd(ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(rab_p), _ptr(rab_t), _ptr(dout), _ptr(dq), _ptr(dk),
                                      _ptr(dv), _ptr(drp), _ptr(drt)), "attn_bwd")
    return dq, dk, dv, drp, drt


def attn_drab(p: Problem, q, k, v, rab_p, rab_t, dout):
    """(drab_p, drab_t) in full, float64: the bias-table gradients of
    ``attn_bwd`` without its dq / dk / dv sums, split by (sequence, head, 64
    query rows) so that a single long sequence keeps every thread busy."""
    q, k, v, rab_p, rab_t, dout = map(_f64, (q, k, v, rab_p, rab_t, dout))
    drp = np.zeros(rab_p.shape)
    drt = np.zeros(rab_t.shape)
    _check(lib().hstu_oracle_attn_drab(ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(rab_p), _ptr(rab_t), _ptr(dout), _ptr(drp),
                                       _ptr(drt)), "attn_drab")
    return drp, drt


def attn_bwd_sampled(p: Problem, q, k, v, rab_p, rab_t, dout, dq_rows=(), kv_cols=(),
                     drab_p_band: int = 0):
    """dQ on sampled query tokens, dK/dV on sampled key tokens, and drab_p
    restricted to the buckets below ``drab_p_band`` (exact for those buckets)."""
    q, k, v, rab_p, rab_t, dout = map(_f64, (q, k, v, rab_p, rab_t, dout))
    H = p.num_heads
    rows = np.ascontiguousarray(dq_rows, dtype=np.int64)
    cols = np.ascontiguousarray(kv_cols, dtype=np.int64)
    dq = np.zeros((len(rows), H, p.d_qk))
    dk = np.zeros((len(cols), H, p.d_qk))
    dv = np.zeros((len(cols), H, p.d_v))
    drp = np.zeros(rab_p.shape) if drab_p_band > 0 else None
    _check(lib().hstu_oracle_attn_bwd_sampled(
        ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(rab_p), _ptr(rab_t), _ptr(dout),
        _ptr(rows) if len(rows) else None, len(rows), _ptr(dq) if len(rows) else None,
        _ptr(cols) if len(cols) else None, len(cols), _ptr(dk) if len(cols) else None,
        _ptr(dv) if len(cols) else None, int(drab_p_band), _ptr(drp)), "attn_bwd_sampled")
    return dq, dk, dv, drp


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def layer_fwd(p: Problem, x, w1, b1, ln_gamma, ln_beta, w2, b2, rab_p, rab_t,
              ln_eps: float = 1e-5, residual: bool = True) -> np.ndarray:
    """One HSTU layer, float64 (readings R8-R11 in the module docstring).

    x [T, d_model]; w1 [2 H d_v + 2 H d_qk, d_model] (rows U | V | Q | K);
    b1 [N1]; ln_gamma, ln_beta [H d_v]; w2 [d_model, H d_v]; b2 [d_model]."""
    x, w1, b1, g, bta, w2, b2 = map(_f64, (x, w1, b1, ln_gamma, ln_beta, w2, b2))
    T, H, dqk, dv = p.total_tokens, p.num_heads, p.d_qk, p.d_v
    proj = silu(x @ w1.T + b1)                        # [T, N1]
    u = proj[:, :H * dv]
    vv = proj[:, H * dv:2 * H * dv].reshape(T, H, dv)
    q = proj[:, 2 * H * dv:2 * H * dv + H * dqk].reshape(T, H, dqk)
    k = proj[:, 2 * H * dv + H * dqk:].reshape(T, H, dqk)
    a = attn_fwd(p, q, k, vv, rab_p, rab_t).reshape(T, H * dv)
    mean = a.mean(axis=1, keepdims=True)
    var = ((a - mean) ** 2).mean(axis=1, keepdims=True)
    ln = (a - mean) / np.sqrt(var + ln_eps) * g + bta
    y = (ln * u) @ w2.T + b2
    return x + y if residual else y


def silu_grad(x: np.ndarray) -> np.ndarray:
    """d SiLU / dx = sigma(x) (1 + x (1 - sigma(x)))."""
    sg = 1.0 / (1.0 + np.exp(-x))
    return sg * (1.0 + x * (1.0 - sg))


def layer_bwd(p: Problem, x, w1, b1, ln_gamma, ln_beta, w2, b2, rab_p, rab_t, dy,
              ln_eps: float = 1e-5, residual: bool = True):
    """Gradients of one HSTU layer (``layer_fwd``) for an upstream gradient dy
    [T, d_model], float64, by the chain rule through its four steps in reverse:

      y = x + G W2^T + b2           dG = dy W2, dW2 = dy^T G, db2 = sum_t dy
      G = LN(A) (.) U               dU = dG (.) LN(A), dLN = dG (.) U
      LN(A) = xhat gamma + beta     dgamma = sum_t dLN (.) xhat, dbeta = sum_t dLN,
        xhat = (A - mean) / sigma   dA = (dxh - mean(dxh) - xhat mean(dxh (.) xhat)) / sigma
                                    with dxh = dLN (.) gamma, sigma = sqrt(var + eps)
      A = attention(Q, K, V)        dQ, dK, dV, drab_p, drab_t = attn_bwd(dA)
      [U|V|Q|K] = SiLU(Z),          dZ = [dU|dV|dQ|dK] (.) SiLU'(Z)
        Z = x W1^T + b1             dW1 = dZ^T x, db1 = sum_t dZ, dx = dZ W1 (+ dy)

    Returns (dx, dw1, db1, dgamma, dbeta, dw2, db2, drab_p, drab_t)."""
    x, w1, b1, g, bta, w2, b2, dy = map(_f64, (x, w1, b1, ln_gamma, ln_beta, w2, b2, dy))
    T, H, dqk, dv = p.total_tokens, p.num_heads, p.d_qk, p.d_v
    F = H * dv
    z = x @ w1.T + b1                                 # [T, N1]
    proj = silu(z)
    u = proj[:, :F]
    vv = proj[:, F:2 * F].reshape(T, H, dv)
    q = proj[:, 2 * F:2 * F + H * dqk].reshape(T, H, dqk)
    k = proj[:, 2 * F + H * dqk:].reshape(T, H, dqk)
    a = attn_fwd(p, q, k, vv, rab_p, rab_t).reshape(T, F)
    mean = a.mean(axis=1, keepdims=True)
    var = ((a - mean) ** 2).mean(axis=1, keepdims=True)
    sigma = np.sqrt(var + ln_eps)
    xhat = (a - mean) / sigma
    ln = xhat * g + bta
    G = ln * u
    # output projection
    dG = dy @ w2                                      # [T, F]
    dw2 = dy.T @ G                                    # [d_model, F]
    db2 = dy.sum(axis=0)
    # gating
    du = dG * ln
    dln = dG * u
    # LayerNorm
    dgamma = (dln * xhat).sum(axis=0)
    dbeta = dln.sum(axis=0)
    dxh = dln * g
    da = (dxh - dxh.mean(axis=1, keepdims=True)
          - xhat * (dxh * xhat).mean(axis=1, keepdims=True)) / sigma
    # attention
    dq, dk, dvv, drab_p, drab_t = attn_bwd(p, q, k, vv, rab_p, rab_t, da.reshape(T, H, dv))
    dproj = np.concatenate([du, dvv.reshape(T, F), dq.reshape(T, H * dqk),
                            dk.reshape(T, H * dqk)], axis=1)
    # projection
    dz = dproj * silu_grad(z)
    dw1 = dz.T @ x
    db1 = dz.sum(axis=0)
    dx = dz @ w1
    if residual:
        dx = dx + dy
    return dx, dw1, db1, dgamma, dbeta, dw2, db2, drab_p, drab_t


# ---------------------------------------------------------------------------
# M-FALCON candidate micro-batches against a cached history
# ---------------------------------------------------------------------------

def attn_fwd_candidates(p: Problem, hist_offsets, cand_offsets, hist_timestamps,
                        cand_timestamps, q_cand, k_cand, v_cand, k_hist, v_hist, rab_p, rab_t):
    """Outputs [Tc, H, d_v] of one candidate micro-batch, float64.

    The definition restated: a candidate sees every history token of its
    sequence and itself, at position n_h (the M-FALCON mask of ``attn_fwd``;
    the "Actions Speak Louder than Words" contribution list for M-FALCON, the
    DLRMv4 article's "How one training sample is processed by HSTU" for
    candidates compared with the whole history).  So each sequence's
    micro-batch is evaluated as the one-pass M-FALCON forward of
    [history ; these candidates] with n_c = the micro-batch size, keeping the
    candidate rows.  ``p`` supplies the head sizes, buckets and scales (its
    offsets / timestamps are not used)."""
    hoff = np.asarray(hist_offsets, np.int64)
    coff = np.asarray(cand_offsets, np.int64)
    H, dqk, dv = p.num_heads, p.d_qk, p.d_v
    out = np.zeros((int(coff[-1]), H, dv), np.float64)
    for b in range(len(hoff) - 1):
        h0, h1, c0, c1 = int(hoff[b]), int(hoff[b + 1]), int(coff[b]), int(coff[b + 1])
        if c1 == c0:
            continue
        nh, nc = h1 - h0, c1 - c0
        q = np.concatenate([np.zeros((nh, H, dqk)), _f64(q_cand[c0:c1])])
        k = np.concatenate([_f64(k_hist[h0:h1]), _f64(k_cand[c0:c1])])
        v = np.concatenate([_f64(v_hist[h0:h1]), _f64(v_cand[c0:c1])])
        ts = np.concatenate([np.asarray(hist_timestamps[h0:h1], np.int64),
                             np.asarray(cand_timestamps[c0:c1], np.int64)])
        one = Problem(offsets=np.array([0, nh + nc], np.int64), timestamps=ts, num_heads=H,
                      d_qk=dqk, d_v=dv, num_pos_buckets=p.num_pos_buckets,
                      num_time_buckets=p.num_time_buckets,
                      time_bucket_sub_bits=p.time_bucket_sub_bits, alpha=p.alpha,
                      silu_scale=p.silu_scale, num_candidates=np.array([nc], np.int32),
                      rab_per_head=p.rab_per_head)
        rows = np.arange(nh, nh + nc, dtype=np.int64)
        out[c0:c1] = attn_fwd(one, q, k, v, rab_p, rab_t, rows=rows)
    return out


def layer_proj(x, w1, b1) -> np.ndarray:
    """[U|V|Q|K] = SiLU(x W1^T + b1), float64 (the first step of ``layer_fwd``)."""
    x, w1, b1 = map(_f64, (x, w1, b1))
    return silu(x @ w1.T + b1)


def layer_fwd_candidates(p: Problem, hist_offsets, cand_offsets, hist_timestamps,
                         cand_timestamps, x_cand, hist_proj, w1, b1, ln_gamma, ln_beta, w2, b2,
                         rab_p, rab_t, ln_eps: float = 1e-5, residual: bool = True):
    """One layer (``layer_fwd``'s steps) on candidate rows only, their
    attention against the history's V and K columns of ``hist_proj``."""
    x, g, bta, w2_, b2_ = map(_f64, (x_cand, ln_gamma, ln_beta, w2, b2))
    Tc, H, dqk, dv = x.shape[0], p.num_heads, p.d_qk, p.d_v
    F = H * dv
    proj = layer_proj(x, w1, b1)
    hp = _f64(hist_proj)
    Th = hp.shape[0]
    u = proj[:, :F]
    a = attn_fwd_candidates(
        p, hist_offsets, cand_offsets, hist_timestamps, cand_timestamps,
        proj[:, 2 * F:2 * F + H * dqk].reshape(Tc, H, dqk),
        proj[:, 2 * F + H * dqk:].reshape(Tc, H, dqk), proj[:, F:2 * F].reshape(Tc, H, dv),
        hp[:, 2 * F + H * dqk:].reshape(Th, H, dqk), hp[:, F:2 * F].reshape(Th, H, dv),
        rab_p, rab_t).reshape(Tc, F)
    mean = a.mean(axis=1, keepdims=True)
    var = ((a - mean) ** 2).mean(axis=1, keepdims=True)
    ln = (a - mean) / np.sqrt(var + ln_eps) * g + bta
    y = (ln * u) @ w2_.T + b2_
    return x + y if residual else y
