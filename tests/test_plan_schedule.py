"""The jagged tile schedule (the work lists every attention call builds on the
host) against a brute-force enumeration of the visible blocks.

The visibility rule is the causal / M-FALCON mask of the DLRMv4 article,
section "How one training sample is processed by HSTU" (history tokens see
their past, candidates appended at the end see the whole history and
themselves), restated here as a dense boolean matrix per sequence.  Every
(query tile, key tile) block of the forward and every (key tile, 64-query
block) block of the backward that holds a visible pair must be covered by
exactly one work item; nothing outside a sequence may be scheduled.  Host
only: hstu_debug_plan makes no CUDA call.
"""
import numpy as np
import pytest

from hstu_pointwise_attention_b200 import ops

UNSPLIT = 0x7FFFFFFF


def _params(batch, heads, d, max_len, mfalcon):
    p = ops.AttnParams()
    p.batch, p.num_heads, p.d_qk, p.d_v = batch, heads, d, d
    p.max_seq_len = max_len
    p.num_pos_buckets = p.num_time_buckets = 128
    p.time_bucket_sub_bits = 3
    p.mask = ops.MASK_MFALCON if mfalcon else ops.MASK_CAUSAL
    p.dtype = ops.BF16
    for f in ("q_row_stride", "k_row_stride", "v_row_stride", "o_row_stride", "do_row_stride",
              "dq_row_stride", "dk_row_stride", "dv_row_stride"):
        setattr(p, f, heads * d)
    p.alpha, p.silu_scale = 0.1, 0.01
    return p


def _visible(L, nh):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    hist = (i < nh) & (j <= i)
    cand = (i >= nh) & ((j < nh) | (j == i))
    return hist | cand


def _blocks(vis, rows, cols):
    L = vis.shape[0]
    nr, nc = -(-L // rows), -(-L // cols)
    out = np.zeros((nr, nc), dtype=bool)
    for a in range(nr):
        for b in range(nc):
            out[a, b] = vis[a * rows:(a + 1) * rows, b * cols:(b + 1) * cols].any()
    return out


def _check(lengths, cands, heads=8, d=128):
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    mf = cands is not None
    p = _params(len(lengths), heads, d, max(1, max(lengths, default=1)), mf)
    fwd, bwd = ops.debug_plan(p, off, cands)
    fcover, bcover = {}, {}
    for b, L in enumerate(lengths):
        nh = L - (cands[b] if mf else 0)
        vis = _visible(L, nh)
        fcover[b] = (_blocks(vis, 128, 128), np.zeros((-(-L // 128),) * 2, dtype=int))
        bcover[b] = (_blocks(vis.T, 128, 64), np.zeros((-(-L // 128), -(-L // 64)), dtype=int))
    # forward: item {b, pair, first, end}; an unsplit item walks key tiles
    # 0 .. the pair's last query tile
    cost = []
    for b, pr, z, w in fwd:
        L = lengths[b]
        n_qt = -(-L // 128)
        assert 0 <= 2 * pr < n_qt
        last = min(2 * pr + 1, n_qt - 1)
        lo, hi = (0, last + 1) if w == UNSPLIT else (z, w)
        assert 0 <= lo < hi <= last + 1
        cost.append(hi - lo)
        for qt in (2 * pr, 2 * pr + 1):
            if qt < n_qt:
                fcover[b][1][qt, lo:hi] += 1
    assert cost == sorted(cost, reverse=True)   # longest first
    for b, (need, got) in fcover.items():
        assert (got[need] == 1).all(), f"sequence {b}: a visible forward block is not covered once"
        assert (got <= 1).all()
    # backward: item {b, key tile, first block, end block}; an unsplit item
    # walks the run from the tile's first key to the sequence end (history
    # keys) or to the block of its last candidate
    cost = []
    for b, kt, z, w in bwd:
        L = lengths[b]
        nh = L - (cands[b] if mf else 0)
        ks = 128 * kt
        assert 0 <= ks < L
        n_qb = -(-L // 64)
        end = n_qb if ks < nh else -(-min(ks + 128, L) // 64)
        lo, hi = (2 * kt, end) if w == UNSPLIT else (max(z, 2 * kt), min(w, end))
        assert 2 * kt <= lo < hi <= end
        cost.append(hi - lo if w != UNSPLIT else end - 2 * kt)
        bcover[b][1][kt, lo:hi] += 1
    assert cost == sorted(cost, reverse=True)
    for b, (need, got) in bcover.items():
        assert (got[need] == 1).all(), f"sequence {b}: a visible backward block is not covered once"
        assert (got <= 1).all()
    return fwd, bwd


@pytest.mark.parametrize("seed", range(6))
def test_schedule_covers_every_visible_block_once(seed):
    rng = np.random.default_rng(seed)
    lengths = [int(x) for x in rng.integers(0, 1300, size=int(rng.integers(1, 9)))]
    lengths += [0, 1, 128, 129, 256]
    _check(lengths, None)
    cands = [int(rng.integers(0, L + 1)) for L in lengths]
    _check(lengths, cands)


def test_schedule_splits_a_lone_long_sequence_and_still_covers_once():
    # one long sequence among short ones, 2 heads: items above four times the
    # average work per SM are split into key-tile / query-block ranges
    lengths = [4096] + [64] * 20
    fwd, bwd = _check(lengths, None, heads=2)
    assert (fwd[:, 3] != UNSPLIT).any() and (bwd[:, 3] != UNSPLIT).any()
    _check(lengths, [512] + [8] * 20, heads=2)


def test_full_size_workload_is_never_split():
    fwd, bwd = _check([8192] * 4, None)
    assert (fwd[:, 3] == UNSPLIT).all() and (bwd[:, 3] == UNSPLIT).all()
    assert len(fwd) == 4 * 32 and len(bwd) == 4 * 64


def test_plan_rejects_small_capacity_and_reports_counts():
    import ctypes
    p = _params(1, 1, 64, 1000, False)
    off = np.array([0, 1000], dtype=np.int64)
    nf, nb = ctypes.c_int32(0), ctypes.c_int32(0)
    buf = np.zeros((1, 4), dtype=np.int32)
    rc = ops.LIB.hstu_debug_plan(ctypes.byref(p), off.ctypes.data, None, 1, buf.ctypes.data,
                                 ctypes.byref(nf), buf.ctypes.data, ctypes.byref(nb))
    assert rc == 1 and nf.value > 1 and nb.value > 1   # counts reported, nothing written
    cap = max(nf.value, nb.value)
    fi, bi = np.zeros((cap, 4), dtype=np.int32), np.zeros((cap, 4), dtype=np.int32)
    rc = ops.LIB.hstu_debug_plan(ctypes.byref(p), off.ctypes.data, None, cap, fi.ctypes.data,
                                 ctypes.byref(nf), bi.ctypes.data, ctypes.byref(nb))
    assert rc == 0 and max(nf.value, nb.value) == cap
