"""GPU parity of libhstu.so's attention (forward, backward, buckets) against
the CPU oracle, through the C ABI, element by element at small sizes and on
sampled outputs at the full workload sizes."""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_pointwise_attention_b200 import workloads as W

from gpu_common import (assert_close, gpu_bwd, gpu_fwd, oracle_bwd, oracle_fwd, problem_of,
                        sample_rows, to_device, kwargs_of)

pytestmark = pytest.mark.gpu


def attn(lengths, H=2, d=128, nb=128, s=2, seed=5, nc=None, dtype="bf16", **kw):
    return W.make_attention("case", lengths, H, d, nb, s, dtype, seed, num_candidates=nc,
                            with_grad=True, **kw)


RAGGED = [1, 37, 128, 129, 300, 513, 1000]


# ----------------------------------------------------------------------------
# Forward
# ----------------------------------------------------------------------------

def test_tiny_f32_forward():
    w = W.tiny_f32_fwd()
    assert_close(gpu_fwd(w), oracle_fwd(w), "f32", "tiny f32 fwd")


@pytest.mark.parametrize("impl", ["auto", "simt"])
@pytest.mark.parametrize("d", [64, 128])
def test_bf16_forward_ragged(impl, d):
    w = attn(RAGGED, d=d)
    assert_close(gpu_fwd(w, impl), oracle_fwd(w), "bf16", f"ragged d={d} {impl}")


@pytest.mark.parametrize("impl", ["auto", "simt"])
def test_bf16_forward_mfalcon(impl):
    w = attn([300, 640, 77, 1030], nc=[100, 128, 77, 6])
    assert_close(gpu_fwd(w, impl), oracle_fwd(w), "bf16", "mfalcon")


@pytest.mark.parametrize("kw", [
    dict(rab_per_head=True),
    dict(nb=32, s=0),
    dict(nb=256, s=3),
    dict(nb=8, s=1, nb_t=300),
    dict(time_gap_scale=50000.0),      # spans beyond 2^24 s: int64 time path
])
def test_bf16_forward_bias_variants(kw):
    w = attn([200, 333, 1], **kw)
    assert_close(gpu_fwd(w), oracle_fwd(w), "bf16", str(kw))


def test_forward_writes_every_row_and_empty_sequences():
    w = attn([0, 5, 0, 130, 0])
    assert_close(gpu_fwd(w), oracle_fwd(w), "bf16", "empty sequences")


def test_forward_all_candidates_and_no_candidates():
    w = attn([129, 200], nc=[129, 0])
    assert_close(gpu_fwd(w), oracle_fwd(w), "bf16", "all candidates")


def test_forward_causality_on_gpu():
    """Changing future tokens leaves earlier outputs bit-identical."""
    w = attn([700])
    base = gpu_fwd(w)
    w2 = attn([700])
    w2.k[400:] = W.round_bf16(w2.k[400:] * 1.5)
    w2.v[400:] = W.round_bf16(-w2.v[400:])
    out = gpu_fwd(w2)
    np.testing.assert_array_equal(out[:400], base[:400])


def test_forward_jagged_independence_on_gpu():
    w = attn([300, 500, 260])
    base = gpu_fwd(w)
    w.q[300:800] = W.round_bf16(w.q[300:800] * -1.0)
    w.v[300:800] = W.round_bf16(w.v[300:800] * 2.0)
    out = gpu_fwd(w)
    np.testing.assert_array_equal(out[:300], base[:300])
    np.testing.assert_array_equal(out[800:], base[800:])


def test_mfalcon_candidates_independent_on_gpu():
    w = attn([512 + 300], nc=[300])
    base = gpu_fwd(w)
    w.k[600:] = W.round_bf16(w.k[600:] + 1.0)
    w.v[600:] = W.round_bf16(w.v[600:] * 3.0)
    out = gpu_fwd(w)
    np.testing.assert_array_equal(out[:600], base[:600])


# ----------------------------------------------------------------------------
# Backward
# ----------------------------------------------------------------------------

def test_tiny_f32_backward():
    w = W.tiny_f32_fwd()
    got = gpu_bwd(w)
    want = oracle_bwd(w)
    for g, r, name in zip(got, want, ("dq", "dk", "dv", "drab_p", "drab_t")):
        assert_close(g, r, "f32", name)


@pytest.mark.parametrize("impl", ["auto", "simt"])
@pytest.mark.parametrize("d", [64, 128])
def test_bf16_backward_ragged(impl, d):
    w = attn(RAGGED[:6], d=d)
    got = gpu_bwd(w, impl)
    want = oracle_bwd(w)
    for g, r, name in zip(got, want, ("dq", "dk", "dv", "drab_p", "drab_t")):
        assert_close(g, r, "bf16", f"{name} d={d} {impl}")


@pytest.mark.parametrize("impl", ["auto", "simt"])
def test_bf16_backward_mfalcon(impl):
    w = attn([300, 640, 77], nc=[100, 128, 77])
    got = gpu_bwd(w, impl)
    want = oracle_bwd(w)
    for g, r, name in zip(got, want, ("dq", "dk", "dv", "drab_p", "drab_t")):
        assert_close(g, r, "bf16", name)


@pytest.mark.parametrize("kw", [dict(rab_per_head=True), dict(time_gap_scale=50000.0),
                                dict(nb=256, s=3)])
def test_bf16_backward_bias_variants(kw):
    w = attn([260, 131], **kw)
    got = gpu_bwd(w)
    want = oracle_bwd(w)
    for g, r, name in zip(got, want, ("dq", "dk", "dv", "drab_p", "drab_t")):
        assert_close(g, r, "bf16", f"{name} {kw}")


# ----------------------------------------------------------------------------
# Integer work: buckets bit-exact
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("case", ["tiny", "mfalcon", "wide", "edges"])
def test_buckets_bit_exact(case):
    from hstu_pointwise_attention_b200 import ops
    if case == "tiny":
        w = W.tiny_f32_fwd()
    elif case == "mfalcon":
        w = attn([70, 140], nc=[20, 40], nb=64, s=2)
    elif case == "wide":
        w = attn([90, 50], time_gap_scale=3e5, nb=256, s=3)
    else:
        w = attn([9], nb=16, s=2)
        # dt = 0, 1, 2, 3, 2^k - 1, 2^k, near 2^24, and a decreasing step (dt < 0)
        w.timestamps = np.array([0, 0, 1, 3, 2, 10, 2**20 - 1, 2**23, 2**24 - 2],
                                np.int64) + 1_700_000_000
    ts = torch.from_numpy(w.timestamps).cuda()
    bp, bt, btf = ops.debug_buckets(w.offsets, ts, num_heads=w.num_heads, d_qk=w.d_qk,
                                    d_v=w.d_v, max_seq_len=w.max_seq_len,
                                    num_pos_buckets=w.num_pos_buckets,
                                    num_time_buckets=w.num_time_buckets,
                                    time_bucket_sub_bits=w.time_bucket_sub_bits,
                                    num_candidates=w.num_candidates)
    ref = O.buckets(problem_of(w))
    want_p = np.concatenate([r[0].ravel() for r in ref])
    want_t = np.concatenate([r[1].ravel() for r in ref])
    np.testing.assert_array_equal(bp.cpu().numpy(), want_p)
    np.testing.assert_array_equal(bt.cpu().numpy(), want_t)
    fast = btf.cpu().numpy()
    vis = want_t >= 0
    np.testing.assert_array_equal(fast[~vis], want_t[~vis])   # -1 where not visible
    if case == "wide":
        assert np.all(fast[vis] == -2)    # span beyond 2^24 s: no float path
    else:
        np.testing.assert_array_equal(fast, want_t)


# ----------------------------------------------------------------------------
# Full workload sizes, sampled outputs
# ----------------------------------------------------------------------------

def _full_size_check(w, rows_per_seq, kv_per_seq, seed, band):
    d = to_device(w)
    out = gpu_fwd(w, dev_inputs=d)
    rows = sample_rows(w, rows_per_seq, seed)
    assert_close(out[rows], oracle_fwd(w, rows=rows), "bf16", f"{w.name} fwd rows")
    dq, dk, dv, drp, drt = gpu_bwd(w, dev_inputs=d)
    cols = sample_rows(w, kv_per_seq, seed + 1)
    oq, ok, ov, odrp = O.attn_bwd_sampled(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t,
                                          w.dout, dq_rows=rows, kv_cols=cols,
                                          drab_p_band=band)
    assert_close(dq[rows], oq, "bf16", "dq rows")
    assert_close(dk[cols], ok, "bf16", "dk cols")
    assert_close(dv[cols], ov, "bf16", "dv cols")
    assert_close(drp[..., :band], odrp[..., :band], "bf16", "drab_p band")
    # every pair adds its dS once to each table
    tot_p, tot_t = float(drp.sum()), float(drt.sum())
    assert abs(tot_p - tot_t) <= 2e-2 * max(abs(tot_p), float(np.abs(drt).max()), 1e-30)


def test_zipf_workload_full_size():
    _full_size_check(W.zipf_bf16_fwd_bwd(), 24, 12, seed=7, band=48)


def test_long_workload_full_size():
    _full_size_check(W.long_bf16_fwd_bwd(), 24, 12, seed=8, band=32)


# ----------------------------------------------------------------------------
# All five gradients in full against the oracle: every bias-table bucket,
# including the saturated last position bucket, the long-range time buckets
# and the run flushes that only long rows reach
# ----------------------------------------------------------------------------

def _all_gradients_check(w, fwd_too=False):
    d = to_device(w)
    p = problem_of(w)
    if fwd_too:
        assert_close(gpu_fwd(w, dev_inputs=d), oracle_fwd(w), "bf16", f"{w.name} fwd (all rows)")
    dq, dk, dv, drp, drt = gpu_bwd(w, dev_inputs=d)
    every = np.arange(w.total_tokens, dtype=np.int64)
    oq, ok, ov, _ = O.attn_bwd_sampled(p, w.q, w.k, w.v, w.rab_p, w.rab_t, w.dout,
                                       dq_rows=every, kv_cols=every)
    odrp, odrt = O.attn_drab(p, w.q, w.k, w.v, w.rab_p, w.rab_t, w.dout)
    assert_close(dq, oq, "bf16", f"{w.name} dq (all rows)")
    assert_close(dk, ok, "bf16", f"{w.name} dk (all rows)")
    assert_close(dv, ov, "bf16", f"{w.name} dv (all rows)")
    assert_close(drp, odrp, "bf16", f"{w.name} drab_p (every bucket)")
    assert_close(drt, odrt, "bf16", f"{w.name} drab_t (every bucket)")
    # the full-size sequence reaches the saturated position bucket and many time buckets
    assert np.count_nonzero(odrt) > w.num_time_buckets // 4


def test_long_sequence_all_five_gradients_in_full():
    """One 8192-token sequence with the long workload's settings (2 heads,
    d 128, 256 position + 256 time buckets, sub_bits 3)."""
    w = W.make_attention("long_one_seq", [8192], 2, 128, 256, 3, "bf16", seed=9,
                         max_seq_len=8192, with_grad=True)
    _all_gradients_check(w, fwd_too=True)


def test_zipf_workload_all_five_gradients_in_full():
    _all_gradients_check(W.zipf_bf16_fwd_bwd(), fwd_too=True)


def test_prefix_context_tokens_forward_and_backward():
    """Context tokens at the head of every sequence (the same timestamp as the
    first event) ahead of the events, with and without candidates: ordinary
    tokens of the causal sequence, so the whole path must match the oracle."""
    for nc in (None, [40, 3, 0]):
        w = attn([300, 129, 70], nc=nc, num_prefix=8)
        assert_close(gpu_fwd(w), oracle_fwd(w), "bf16", f"prefix fwd nc={nc}")
        for g, r, name in zip(gpu_bwd(w), oracle_bwd(w), ("dq", "dk", "dv", "drab_p", "drab_t")):
            assert_close(g, r, "bf16", f"prefix {name} nc={nc}")


@pytest.mark.parametrize("nc", [None, [300, 20, 1]])
def test_short_batch_split_items_match_oracle(nc):
    """A batch too small to fill the GPU: one head, one long sequence and two
    short ones.  The schedule splits the long sequence's work items (forward
    query-tile pairs over key ranges, backward key tiles over query runs) and
    adds the pieces' float32 partial sums; every output must still match."""
    w = attn([2048, 100, 1], H=1, nc=nc, seed=71)
    assert_close(gpu_fwd(w), oracle_fwd(w), "bf16", f"split fwd nc={nc}")
    for g, r, name in zip(gpu_bwd(w), oracle_bwd(w), ("dq", "dk", "dv", "drab_p", "drab_t")):
        assert_close(g, r, "bf16", f"split {name} nc={nc}")
