"""Pins of the CPU oracle against things other than itself.

Every check here is independent of the oracle's own code: a pure-Python
brute-force evaluator written separately from the definition, a numpy dense
restatement, hand-derived bucket tables (tests/golden/), closed forms,
invariants that the definition implies, and finite differences.  A dropped
term, a wrong sign or index, or a transposed operand in the oracle fails at
least one of them.

Definition pinned (DLRMv4 article, section "Model architecture: HSTU replaces
the feature-interaction stack"; readings R1-R11 of the design notes): see
oracle/hstu_oracle.h.
"""
import math
import os

import numpy as np
import pytest

from oracle import hstu_oracle as O
from hstu_pointwise_attention_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def problem_of(w: W.AttnWorkload) -> O.Problem:
    return O.Problem(offsets=w.offsets, timestamps=w.timestamps, num_heads=w.num_heads,
                     d_qk=w.d_qk, d_v=w.d_v, num_pos_buckets=w.num_pos_buckets,
                     num_time_buckets=w.num_time_buckets,
                     time_bucket_sub_bits=w.time_bucket_sub_bits, alpha=w.alpha,
                     silu_scale=w.silu_scale, num_candidates=w.num_candidates,
                     rab_per_head=w.rab_per_head)


# --------------------------------------------------------------------------
# Independent pure-Python restatement (python ints, math.exp, explicit loops)
# --------------------------------------------------------------------------

def py_time_bucket(dt: int, s: int, nb: int) -> int:
    if dt <= 0:
        b = 0
    elif dt < (1 << s):
        b = dt
    else:
        e = dt.bit_length() - 1
        b = (e - s + 1) * (1 << s) + (dt >> (e - s)) - (1 << s)
    return min(b, nb - 1)


def py_pairs(w, b):
    """Yield (i, j, bp, bt) for the visible pairs of sequence b (local indices)."""
    o, L = int(w.offsets[b]), int(w.offsets[b + 1] - w.offsets[b])
    nc = 0 if w.num_candidates is None else int(w.num_candidates[b])
    nh = L - nc
    for i in range(L):
        for j in range(L):
            vis = (j <= i) if i < nh else (j < nh or j == i)
            if not vis:
                continue
            pi = i if i < nh else nh
            pj = j if j < nh else nh
            bp = min(w.num_pos_buckets - 1, pi - pj)
            bt = py_time_bucket(int(w.timestamps[o + i]) - int(w.timestamps[o + j]),
                                w.time_bucket_sub_bits, w.num_time_buckets)
            yield i, j, bp, bt


def py_tables(w, h):
    rp = w.rab_p[h] if w.rab_per_head else w.rab_p
    rt = w.rab_t[h] if w.rab_per_head else w.rab_t
    return [float(x) for x in rp], [float(x) for x in rt]


def py_logit(w, h, gi, gj, bp, bt):
    rp, rt = py_tables(w, h)
    dot = 0.0
    for c in range(w.d_qk):
        dot += float(w.q[gi, h, c]) * float(w.k[gj, h, c])
    return w.alpha * dot + rp[bp] + rt[bt]


def py_fwd(w):
    T, H = w.total_tokens, w.num_heads
    out = [[[0.0] * w.d_v for _ in range(H)] for _ in range(T)]
    for b in range(w.batch):
        o = int(w.offsets[b])
        for h in range(H):
            for i, j, bp, bt in py_pairs(w, b):
                s = py_logit(w, h, o + i, o + j, bp, bt)
                a = w.silu_scale * s / (1.0 + math.exp(-s))
                for c in range(w.d_v):
                    out[o + i][h][c] += a * float(w.v[o + j, h, c])
    return np.array(out)


def tiny(lengths=(3, 5, 1), H=2, d=3, nb=4, s=1, seed=11, nc=None, per_head=False, dv=None,
         dtype="f32", nb_t=None):
    return W.make_attention("tiny", list(lengths), H, d, nb, s, dtype, seed, num_candidates=nc,
                            with_grad=True, rab_per_head=per_head, d_v=dv, nb_t=nb_t)


# --------------------------------------------------------------------------
# Integer parts: buckets, positions, visibility
# --------------------------------------------------------------------------

def test_time_bucket_matches_hand_table():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "time_buckets.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) > 30
    for dt, s, nb, want in rows:
        assert O.time_bucket(int(dt), int(s), int(nb)) == int(want), (dt, s, nb)


def test_time_bucket_sub_bits_zero_is_bit_length():
    rng = np.random.default_rng(5)
    for dt in list(range(-3, 300)) + [int(x) for x in rng.integers(1, 2**62, 200)]:
        want = min(31, max(0, int(dt)).bit_length())
        assert O.time_bucket(dt, 0, 32) == want


@pytest.mark.parametrize("s", [1, 2, 3, 4])
def test_time_bucket_octaves_split_evenly(s):
    """Each octave [2^e, 2^(e+1)), e >= s, is cut into 2^s equal buckets and
    bucket(2^e) = (e - s + 1) 2^s; below 2^s every integer has its own bucket."""
    nb = 1 << 20
    for dt in range(1, 1 << s):
        assert O.time_bucket(dt, s, nb) == dt
    for e in range(s, 40):
        base = O.time_bucket(1 << e, s, nb)
        assert base == (e - s + 1) << s
        width = 1 << (e - s)
        for m in range(1 << s):
            lo = (1 << e) + m * width
            assert O.time_bucket(lo, s, nb) == base + m
            assert O.time_bucket(lo + width - 1, s, nb) == base + m


def test_time_bucket_monotone_and_saturating():
    prev = 0
    for dt in range(0, 5000):
        b = O.time_bucket(dt, 2, 40)
        assert prev <= b <= 39
        prev = b
    assert O.time_bucket(2**62, 2, 40) == 39


def test_pos_bucket():
    assert [O.pos_bucket(d, 5) for d in range(0, 9)] == [0, 1, 2, 3, 4, 4, 4, 4, 4]


def test_visibility_and_position_mfalcon_by_hand():
    # L = 6, n_hist = 4: history causal, candidates 4 and 5 see history + self.
    want = {(i, j) for i in range(4) for j in range(i + 1)}
    want |= {(4, 0), (4, 1), (4, 2), (4, 3), (4, 4), (5, 0), (5, 1), (5, 2), (5, 3), (5, 5)}
    got = {(i, j) for i in range(6) for j in range(6) if O.visible(i, j, 4)}
    assert got == want
    assert [O.position(i, 4) for i in range(6)] == [0, 1, 2, 3, 4, 4]


def test_bucket_matrices_match_brute_force():
    for w in (tiny(), tiny(lengths=(7, 6), nc=[2, 3]), W.tiny_f32_fwd()):
        got = O.buckets(problem_of(w))
        for b in range(w.batch):
            L = int(w.lengths[b])
            bp = -np.ones((L, L), np.int32)
            bt = -np.ones((L, L), np.int32)
            for i, j, p_, t_ in py_pairs(w, b):
                bp[i, j], bt[i, j] = p_, t_
            np.testing.assert_array_equal(got[b][0], bp)
            np.testing.assert_array_equal(got[b][1], bt)


# --------------------------------------------------------------------------
# Forward
# --------------------------------------------------------------------------

@pytest.mark.parametrize("kw", [
    dict(),
    dict(lengths=(6, 4), nc=[2, 1]),
    dict(per_head=True, dv=5),
    dict(lengths=(9,), nb=3, s=0, nb_t=6),
    dict(lengths=(1, 2, 1)),
])
def test_fwd_matches_brute_force(kw):
    w = tiny(**kw)
    got = O.attn_fwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t)
    want = py_fwd(w)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-15)


def dense_fwd_numpy(w):
    """Dense restatement: S = alpha Q K^T + B (B gathered from bucket matrices), A = mask *
    silu_scale * S sigmoid(S), O = A V, per sequence and head with numpy einsum."""
    outs = []
    for b in range(w.batch):
        o, L = int(w.offsets[b]), int(w.lengths[b])
        mask = np.zeros((L, L), bool)
        bpm = np.zeros((L, L), np.int64)
        btm = np.zeros((L, L), np.int64)
        for i, j, p_, t_ in py_pairs(w, b):
            mask[i, j], bpm[i, j], btm[i, j] = True, p_, t_
        q = w.q[o:o + L].astype(np.float64)
        k = w.k[o:o + L].astype(np.float64)
        v = w.v[o:o + L].astype(np.float64)
        s = w.alpha * np.einsum("ihc,jhc->hij", q, k)
        for h in range(w.num_heads):
            rp, rt = (w.rab_p[h], w.rab_t[h]) if w.rab_per_head else (w.rab_p, w.rab_t)
            s[h] += rp.astype(np.float64)[bpm] + rt.astype(np.float64)[btm]
        a = np.where(mask[None], w.silu_scale * s / (1 + np.exp(-s)), 0.0)
        outs.append(np.einsum("hij,jhc->ihc", a, v))
    return np.concatenate(outs)


def test_fwd_matches_dense_numpy_tiny_f32_workload():
    w = W.tiny_f32_fwd()
    got = O.attn_fwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t)
    np.testing.assert_allclose(got, dense_fwd_numpy(w), rtol=1e-11, atol=1e-14)


def test_fwd_rows_subset_equals_full():
    w = tiny(lengths=(8, 5), nc=[3, 0])
    p = problem_of(w)
    full = O.attn_fwd(p, w.q, w.k, w.v, w.rab_p, w.rab_t)
    rows = np.array([12, 0, 7, 5])
    np.testing.assert_array_equal(O.attn_fwd(p, w.q, w.k, w.v, w.rab_p, w.rab_t, rows=rows),
                                  full[rows])


def test_fwd_single_token_closed_form():
    w = tiny(lengths=(1,), H=1, d=4)
    s = w.alpha * float(np.dot(w.q[0, 0].astype(np.float64), w.k[0, 0])) + \
        float(w.rab_p[0]) + float(w.rab_t[0])
    want = w.silu_scale * s / (1 + math.exp(-s)) * w.v[0, 0].astype(np.float64)
    got = O.attn_fwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t)[0, 0]
    np.testing.assert_allclose(got, want, rtol=1e-14)


def test_fwd_zero_query_gives_bias_only_weights():
    """q = 0: every logit is rab_p[bp] + rab_t[bt]; with both tables 0 the SiLU is 0."""
    w = tiny(lengths=(5,))
    w.q[:] = 0
    w.rab_p[:] = 0
    w.rab_t[:] = 0
    got = O.attn_fwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t)
    assert np.all(got == 0.0)


def test_causality():
    w = tiny(lengths=(9,), seed=3)
    p = problem_of(w)
    base = O.attn_fwd(p, w.q, w.k, w.v, w.rab_p, w.rab_t)
    for cut in (0, 4, 7):
        k2, v2, q2 = w.k.copy(), w.v.copy(), w.q.copy()
        k2[cut + 1:] += 1.0
        v2[cut + 1:] -= 2.0
        q2[cut + 1:] *= 3.0
        out = O.attn_fwd(p, q2, k2, v2, w.rab_p, w.rab_t)
        np.testing.assert_array_equal(out[:cut + 1], base[:cut + 1])
        assert not np.array_equal(out[cut + 1:], base[cut + 1:])


def test_jagged_independence():
    w = tiny(lengths=(4, 6, 3), seed=4)
    p = problem_of(w)
    base = O.attn_fwd(p, w.q, w.k, w.v, w.rab_p, w.rab_t)
    q2, k2, v2 = w.q.copy(), w.k.copy(), w.v.copy()
    q2[4:10] = -q2[4:10]
    k2[4:10] += 0.5
    v2[4:10] *= 2
    out = O.attn_fwd(p, q2, k2, v2, w.rab_p, w.rab_t)
    np.testing.assert_array_equal(out[:4], base[:4])
    np.testing.assert_array_equal(out[10:], base[10:])


def test_mfalcon_candidate_equals_history_plus_candidate_alone():
    nh, nc = 6, 3
    w = tiny(lengths=(nh + nc,), nc=[nc], seed=8)
    got = O.attn_fwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t)
    # other candidates do not influence candidate c
    for c in range(nc):
        idx = list(range(nh)) + [nh + c]
        sub = W.AttnWorkload(**{**w.__dict__, "offsets": np.array([0, nh + 1]),
                                "timestamps": w.timestamps[idx], "q": w.q[idx], "k": w.k[idx],
                                "v": w.v[idx], "num_candidates": None})
        alone = O.attn_fwd(problem_of(sub), sub.q, sub.k, sub.v, sub.rab_p, sub.rab_t)
        np.testing.assert_allclose(got[nh + c], alone[nh], rtol=1e-13, atol=1e-16)
        np.testing.assert_allclose(got[:nh], alone[:nh], rtol=1e-13, atol=1e-16)


def test_linearity_in_v():
    w = tiny(lengths=(5, 4), seed=9)
    p = problem_of(w)
    v2 = np.random.default_rng(0).standard_normal(w.v.shape)
    o1 = O.attn_fwd(p, w.q, w.k, w.v, w.rab_p, w.rab_t)
    o2 = O.attn_fwd(p, w.q, w.k, v2, w.rab_p, w.rab_t)
    o3 = O.attn_fwd(p, w.q, w.k, 2.0 * w.v - 3.0 * v2, w.rab_p, w.rab_t)
    np.testing.assert_allclose(o3, 2.0 * o1 - 3.0 * o2, rtol=1e-12, atol=1e-14)


def test_rab_shift_is_a_logit_shift():
    """Adding c to every position bucket or to every time bucket shifts every
    logit by c, so both give the same output."""
    w = tiny(lengths=(6, 3), seed=10)
    p = problem_of(w)
    rp, rt = w.rab_p.astype(np.float64), w.rab_t.astype(np.float64)
    a = O.attn_fwd(p, w.q, w.k, w.v, rp + 0.3, rt)
    b = O.attn_fwd(p, w.q, w.k, w.v, rp, rt + 0.3)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)
    c = O.attn_fwd(p, w.q, w.k, w.v, w.rab_p, w.rab_t)
    assert not np.allclose(a, c)


# --------------------------------------------------------------------------
# Backward: finite differences of the (brute-force-pinned) forward
# --------------------------------------------------------------------------

def _loss(p, w, q, k, v, rp, rt):
    return float((O.attn_fwd(p, q, k, v, rp, rt) * w.dout.astype(np.float64)).sum())


@pytest.mark.parametrize("kw", [dict(), dict(lengths=(5, 3), nc=[2, 0]),
                                dict(per_head=True, dv=2)])
def test_bwd_matches_finite_differences(kw):
    w = tiny(**kw)
    p = problem_of(w)
    args = [x.astype(np.float64) for x in (w.q, w.k, w.v, w.rab_p, w.rab_t)]
    grads = O.attn_bwd(p, *args, w.dout)
    eps = 1e-6
    for which in range(5):
        x = args[which]
        for flat in range(x.size):
            xp, xm = [a.copy() for a in args], [a.copy() for a in args]
            xp[which].flat[flat] += eps
            xm[which].flat[flat] -= eps
            fd = (_loss(p, w, *xp) - _loss(p, w, *xm)) / (2 * eps)
            an = grads[which].flat[flat]
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)) + 1e-9, (which, flat, fd, an)


def test_bwd_drab_sum_rule():
    """Every visible pair adds its dS once to drab_p and once to drab_t."""
    w = tiny(lengths=(7, 5), nc=[0, 2])
    _, _, _, drp, drt = O.attn_bwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t, w.dout)
    assert abs(drp.sum() - drt.sum()) <= 1e-12 * max(1.0, abs(drp.sum()))


def test_bwd_sampled_equals_full():
    w = tiny(lengths=(9, 6), nc=[3, 0], nb=5, seed=12)
    p = problem_of(w)
    dq, dk, dv, drp, _ = O.attn_bwd(p, w.q, w.k, w.v, w.rab_p, w.rab_t, w.dout)
    rows, cols = np.array([0, 8, 10, 3]), np.array([14, 2, 6, 7])
    sq, sk, sv, sdrp = O.attn_bwd_sampled(p, w.q, w.k, w.v, w.rab_p, w.rab_t, w.dout,
                                          dq_rows=rows, kv_cols=cols, drab_p_band=3)
    np.testing.assert_allclose(sq, dq[rows], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(sk, dk[cols], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(sv, dv[cols], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(sdrp[:3], drp[:3], rtol=1e-12, atol=1e-15)
    assert np.all(sdrp[3:] == 0)


@pytest.mark.parametrize("kw", [dict(), dict(per_head=True, lengths=(5, 3), nc=[2, 0])])
def test_drab_full_matches_finite_differences(kw):
    """attn_drab (both bias tables in full, work split by query rows) against
    central differences of the brute-force-pinned forward in the tables."""
    w = tiny(**kw)
    p = problem_of(w)
    args = [x.astype(np.float64) for x in (w.q, w.k, w.v, w.rab_p, w.rab_t)]
    drp, drt = O.attn_drab(p, *args, w.dout)
    eps = 1e-6
    for which, an_all in ((3, drp), (4, drt)):
        for flat in range(args[which].size):
            xp, xm = [a.copy() for a in args], [a.copy() for a in args]
            xp[which].flat[flat] += eps
            xm[which].flat[flat] -= eps
            fd = (_loss(p, w, *xp) - _loss(p, w, *xm)) / (2 * eps)
            an = an_all.flat[flat]
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)) + 1e-9, (which, flat, fd, an)


def test_drab_full_equals_full_backward_on_long_rows():
    """Several 64-row pieces per sequence, saturated position and time buckets,
    candidates: the row-split sums equal the full backward's tables."""
    w = tiny(lengths=(150, 70, 1), nc=[20, 0, 1], nb=8, seed=13)
    p = problem_of(w)
    _, _, _, drp, drt = O.attn_bwd(p, w.q, w.k, w.v, w.rab_p, w.rab_t, w.dout)
    fp, ft = O.attn_drab(p, w.q, w.k, w.v, w.rab_p, w.rab_t, w.dout)
    np.testing.assert_allclose(fp, drp, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(ft, drt, rtol=1e-11, atol=1e-14)
    assert np.abs(fp[-1]) > 0 and np.abs(ft).sum() > 0


# --------------------------------------------------------------------------
# Layer
# --------------------------------------------------------------------------

def py_layer(lw: W.LayerWorkload, layer: W.LayerWeights):
    """Per-token pure-Python restatement of one layer (loops, math.exp)."""
    a = lw.attn
    T, H, d, D = a.total_tokens, a.num_heads, a.d_qk, lw.d_model
    silu = lambda z: z / (1.0 + math.exp(-z))
    proj = [[silu(sum(float(lw.x[t, m]) * float(layer.w1[n, m]) for m in range(D))
                  + float(layer.b1[n])) for n in range(4 * H * d)] for t in range(T)]
    aw = W.AttnWorkload(**a.__dict__)
    aw.q = np.array([[proj[t][2 * H * d + h * d: 2 * H * d + (h + 1) * d] for h in range(H)]
                     for t in range(T)])
    aw.k = np.array([[proj[t][3 * H * d + h * d: 3 * H * d + (h + 1) * d] for h in range(H)]
                     for t in range(T)])
    aw.v = np.array([[proj[t][H * d + h * d: H * d + (h + 1) * d] for h in range(H)]
                     for t in range(T)])
    aw.rab_p, aw.rab_t = layer.rab_p, layer.rab_t
    att = py_fwd(aw)
    y = []
    for t in range(T):
        row = [float(att[t, h, c]) for h in range(H) for c in range(d)]
        mean = sum(row) / len(row)
        var = sum((r - mean) ** 2 for r in row) / len(row)
        g = [((row[n] - mean) / math.sqrt(var + lw.ln_eps) * float(layer.ln_gamma[n])
              + float(layer.ln_beta[n])) * proj[t][n] for n in range(H * d)]
        y.append([float(lw.x[t, m]) + float(layer.b2[m]) +
                  sum(g[n] * float(layer.w2[m, n]) for n in range(H * d)) for m in range(D)])
    return np.array(y)


def test_layer_matches_pure_python():
    lw = W.make_layer("tiny_layer", [4, 3], 2, 2, 5, 4, 1, seed=21, num_candidates=[1, 0])
    a, L0 = lw.attn, lw.layers[0]
    rng = np.random.default_rng(3)
    L0.b1 = rng.standard_normal(L0.b1.shape).astype(np.float32) * 0.1
    L0.b2 = rng.standard_normal(L0.b2.shape).astype(np.float32) * 0.1
    L0.ln_gamma = (1 + 0.1 * rng.standard_normal(L0.ln_gamma.shape)).astype(np.float32)
    L0.ln_beta = (0.1 * rng.standard_normal(L0.ln_beta.shape)).astype(np.float32)
    got = O.layer_fwd(problem_of(a), lw.x, L0.w1, L0.b1, L0.ln_gamma, L0.ln_beta, L0.w2, L0.b2,
                      L0.rab_p, L0.rab_t, ln_eps=lw.ln_eps)
    np.testing.assert_allclose(got, py_layer(lw, L0), rtol=1e-10, atol=1e-12)


def test_layer_zero_output_projection_is_identity_plus_bias():
    lw = W.make_layer("tiny_layer", [5], 2, 4, 6, 4, 1, seed=22)
    a, L0 = lw.attn, lw.layers[0]
    b2 = np.arange(6, dtype=np.float32)
    got = O.layer_fwd(problem_of(a), lw.x, L0.w1, L0.b1, L0.ln_gamma, L0.ln_beta,
                      np.zeros_like(L0.w2), b2, L0.rab_p, L0.rab_t)
    np.testing.assert_allclose(got, lw.x.astype(np.float64) + b2, rtol=0, atol=0)


# --------------------------------------------------------------------------
# Layer backward: central differences of the (pure-Python-pinned) layer_fwd
# --------------------------------------------------------------------------

def _layer_case(seed=31, nc=(1, 0), residual=True):
    lw = W.make_layer("tiny_layer_bwd", [4, 3], 2, 2, 6, 4, 1, seed=seed,
                      num_candidates=list(nc))
    rng = np.random.default_rng(seed + 1)
    L0 = lw.layers[0]
    L0.b1 = rng.standard_normal(L0.b1.shape) * 0.1
    L0.b2 = rng.standard_normal(L0.b2.shape) * 0.1
    L0.ln_gamma = 1 + 0.1 * rng.standard_normal(L0.ln_gamma.shape)
    L0.ln_beta = 0.1 * rng.standard_normal(L0.ln_beta.shape)
    L0.rab_p = rng.standard_normal(L0.rab_p.shape) * 0.3
    L0.rab_t = rng.standard_normal(L0.rab_t.shape) * 0.3
    dy = rng.standard_normal(lw.x.shape)
    lw.residual = residual
    return lw, L0, dy


@pytest.mark.parametrize("residual", [True, False])
def test_layer_bwd_matches_finite_differences(residual):
    lw, L0, dy = _layer_case(residual=residual)
    p = problem_of(lw.attn)
    args = [np.asarray(a, np.float64) for a in (lw.x, L0.w1, L0.b1, L0.ln_gamma, L0.ln_beta,
                                                 L0.w2, L0.b2, L0.rab_p, L0.rab_t)]

    def loss(a):
        y = O.layer_fwd(p, *a, ln_eps=lw.ln_eps, residual=residual)
        return float((y * dy).sum())

    grads = O.layer_bwd(p, *args, dy, ln_eps=lw.ln_eps, residual=residual)
    eps = 1e-6
    for which in range(len(args)):
        for flat in range(args[which].size):
            xp, xm = [a.copy() for a in args], [a.copy() for a in args]
            xp[which].flat[flat] += eps
            xm[which].flat[flat] -= eps
            fd = (loss(xp) - loss(xm)) / (2 * eps)
            an = grads[which].flat[flat]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)) + 1e-8, (which, flat, fd, an)


# --------------------------------------------------------------------------
# M-FALCON micro-batches against a cached history
# --------------------------------------------------------------------------

def _py_candidate_out(w, b, c_rows, c):
    """Pure-Python restatement for one candidate c (global row in w) of
    sequence b whose history is w's first n_h tokens: its attention over the
    history and itself, position n_h."""
    o = int(w.offsets[b])
    nh = int(w.lengths[b]) - int(w.num_candidates[b])
    H, d = w.num_heads, w.d_v
    out = np.zeros((H, d))
    for h in range(H):
        for j in list(range(nh)) + [c]:
            jj = o + j if j < nh else c
            dot = sum(float(w.q[c, h, e]) * float(w.k[jj, h, e]) for e in range(w.d_qk))
            dp = nh - (j if j < nh else nh)
            bp = min(w.num_pos_buckets - 1, dp)
            bt = O.time_bucket(int(w.timestamps[c]) - int(w.timestamps[jj]),
                               w.time_bucket_sub_bits, w.num_time_buckets)
            s = w.alpha * dot + float(w.rab_p[bp]) + float(w.rab_t[bt])
            a = w.silu_scale * s / (1.0 + math.exp(-s))
            out[h] += a * w.v[jj, h].astype(np.float64)
    return out


def _split_candidates(w, sizes):
    """Cut every sequence's candidates into micro-batches of the given sizes."""
    hist, batches = [], []
    for b in range(w.batch):
        o, L, nc = int(w.offsets[b]), int(w.lengths[b]), int(w.num_candidates[b])
        hist.append((o, o + L - nc))
        c, mb = o + L - nc, []
        for n in sizes:
            mb.append((c, min(c + n, o + L)))
            c = min(c + n, o + L)
        mb.append((c, o + L))
        batches.append(mb)
    return hist, batches


@pytest.mark.parametrize("sizes", [(1,), (2, 3), (100,)])
def test_candidate_microbatches_equal_one_pass_mfalcon(sizes):
    """Scoring candidates in micro-batches against the cached history gives
    every candidate the one-pass M-FALCON output; a pure-Python restatement
    pins one candidate per sequence."""
    w = tiny(lengths=(9, 7, 4), nc=[4, 5, 4], nb=6, seed=17)
    p = problem_of(w)
    full = O.attn_fwd(p, w.q, w.k, w.v, w.rab_p, w.rab_t)
    hist, batches = _split_candidates(w, sizes)
    hidx = np.concatenate([np.arange(a, b) for a, b in hist]).astype(np.int64)
    hoff = np.concatenate([[0], np.cumsum([b - a for a, b in hist])]).astype(np.int64)
    for m in range(len(batches[0])):
        cidx = np.concatenate([np.arange(*batches[b][m]) for b in range(w.batch)]).astype(np.int64)
        coff = np.concatenate([[0], np.cumsum([batches[b][m][1] - batches[b][m][0]
                                               for b in range(w.batch)])]).astype(np.int64)
        got = O.attn_fwd_candidates(p, hoff, coff, w.timestamps[hidx], w.timestamps[cidx],
                                    w.q[cidx], w.k[cidx], w.v[cidx], w.k[hidx], w.v[hidx],
                                    w.rab_p, w.rab_t)
        np.testing.assert_allclose(got, full[cidx], rtol=1e-12, atol=1e-14)
    for b in range(w.batch):
        c = int(w.offsets[b + 1]) - 1
        np.testing.assert_allclose(_py_candidate_out(w, b, None, c), full[c], rtol=1e-12,
                                   atol=1e-14)


def test_candidate_layer_stack_equals_one_pass_stack():
    """Two stacked layers: a causal history pass keeping each layer's
    projection, then candidate micro-batches layer by layer, give the
    candidates the one-pass M-FALCON stack's outputs."""
    lw = W.make_layer("tiny_mf", [6, 5], 2, 2, 6, 4, 1, seed=23, n_layers=2,
                      num_candidates=[3, 2])
    a = lw.attn
    p = problem_of(a)
    x = lw.x.astype(np.float64)
    for L in lw.layers:
        x = O.layer_fwd(p, x, L.w1, L.b1, L.ln_gamma, L.ln_beta, L.w2, L.b2, L.rab_p, L.rab_t,
                        ln_eps=lw.ln_eps, residual=lw.residual)
    one_pass = x
    nh = [int(L) - int(c) for L, c in zip(a.lengths, a.num_candidates)]
    hidx = np.concatenate([np.arange(a.offsets[b], a.offsets[b] + nh[b])
                           for b in range(a.batch)]).astype(np.int64)
    hoff = np.concatenate([[0], np.cumsum(nh)]).astype(np.int64)
    ph = O.Problem(offsets=hoff, timestamps=a.timestamps[hidx], num_heads=a.num_heads,
                   d_qk=a.d_qk, d_v=a.d_v, num_pos_buckets=a.num_pos_buckets,
                   num_time_buckets=a.num_time_buckets,
                   time_bucket_sub_bits=a.time_bucket_sub_bits, alpha=a.alpha,
                   silu_scale=a.silu_scale)
    xh, projs = lw.x[hidx].astype(np.float64), []
    for L in lw.layers:
        projs.append(O.layer_proj(xh, L.w1, L.b1))
        xh = O.layer_fwd(ph, xh, L.w1, L.b1, L.ln_gamma, L.ln_beta, L.w2, L.b2, L.rab_p,
                         L.rab_t, ln_eps=lw.ln_eps, residual=lw.residual)
    for cut in (1, 2):      # candidates split into micro-batches of `cut` per sequence
        for m in range(3):
            rows = [np.arange(a.offsets[b] + nh[b] + m * cut,
                              min(a.offsets[b] + nh[b] + (m + 1) * cut, a.offsets[b + 1]))
                    for b in range(a.batch)]
            cidx = np.concatenate(rows).astype(np.int64)
            if cidx.size == 0:
                continue
            coff = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int64)
            xc = lw.x[cidx].astype(np.float64)
            for L, hp in zip(lw.layers, projs):
                xc = O.layer_fwd_candidates(p, hoff, coff, a.timestamps[hidx],
                                            a.timestamps[cidx], xc, hp, L.w1, L.b1, L.ln_gamma,
                                            L.ln_beta, L.w2, L.b2, L.rab_p, L.rab_t,
                                            ln_eps=lw.ln_eps, residual=lw.residual)
            np.testing.assert_allclose(xc, one_pass[cidx], rtol=1e-10, atol=1e-12)


def test_prefix_tokens_are_a_causal_head_with_zero_time_distance():
    """Prefix context tokens (the first event's timestamp) ahead of the events:
    their outputs depend on nothing after them, they all lie in time bucket 0
    of one another, and each prefix token's output is the closed form over
    the prefix tokens before it."""
    w = tiny(lengths=(9,), nb=6, seed=19)
    w2 = W.make_attention("tiny_prefix", [9], w.num_heads, w.d_qk, 6, 1, "f32", 19,
                          with_grad=True, num_prefix=4)
    p = problem_of(w2)
    (bp, bt), = O.buckets(p)
    assert np.all(bt[:4, :4][np.tril_indices(4)] == 0)
    out = O.attn_fwd(p, w2.q, w2.k, w2.v, w2.rab_p, w2.rab_t)
    w3 = W.AttnWorkload(**w2.__dict__)
    w3.k = w2.k.copy(); w3.v = w2.v.copy()
    w3.k[4:] += 1.0; w3.v[4:] *= -2.0
    out3 = O.attn_fwd(problem_of(w3), w3.q, w3.k, w3.v, w3.rab_p, w3.rab_t)
    np.testing.assert_array_equal(out[:4], out3[:4])
    for i in range(4):
        for h in range(w2.num_heads):
            want = np.zeros(w2.d_v)
            for j in range(i + 1):
                s = (w2.alpha * float(np.dot(w2.q[i, h].astype(np.float64), w2.k[j, h]))
                     + float(w2.rab_p[min(5, i - j)]) + float(w2.rab_t[0]))
                want += w2.silu_scale * s / (1 + math.exp(-s)) * w2.v[j, h].astype(np.float64)
            np.testing.assert_allclose(out[i, h], want, rtol=1e-12, atol=1e-15)
