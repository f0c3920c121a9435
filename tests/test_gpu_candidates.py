"""GPU parity of the M-FALCON candidate path: candidate micro-batches scored
against cached history keys and values (hstu_attn_fwd_candidates) and the
candidate-only layer (hstu_layer_fwd_candidates after a history pass with
hstu_layer_fwd_keep_proj), against the oracle and against the one-pass
M-FALCON forward on the GPU: every candidate must get the one-pass output,
whatever the micro-batch split."""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_pointwise_attention_b200 import workloads as W

from gpu_common import assert_close, gpu_fwd, problem_of, to_device

pytestmark = pytest.mark.gpu


def _views(w: W.AttnWorkload):
    """Global row indices of every sequence's history and candidates."""
    hist, cand = [], []
    for b in range(w.batch):
        o, L = int(w.offsets[b]), int(w.lengths[b])
        nc = int(w.num_candidates[b])
        hist.append(np.arange(o, o + L - nc))
        cand.append(np.arange(o + L - nc, o + L))
    return hist, cand


def _offsets(parts):
    return np.concatenate([[0], np.cumsum([len(x) for x in parts])]).astype(np.int64)


def _micro(cand, m, size):
    return [c[m * size:(m + 1) * size] for c in cand]


def gpu_candidates(w, d, hist, mb):
    from hstu_pointwise_attention_b200 import ops
    hidx = np.concatenate(hist).astype(np.int64)
    cidx = np.concatenate(mb).astype(np.int64)
    th, tc = torch.from_numpy(hidx).cuda(), torch.from_numpy(cidx).cuda()
    out = ops.attn_fwd_candidates(d["q"][tc], d["k"][tc], d["v"][tc], d["k"][th], d["v"][th],
                                  _offsets(hist), _offsets(mb), d["ts"][th], d["ts"][tc],
                                  d["rab_p"], d["rab_t"], max_seq_len=w.max_seq_len,
                                  time_bucket_sub_bits=w.time_bucket_sub_bits, alpha=w.alpha,
                                  silu_scale=w.silu_scale, rab_per_head=w.rab_per_head)
    torch.cuda.synchronize()
    return cidx, out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("d_head, size", [(128, 64), (128, 1000), (64, 100)])
def test_attention_candidates_match_one_pass_and_oracle(d_head, size):
    # ragged: no history, tile-edge histories and candidate counts, one candidate
    w = W.make_attention("cand", [1 + 3, 128 + 129, 300 + 1, 513 + 200, 0 + 5], 2, d_head, 128,
                         2, "bf16", seed=61, num_candidates=[3, 129, 1, 200, 5],
                         max_seq_len=713)
    d = to_device(w)
    one_pass = gpu_fwd(w, dev_inputs=d)
    ref = O.attn_fwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t)
    hist, cand = _views(w)
    n_mb = (max(len(c) for c in cand) + size - 1) // size
    for m in range(n_mb):
        cidx, got = gpu_candidates(w, d, hist, _micro(cand, m, size))
        if cidx.size == 0:
            continue
        assert_close(got, ref[cidx], "bf16", f"micro-batch {m} vs oracle")
        assert_close(got, one_pass[cidx], "bf16", f"micro-batch {m} vs one-pass GPU")


@pytest.mark.parametrize("n_users", [2, 20])
def test_attention_candidates_split_and_unsplit_history(n_users):
    # 2 users x 8 heads leave most SMs idle, so each pair's history key tiles
    # are split into ranges whose partial outputs are summed; 20 users x 8
    # heads fill a wave and stay unsplit.  Both must give the oracle's and
    # the one-pass output.
    rng = np.random.default_rng(71)
    hist_len = [int(x) for x in rng.integers(130, 700, size=n_users)]
    n_cand = [int(x) for x in rng.integers(1, 200, size=n_users)]
    lengths = [h + c for h, c in zip(hist_len, n_cand)]
    w = W.make_attention("cand_split", lengths, 8, 128, 128, 2, "bf16", seed=72,
                         num_candidates=n_cand, max_seq_len=max(lengths))
    d = to_device(w)
    one_pass = gpu_fwd(w, dev_inputs=d)
    ref = O.attn_fwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t)
    hist, cand = _views(w)
    cidx, got = gpu_candidates(w, d, hist, cand)
    assert_close(got, ref[cidx], "bf16", "candidates vs oracle")
    assert_close(got, one_pass[cidx], "bf16", "candidates vs one-pass GPU")


def test_attention_candidates_bias_variants():
    w = W.make_attention("cand_b", [400 + 64, 90 + 30], 2, 128, 256, 3, "bf16", seed=62,
                         num_candidates=[64, 30], max_seq_len=464, rab_per_head=True)
    d = to_device(w)
    ref = O.attn_fwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t)
    hist, cand = _views(w)
    cidx, got = gpu_candidates(w, d, hist, cand)
    assert_close(got, ref[cidx], "bf16", "per-head tables, 256 buckets")


def test_attention_candidates_wide_time_span():
    # history spans beyond 2^24 s: the exact int64 time path
    w = W.make_attention("cand_w", [300 + 40], 2, 128, 128, 2, "bf16", seed=63,
                         num_candidates=[40], time_gap_scale=50000.0)
    d = to_device(w)
    ref = O.attn_fwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t)
    hist, cand = _views(w)
    cidx, got = gpu_candidates(w, d, hist, cand)
    assert_close(got, ref[cidx], "bf16", "int64 times")


def _dev(z, dt=torch.bfloat16):
    return torch.from_numpy(np.ascontiguousarray(z)).cuda().to(dt)


def _params(L):
    f32 = torch.float32
    return (_dev(L.w1), _dev(L.b1, f32), _dev(L.ln_gamma, f32), _dev(L.ln_beta, f32),
            _dev(L.w2), _dev(L.b2, f32), _dev(L.rab_p, f32), _dev(L.rab_t, f32))


def gpu_candidate_stack(lw, mb_size):
    """History pass keeping each layer's projection, then candidate
    micro-batches of mb_size per sequence through every layer."""
    from hstu_pointwise_attention_b200 import ops
    a = lw.attn
    hist, cand = _views(a)
    hidx = np.concatenate(hist).astype(np.int64)
    hoff = _offsets(hist)
    ts = torch.from_numpy(a.timestamps).cuda()
    th = torch.from_numpy(hidx).cuda()
    kw = dict(num_heads=a.num_heads, d_qk=a.d_qk, d_v=a.d_v, max_seq_len=a.max_seq_len,
              time_bucket_sub_bits=a.time_bucket_sub_bits, alpha=a.alpha,
              silu_scale=a.silu_scale, ln_eps=lw.ln_eps, residual=lw.residual)
    xh = _dev(lw.x)[th]
    projs = []
    for L in lw.layers:
        xh, proj = ops.layer_fwd_keep_proj(xh, *_params(L), hoff, ts[th], **kw)
        projs.append(proj)
    out = {}
    n_mb = (max(len(c) for c in cand) + mb_size - 1) // mb_size
    for m in range(n_mb):
        mb = _micro(cand, m, mb_size)
        cidx = np.concatenate(mb).astype(np.int64)
        if cidx.size == 0:
            continue
        tc = torch.from_numpy(cidx).cuda()
        xc = _dev(lw.x)[tc]
        for L, proj in zip(lw.layers, projs):
            xc = ops.layer_fwd_candidates(xc, *_params(L), proj, hoff, _offsets(mb), ts[th],
                                          ts[tc], **kw)
        torch.cuda.synchronize()
        for r, row in zip(cidx, xc.float().cpu().numpy().astype(np.float64)):
            out[int(r)] = row
    return out


def oracle_stack(lw):
    a = lw.attn
    x = lw.x.astype(np.float64)
    for L in lw.layers:
        x = O.layer_fwd(problem_of(a), x, L.w1, L.b1, L.ln_gamma, L.ln_beta, L.w2, L.b2,
                        L.rab_p, L.rab_t, ln_eps=lw.ln_eps, residual=lw.residual)
    return x


def test_candidate_layer_stack_matches_one_pass_oracle():
    lw = W.make_layer("cand_stack", [300 + 100, 129 + 60, 0 + 7], 2, 128, 256, 64, 2, seed=64,
                      n_layers=2, num_candidates=[100, 60, 7], max_seq_len=400)
    got = gpu_candidate_stack(lw, 50)
    ref = oracle_stack(lw)
    rows = np.array(sorted(got))
    assert_close(np.stack([got[r] for r in rows]), ref[rows], "bf16", "2-layer candidate stack")


def test_mfalcon_workload_candidates_in_micro_batches():
    """The M-FALCON workload (8 users x (4096 history + 1024 candidates), 3
    layers, d_model 512): candidates in 4 micro-batches of 256 per user match
    the one-pass oracle for users 0 and 5 (sequences are independent)."""
    from test_gpu_layer import _one_user, oracle_layers
    lw = W.mfalcon_bf16_fwd()
    got = gpu_candidate_stack(lw, 256)
    for b in (0, 5):
        one = _one_user(lw, b)
        ref = oracle_layers(one)
        o0 = int(lw.attn.offsets[b])
        nh = int(lw.attn.lengths[b]) - int(lw.attn.num_candidates[b])
        rows = np.arange(o0 + nh, int(lw.attn.offsets[b + 1]))
        assert_close(np.stack([got[int(r)] for r in rows]), ref[rows - o0], "bf16",
                     f"user {b} candidates")
