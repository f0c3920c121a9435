"""GPU parity of hstu_layer_fwd (projection + SiLU, attention, LayerNorm
gating, output projection + residual) against the oracle, including the
3-layer M-FALCON stack."""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_pointwise_attention_b200 import workloads as W

from gpu_common import assert_close, problem_of

pytestmark = pytest.mark.gpu


def run_layers(lw: W.LayerWorkload, n_layers=None):
    from hstu_pointwise_attention_b200 import ops
    a = lw.attn
    x = torch.from_numpy(lw.x).cuda().to(torch.bfloat16)
    ts = torch.from_numpy(a.timestamps).cuda()
    for L in lw.layers[:n_layers]:
        dev = lambda z, dt=torch.bfloat16: torch.from_numpy(np.ascontiguousarray(z)).cuda().to(dt)
        y = ops.layer_fwd(x, dev(L.w1), dev(L.b1, torch.float32), dev(L.ln_gamma, torch.float32),
                          dev(L.ln_beta, torch.float32), dev(L.w2), dev(L.b2, torch.float32),
                          dev(L.rab_p, torch.float32), dev(L.rab_t, torch.float32), a.offsets, ts,
                          num_heads=a.num_heads, d_qk=a.d_qk, d_v=a.d_v,
                          max_seq_len=a.max_seq_len,
                          time_bucket_sub_bits=a.time_bucket_sub_bits, alpha=a.alpha,
                          silu_scale=a.silu_scale, num_candidates=a.num_candidates,
                          ln_eps=lw.ln_eps, residual=lw.residual)
        x = y
    torch.cuda.synchronize()
    return x.float().cpu().numpy().astype(np.float64)


def oracle_layers(lw: W.LayerWorkload, n_layers=None):
    a = lw.attn
    x = lw.x.astype(np.float64)
    for L in lw.layers[:n_layers]:
        x = O.layer_fwd(problem_of(a), x, L.w1, L.b1, L.ln_gamma, L.ln_beta, L.w2, L.b2,
                        L.rab_p, L.rab_t, ln_eps=lw.ln_eps, residual=lw.residual)
    return x


def test_small_layer_ragged():
    lw = W.make_layer("small", [1, 100, 129, 300], 2, 64, 128, 64, 2, seed=31,
                      max_seq_len=300)
    assert_close(run_layers(lw), oracle_layers(lw), "bf16", "small layer")


def test_small_layer_mfalcon_two_stacked():
    lw = W.make_layer("small", [200, 260], 2, 128, 256, 64, 2, seed=32, n_layers=2,
                      num_candidates=[50, 4], max_seq_len=260)
    assert_close(run_layers(lw), oracle_layers(lw), "bf16", "mfalcon 2 layers")


def test_layer_workload_full_size():
    lw = W.layer_bf16_fwd()
    assert_close(run_layers(lw), oracle_layers(lw), "bf16", "layer workload")


def _one_user(lw: W.LayerWorkload, b: int) -> W.LayerWorkload:
    """The same layers restricted to sequence b (sequences are independent)."""
    a = lw.attn
    o0, o1 = int(a.offsets[b]), int(a.offsets[b + 1])
    sub = W.AttnWorkload(**{**a.__dict__, "offsets": np.array([0, o1 - o0], np.int64),
                            "timestamps": a.timestamps[o0:o1], "q": a.q[o0:o1],
                            "k": a.k[o0:o1], "v": a.v[o0:o1], "dout": None,
                            "num_candidates": (None if a.num_candidates is None
                                               else a.num_candidates[b:b + 1])})
    return W.LayerWorkload(name=lw.name, attn=sub, d_model=lw.d_model, x=lw.x[o0:o1],
                           layers=lw.layers, ln_eps=lw.ln_eps, residual=lw.residual)


def test_mfalcon_workload_full_size_sampled_users():
    lw = W.mfalcon_bf16_fwd()
    got = run_layers(lw)
    for b in (0, 5):
        one = _one_user(lw, b)
        o0, o1 = int(lw.attn.offsets[b]), int(lw.attn.offsets[b + 1])
        assert_close(got[o0:o1], oracle_layers(one), "bf16", f"mfalcon user {b}")
