"""GPU parity of hstu_layer_bwd (the HSTU layer's backward: projection,
attention, LayerNorm gating and output projection in reverse) against the
oracle's float64 chain rule (oracle.layer_bwd, pinned by central differences
of the layer forward), on every gradient: dx, dW1, db1, dgamma, dbeta, dW2,
db2 and both bias tables."""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_pointwise_attention_b200 import workloads as W

from gpu_common import assert_close, problem_of

pytestmark = pytest.mark.gpu

NAMES = ("dx", "dw1", "db1", "dgamma", "dbeta", "dw2", "db2", "drab_pos", "drab_time")


def _dev(z, dt=torch.bfloat16):
    return torch.from_numpy(np.ascontiguousarray(z)).cuda().to(dt)


def _kw(lw):
    a = lw.attn
    return dict(num_heads=a.num_heads, d_qk=a.d_qk, d_v=a.d_v, max_seq_len=a.max_seq_len,
                time_bucket_sub_bits=a.time_bucket_sub_bits, alpha=a.alpha,
                silu_scale=a.silu_scale, num_candidates=a.num_candidates, ln_eps=lw.ln_eps,
                residual=lw.residual)


def _params(L):
    f32 = torch.float32
    return (_dev(L.w1), _dev(L.b1, f32), _dev(L.ln_gamma, f32), _dev(L.ln_beta, f32),
            _dev(L.w2), _dev(L.b2, f32), _dev(L.rab_p, f32), _dev(L.rab_t, f32))


def _perturb(lw, seed):
    """Non-trivial biases, gamma, beta and bias tables (the defaults are 0 / 1)."""
    rng = np.random.default_rng(seed)
    for L in lw.layers:
        L.b1 = (rng.standard_normal(L.b1.shape) * 0.1).astype(np.float32)
        L.b2 = (rng.standard_normal(L.b2.shape) * 0.1).astype(np.float32)
        L.ln_gamma = (1 + 0.2 * rng.standard_normal(L.ln_gamma.shape)).astype(np.float32)
        L.ln_beta = (0.2 * rng.standard_normal(L.ln_beta.shape)).astype(np.float32)
        L.rab_p = (rng.standard_normal(L.rab_p.shape) * 0.3).astype(np.float32)
        L.rab_t = (rng.standard_normal(L.rab_t.shape) * 0.3).astype(np.float32)
    return W.round_bf16(rng.standard_normal(lw.x.shape).astype(np.float32))


def gpu_layer_bwd(lw, L, x, dy):
    from hstu_pointwise_attention_b200 import ops
    a = lw.attn
    ts = torch.from_numpy(a.timestamps).cuda()
    dx, g = ops.layer_bwd(_dev(x), *_params(L), a.offsets, ts, _dev(dy), **_kw(lw))
    torch.cuda.synchronize()
    out = [dx] + [g[n] for n in NAMES[1:]]
    return [t.float().cpu().numpy().astype(np.float64) for t in out]


def oracle_layer_bwd(lw, L, x, dy):
    return O.layer_bwd(problem_of(lw.attn), x, L.w1, L.b1, L.ln_gamma, L.ln_beta, L.w2, L.b2,
                       L.rab_p, L.rab_t, dy, ln_eps=lw.ln_eps, residual=lw.residual)


def _check(got, want, what):
    for g, r, n in zip(got, want, NAMES):
        assert_close(g, r, "bf16", f"{what} {n}")


@pytest.mark.parametrize("residual", [True, False])
def test_layer_bwd_small_ragged(residual):
    lw = W.make_layer("small_bwd", [1, 100, 129, 300], 2, 64, 128, 64, 2, seed=51,
                      max_seq_len=300)
    lw.residual = residual
    dy = _perturb(lw, 52)
    L = lw.layers[0]
    _check(gpu_layer_bwd(lw, L, lw.x, dy), oracle_layer_bwd(lw, L, lw.x, dy),
           f"small residual={residual}")


def test_layer_bwd_workload_full_size():
    """The d_model 256 layer workload (32 sequences of 64..1024 tokens, 4 heads, d 64)."""
    lw = W.layer_bf16_fwd()
    dy = _perturb(lw, 53)
    L = lw.layers[0]
    _check(gpu_layer_bwd(lw, L, lw.x, dy), oracle_layer_bwd(lw, L, lw.x, dy), "layer workload")


def test_layer_bwd_mfalcon_two_stacked():
    """Two stacked layers with M-FALCON candidates, d 128: layer 2's dx is
    layer 1's dy."""
    from hstu_pointwise_attention_b200 import ops
    lw = W.make_layer("mf_bwd", [200, 260, 64], 2, 128, 256, 64, 2, seed=54, n_layers=2,
                      num_candidates=[50, 4, 64], max_seq_len=260)
    dy = _perturb(lw, 55)
    a = lw.attn
    ts = torch.from_numpy(a.timestamps).cuda()
    L0, L1 = lw.layers
    # GPU: y1 = layer 0 (x); backward of layer 1 at y1, then of layer 0 with its dx
    y1 = ops.layer_fwd(_dev(lw.x), *_params(L0), a.offsets, ts, **_kw(lw))
    dx1, g1 = ops.layer_bwd(y1, *_params(L1), a.offsets, ts, _dev(dy), **_kw(lw))
    dx0, g0 = ops.layer_bwd(_dev(lw.x), *_params(L0), a.offsets, ts, dx1, **_kw(lw))
    torch.cuda.synchronize()
    p = problem_of(a)
    oy1 = O.layer_fwd(p, lw.x, L0.w1, L0.b1, L0.ln_gamma, L0.ln_beta, L0.w2, L0.b2, L0.rab_p,
                      L0.rab_t, ln_eps=lw.ln_eps, residual=lw.residual)
    r1 = oracle_layer_bwd(lw, L1, oy1, dy)
    r0 = oracle_layer_bwd(lw, L0, lw.x, r1[0])
    to = lambda t: t.float().cpu().numpy().astype(np.float64)
    _check([to(dx1)] + [to(g1[n]) for n in NAMES[1:]], r1, "layer 2")
    _check([to(dx0)] + [to(g0[n]) for n in NAMES[1:]], r0, "layer 1")


def test_layer_bwd_accumulates_into_given_gradients():
    """The float32 parameter gradients are added to: two calls give twice one."""
    from hstu_pointwise_attention_b200 import ops
    lw = W.make_layer("acc_bwd", [70, 33], 2, 64, 128, 64, 2, seed=56, max_seq_len=70)
    dy = _perturb(lw, 57)
    a = lw.attn
    ts = torch.from_numpy(a.timestamps).cuda()
    L = lw.layers[0]
    _, g = ops.layer_bwd(_dev(lw.x), *_params(L), a.offsets, ts, _dev(dy), **_kw(lw))
    once = {n: t.clone() for n, t in g.items()}
    ops.layer_bwd(_dev(lw.x), *_params(L), a.offsets, ts, _dev(dy), grads=g, **_kw(lw))
    torch.cuda.synchronize()
    for n in NAMES[1:]:
        torch.testing.assert_close(g[n], 2 * once[n], rtol=1e-4, atol=1e-6)
