"""The entry points record whole under CUDA stream capture (the tile schedule
reaches the workspace as kernel parameters, not by a host copy): a captured
forward + backward, and a captured layer forward and backward, replayed
several times, give the eager results (forward bit for bit; backward up to the
order of its float32 atomic sums) and match the oracle."""
import numpy as np
import pytest
import torch

from hstu_pointwise_attention_b200 import workloads as W

from gpu_common import assert_close, kwargs_of, oracle_bwd, oracle_fwd, to_device

pytestmark = pytest.mark.gpu


def _attn_calls(w, d, out, grads):
    from hstu_pointwise_attention_b200 import ops
    ops.attn_fwd(d["q"], d["k"], d["v"], w.offsets, d["ts"], d["rab_p"], d["rab_t"], out=out,
                 **kwargs_of(w))
    grads[3].zero_()
    grads[4].zero_()
    ops.attn_bwd(d["q"], d["k"], d["v"], w.offsets, d["ts"], d["rab_p"], d["rab_t"], d["dout"],
                 dq=grads[0], dk=grads[1], dv=grads[2], drab_pos=grads[3], drab_time=grads[4],
                 **kwargs_of(w))


@pytest.mark.parametrize("nc", [None, [40, 3, 0]])
def test_attention_forward_backward_replay_from_a_graph(nc):
    w = W.make_attention("graph", [700, 129, 300], 2, 128, 128, 2, "bf16", seed=81,
                         with_grad=True, num_candidates=nc)
    d = to_device(w)
    out = torch.empty_like(d["v"])
    grads = [torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"]),
             torch.zeros_like(d["rab_p"]), torch.zeros_like(d["rab_t"])]
    _attn_calls(w, d, out, grads)          # eager (also sets the kernels' attributes)
    torch.cuda.synchronize()
    eager = [out.clone()] + [g.clone() for g in grads]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g):
            _attn_calls(w, d, out, grads)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        out.fill_(float("nan"))
        for t in grads[:3]:
            t.fill_(float("nan"))
        g.replay()
    torch.cuda.synchronize()
    torch.testing.assert_close(out, eager[0], rtol=0, atol=0)
    for got, ref in zip(grads, eager[1:]):
        torch.testing.assert_close(got.float(), ref.float(), rtol=1e-2, atol=1e-3)
    f64 = lambda t: t.float().cpu().numpy().astype(np.float64)
    assert_close(f64(out), oracle_fwd(w), "bf16", "graph fwd")
    for got, ref, name in zip(grads, oracle_bwd(w), ("dq", "dk", "dv", "drab_p", "drab_t")):
        assert_close(f64(got), ref, "bf16", "graph " + name)


def test_layer_forward_and_backward_replay_from_a_graph():
    from hstu_pointwise_attention_b200 import ops
    lw = W.make_layer("graph_layer", [300, 129, 64], 2, 64, 128, 64, 2, seed=82,
                      max_seq_len=300)
    a, L = lw.attn, lw.layers[0]
    bf, f32 = torch.bfloat16, torch.float32
    dev = lambda z, dt=bf: torch.from_numpy(np.ascontiguousarray(z)).cuda().to(dt)
    P = (dev(L.w1), dev(L.b1, f32), dev(L.ln_gamma, f32), dev(L.ln_beta, f32), dev(L.w2),
         dev(L.b2, f32), dev(L.rab_p, f32), dev(L.rab_t, f32))
    x, ts = dev(lw.x), torch.from_numpy(a.timestamps).cuda()
    dy = dev(np.random.default_rng(83).standard_normal(lw.x.shape))
    kw = dict(num_heads=a.num_heads, d_qk=a.d_qk, d_v=a.d_v, max_seq_len=a.max_seq_len,
              time_bucket_sub_bits=a.time_bucket_sub_bits, alpha=a.alpha,
              silu_scale=a.silu_scale)
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    grads = {n: torch.zeros(t.shape, dtype=f32, device="cuda")
             for n, t in zip(("dw1", "db1", "dgamma", "dbeta", "dw2", "db2", "drab_pos",
                              "drab_time"), P)}

    def calls():
        for t in grads.values():
            t.zero_()
        ops.layer_fwd(x, *P, a.offsets, ts, out=y, **kw)
        ops.layer_bwd(x, *P, a.offsets, ts, dy, dx=dx, grads=grads, **kw)

    calls()
    torch.cuda.synchronize()
    ref_y, ref_dx = y.clone(), dx.clone()
    ref_g = {n: t.clone() for n, t in grads.items()}
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g):
            calls()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(2):
        y.fill_(float("nan"))
        dx.fill_(float("nan"))
        g.replay()
    torch.cuda.synchronize()
    torch.testing.assert_close(y, ref_y, rtol=0, atol=0)
    torch.testing.assert_close(dx.float(), ref_dx.float(), rtol=1e-2, atol=1e-2)
    for n in grads:
        torch.testing.assert_close(grads[n], ref_g[n], rtol=1e-3, atol=1e-4)
