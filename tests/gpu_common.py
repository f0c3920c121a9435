"""Shared helpers of the GPU parity tests: move a seeded workload to the
device, run the library through its C ABI, run the oracle on the same inputs,
and compare with the stated tolerances.

Tolerances (the design notes' reading R13):
  float32 path: max|got - ref| <= 1e-4 * max|ref|
  bf16 path:    max|got - ref| <= 2e-2 * max|ref|   ("output scale" = largest
                reference magnitude; rounding a bf16 output alone moves an
                element by up to 2^-9 of its own size, so a bound relative to
                the RMS cannot hold for the largest elements of a heavy-tailed
                output), and in addition RMS(got - ref) <= 1e-2 * RMS(ref).
Integer work (buckets, masks) is compared bit for bit.
"""
import numpy as np
import torch

from oracle import hstu_oracle as O
from hstu_pointwise_attention_b200 import workloads as W

F32_TOL = 1e-4
BF16_TOL = 2e-2
BF16_RMS_TOL = 1e-2


def problem_of(w: W.AttnWorkload) -> O.Problem:
    return O.Problem(offsets=w.offsets, timestamps=w.timestamps, num_heads=w.num_heads,
                     d_qk=w.d_qk, d_v=w.d_v, num_pos_buckets=w.num_pos_buckets,
                     num_time_buckets=w.num_time_buckets,
                     time_bucket_sub_bits=w.time_bucket_sub_bits, alpha=w.alpha,
                     silu_scale=w.silu_scale, num_candidates=w.num_candidates,
                     rab_per_head=w.rab_per_head)


def torch_dtype(w):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def to_device(w: W.AttnWorkload, dev="cuda"):
    dt = torch_dtype(w)
    d = dict(
        q=torch.from_numpy(w.q).to(dev).to(dt),
        k=torch.from_numpy(w.k).to(dev).to(dt),
        v=torch.from_numpy(w.v).to(dev).to(dt),
        ts=torch.from_numpy(w.timestamps).to(dev),
        rab_p=torch.from_numpy(np.ascontiguousarray(w.rab_p)).to(dev),
        rab_t=torch.from_numpy(np.ascontiguousarray(w.rab_t)).to(dev),
    )
    if w.dout is not None:
        d["dout"] = torch.from_numpy(w.dout).to(dev).to(dt)
    return d


def kwargs_of(w: W.AttnWorkload):
    return dict(max_seq_len=w.max_seq_len, time_bucket_sub_bits=w.time_bucket_sub_bits,
                alpha=w.alpha, silu_scale=w.silu_scale, num_candidates=w.num_candidates,
                rab_per_head=w.rab_per_head)


def gpu_fwd(w, impl="auto", dev_inputs=None):
    from hstu_pointwise_attention_b200 import ops
    d = dev_inputs or to_device(w)
    out = torch.full((w.total_tokens, w.num_heads, w.d_v), float("nan"),
                     dtype=torch_dtype(w), device="cuda")
    ops.attn_fwd(d["q"], d["k"], d["v"], w.offsets, d["ts"], d["rab_p"], d["rab_t"], out=out,
                 impl=impl, **kwargs_of(w))
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


def gpu_bwd(w, impl="auto", dev_inputs=None):
    from hstu_pointwise_attention_b200 import ops
    d = dev_inputs or to_device(w)
    res = ops.attn_bwd(d["q"], d["k"], d["v"], w.offsets, d["ts"], d["rab_p"], d["rab_t"],
                       d["dout"], impl=impl, **kwargs_of(w))
    torch.cuda.synchronize()
    return [r.float().cpu().numpy().astype(np.float64) for r in res]


def oracle_fwd(w, rows=None):
    return O.attn_fwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t, rows=rows)


def oracle_bwd(w):
    return O.attn_bwd(problem_of(w), w.q, w.k, w.v, w.rab_p, w.rab_t, w.dout)


def err_stats(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU output"
    if not ref.size:
        return 0.0, 0.0, 0.0, 0.0
    err = float(np.max(np.abs(got - ref)))
    rms = float(np.sqrt(np.mean(ref ** 2)))
    mx = float(np.max(np.abs(ref)))
    rms_err = float(np.sqrt(np.mean((got - ref) ** 2)))
    return err, rms, mx, rms_err


def assert_close(got, ref, dtype: str, what: str = ""):
    err, rms, mx, rms_err = err_stats(got, ref)
    if dtype == "f32":
        assert err <= F32_TOL * mx + 1e-30, f"{what}: max err {err:.3e} > 1e-4 * max|ref| ({mx:.3e})"
    else:
        assert err <= BF16_TOL * mx + 1e-30, \
            f"{what}: max err {err:.3e} > 2e-2 * max|ref| ({mx:.3e}); RMS(ref) {rms:.3e}"
        assert rms_err <= BF16_RMS_TOL * rms + 1e-30, \
            f"{what}: RMS err {rms_err:.3e} > 1e-2 * RMS(ref) ({rms:.3e})"
    return err, rms, mx


def sample_rows(w: W.AttnWorkload, per_seq: int, seed: int):
    """Tile edges (0, 127, 128, 255, 256, L-1, candidate boundary) plus random rows."""
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(w.batch):
        o, L = int(w.offsets[b]), int(w.lengths[b])
        if L == 0:
            continue
        pick = {0, L - 1}
        for e in (127, 128, 255, 256, 383, 384):
            if e < L:
                pick.add(e)
        if w.num_candidates is not None:
            nh = L - int(w.num_candidates[b])
            for e in (nh - 1, nh, nh + 1):
                if 0 <= e < L:
                    pick.add(e)
        pick |= set(int(x) for x in rng.integers(0, L, size=per_seq))
        rows += [o + r for r in sorted(pick)]
    return np.array(rows, np.int64)
