"""The data-parallel exchange of the multi-GPU path, run as two gloo ranks on
the CPU: every rank computes the backward of its own batch of sequences with
the same (replicated) rab tables, and the rab-table gradients are summed
across ranks with one all-reduce, as bench.py does with NCCL.  Sequences are
independent, so the summed gradients must equal the backward of the
concatenated batch, and each rank's dq, dk, dv its slice of it."""
import os
import socket
import tempfile

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import hstu_oracle as O
from hstu_pointwise_attention_b200 import workloads as W

WORLD = 2
LENGTHS = {0: [23, 40, 1], 1: [37, 9]}


def shard(rank: int) -> W.AttnWorkload:
    w = W.make_attention("dp", LENGTHS[rank], 2, 16, 32, 1, "f32", 40 + 1000 * rank,
                         max_seq_len=64, with_grad=True)
    tables = W.make_attention("dp", [4], 2, 16, 32, 1, "f32", 7, max_seq_len=64)
    w.rab_p, w.rab_t = tables.rab_p, tables.rab_t      # parameters are replicated
    return w


def problem(w: W.AttnWorkload) -> O.Problem:
    return O.Problem(offsets=w.offsets, timestamps=w.timestamps, num_heads=w.num_heads,
                     d_qk=w.d_qk, d_v=w.d_v, num_pos_buckets=w.num_pos_buckets,
                     num_time_buckets=w.num_time_buckets,
                     time_bucket_sub_bits=w.time_bucket_sub_bits, alpha=w.alpha,
                     silu_scale=w.silu_scale)


def worker(rank: int, port: int, outdir: str):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD)
    w = shard(rank)
    dq, dk, dv, drp, drt = O.attn_bwd(problem(w), w.q, w.k, w.v, w.rab_p, w.rab_t, w.dout)
    t_p, t_t = torch.from_numpy(drp), torch.from_numpy(drt)
    dist.all_reduce(t_p)
    dist.all_reduce(t_t)
    np.savez(os.path.join(outdir, f"rank{rank}.npz"), dq=dq, dk=dk, dv=dv,
             drp=t_p.numpy(), drt=t_t.numpy())
    dist.barrier()
    dist.destroy_process_group()


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_sum_rab_gradients_like_one_concatenated_batch():
    with tempfile.TemporaryDirectory() as outdir:
        mp.start_processes(worker, args=(free_port(), outdir), nprocs=WORLD, join=True,
                           start_method="spawn")
        res = [np.load(os.path.join(outdir, f"rank{r}.npz")) for r in range(WORLD)]
    a, b = shard(0), shard(1)
    T0 = a.total_tokens
    whole = W.AttnWorkload(
        name="dp", dtype="f32", offsets=np.concatenate([a.offsets, b.offsets[1:] + T0]),
        timestamps=np.concatenate([a.timestamps, b.timestamps]), num_heads=a.num_heads,
        d_qk=a.d_qk, d_v=a.d_v, num_pos_buckets=a.num_pos_buckets,
        num_time_buckets=a.num_time_buckets, time_bucket_sub_bits=a.time_bucket_sub_bits,
        max_seq_len=a.max_seq_len, alpha=a.alpha, silu_scale=a.silu_scale,
        q=np.concatenate([a.q, b.q]), k=np.concatenate([a.k, b.k]),
        v=np.concatenate([a.v, b.v]), rab_p=a.rab_p, rab_t=a.rab_t,
        dout=np.concatenate([a.dout, b.dout]))
    dq, dk, dv, drp, drt = O.attn_bwd(problem(whole), whole.q, whole.k, whole.v, whole.rab_p,
                                      whole.rab_t, whole.dout)
    for r in range(WORLD):
        np.testing.assert_allclose(res[r]["drp"], drp, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(res[r]["drt"], drt, rtol=1e-12, atol=1e-12)
    for name, ref in (("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(np.concatenate([res[0][name], res[1][name]]), ref,
                                   rtol=1e-12, atol=1e-12)
    assert np.abs(drp).sum() > 0 and np.abs(drt).sum() > 0
