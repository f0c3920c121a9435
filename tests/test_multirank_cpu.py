"""The data-parallel path, run as two gloo ranks on the CPU.

A global jagged batch is split by the package (``dp.partition``, i.e. the C
library's hstu_partition_batch, which balances visible pairs per rank); each
rank gathers its local batch (``dp.local_batch``), computes the backward of
its sequences with the shared bias tables, and the two table gradients are
summed across ranks with one all-reduce of one buffer (``dp.RabGrads``), as
bench.py does with NCCL.  Sequences are independent, so the summed table
gradients must equal the backward of the whole batch, and each rank's dq,
dk, dv the rows of its own tokens.  (The per-rank backward here is the
oracle's: this checks the split and the exchange, which need no GPU.)"""
import os
import socket
import tempfile

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import hstu_oracle as O
from hstu_pointwise_attention_b200 import dp
from hstu_pointwise_attention_b200 import workloads as W

WORLD = 2
LENGTHS = [23, 40, 1, 37, 9, 0, 17]
CANDS = [3, 0, 1, 5, 0, 0, 2]


def global_batch() -> W.AttnWorkload:
    return W.make_attention("dp", LENGTHS, 2, 16, 32, 1, "f32", 40, max_seq_len=64,
                            with_grad=True, num_candidates=CANDS)


def problem(w, off, ts, nc) -> O.Problem:
    return O.Problem(offsets=off, timestamps=ts, num_heads=w.num_heads, d_qk=w.d_qk, d_v=w.d_v,
                     num_pos_buckets=w.num_pos_buckets, num_time_buckets=w.num_time_buckets,
                     time_bucket_sub_bits=w.time_bucket_sub_bits, alpha=w.alpha,
                     silu_scale=w.silu_scale, num_candidates=nc)


def worker(rank: int, port: int, outdir: str):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD)
    w = global_batch()
    seqs = dp.local_sequences(w.offsets, WORLD, rank, w.num_candidates)
    off, tok, nc = dp.local_batch(w.offsets, seqs, w.num_candidates)
    dq, dk, dv, drp, drt = O.attn_bwd(problem(w, off, w.timestamps[tok], nc), w.q[tok],
                                      w.k[tok], w.v[tok], w.rab_p, w.rab_t, w.dout[tok])
    g = dp.RabGrads(w.rab_p.shape, w.rab_t.shape, "cpu")
    g.pos.copy_(torch.from_numpy(drp))
    g.time.copy_(torch.from_numpy(drt))
    g.all_reduce()
    np.savez(os.path.join(outdir, f"rank{rank}.npz"), tok=tok, dq=dq, dk=dk, dv=dv,
             drp=g.pos.double().numpy(), drt=g.time.double().numpy())
    dist.barrier()
    dist.destroy_process_group()


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_split_and_sum_like_one_batch():
    with tempfile.TemporaryDirectory() as outdir:
        mp.start_processes(worker, args=(free_port(), outdir), nprocs=WORLD, join=True,
                           start_method="spawn")
        res = [np.load(os.path.join(outdir, f"rank{r}.npz")) for r in range(WORLD)]
    w = global_batch()
    dq, dk, dv, drp, drt = O.attn_bwd(problem(w, w.offsets, w.timestamps, w.num_candidates),
                                      w.q, w.k, w.v, w.rab_p, w.rab_t, w.dout)
    # every token is on exactly one rank
    toks = np.concatenate([r["tok"] for r in res])
    assert sorted(toks.tolist()) == list(range(w.total_tokens))
    for r in res:
        # float32 all-reduce of float64 partials
        np.testing.assert_allclose(r["drp"], drp, rtol=1e-5, atol=1e-7)
        np.testing.assert_allclose(r["drt"], drt, rtol=1e-5, atol=1e-7)
        for name, ref in (("dq", dq), ("dk", dk), ("dv", dv)):
            np.testing.assert_allclose(r[name], ref[r["tok"]], rtol=1e-12, atol=1e-12)
    assert np.abs(drp).sum() > 0 and np.abs(drt).sum() > 0
    # both ranks got work
    assert all(len(r["tok"]) > 0 for r in res)
