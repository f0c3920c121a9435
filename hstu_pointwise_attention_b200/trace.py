"""Phase breakdown of the tensor-core attention kernels from their trace build.

    python -m hstu_pointwise_attention_b200.trace [--kernel bwd|fwd]
        [--workload long|zipf] [--no-build] [--json PATH]

Builds the phase-traced library (`build --trace`: the same sources with
-DHSTU_TRACE, into lib_trace/; the product library is not touched), runs one
backward (default) or forward (default workload: 4 x 8192 tokens, 8 heads,
d = 128; zipf: 16 Zipf-length sequences, 8 heads) in a child process that
loads it, and prints for each traced CTA the median and 90th percentile, in
SM clock cycles, of every phase of a 64-query block (backward) or a key tile
(forward); include/hstu.h, hstu_debug_trace_read, lists the recorded events.
Needs one GPU.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys

import numpy as np

PHASES_BWD = [
    ("start_to_load", "block start -> first chunk's tensor-memory load issued"),
    ("tmem_load", "a 16-column chunk's S^T / dP^T load latency"),
    ("chunk_math", "a 16-column chunk's elementwise math"),
    ("store_wait", "last chunk done -> P^T stores complete"),
    ("warp_skew", "first -> last warp of the group handing the block over"),
    ("issuer_delay", "last warp's hand-over -> dQ^T MMAs issued"),
    ("dq_ready", "a warp's hand-over -> dQ^T ready in tensor memory"),
    ("dq_phase", "dQ^T read-out and float32 reductions issued"),
    ("next_wait", "reductions issued -> the group's next block starts"),
]


PHASES_FWD = [
    ("start_to_load", "key tile start -> first chunk's tensor-memory load issued"),
    ("tmem_load", "a 32-key chunk's S load latency"),
    ("chunk_math", "a 32-key chunk's elementwise math"),
    ("store_wait", "last chunk done -> P stores complete"),
    ("warp_skew", "first -> last warp of the tile's group handing P over"),
    ("issuer_delay", "last warp's hand-over -> O += P V issued"),
    ("next_wait", "a warp's hand-over -> its next key tile starts"),
]

GROUPS = {0: [4, 5, 6, 7, 12, 13, 14, 15], 1: [8, 9, 10, 11, 16, 17, 18, 19]}


def _events(buf, slot):
    ev = {}
    for rec in range(buf.shape[1]):
        for e in buf[slot, rec]:
            e = int(e)
            if e:
                ev[(rec, e >> 56, (e >> 40) & 0xffff)] = e & ((1 << 40) - 1)
    return ev


def _stats(ph):
    return {k: (int(np.median(v)), int(np.percentile(v, 90))) if v else None
            for k, v in ph.items()}


def analyse_fwd(buf: np.ndarray) -> dict:
    """Forward: per traced CTA, phase statistics (median, p90) per key tile."""
    out = {}
    for slot in range(buf.shape[0]):
        ev = _events(buf, slot)
        if not ev:
            continue
        ph = {k: [] for k, _ in PHASES_FWD}
        steps = set()
        for x, ws in GROUPS.items():
            ns = sorted({k[2] for k in ev if k[0] in ws and k[1] == 1})
            for idx, n in enumerate(ns):
                steps.add(n)
                hand = []
                for w in ws:
                    s1, st, p2 = ev.get((w, 1, n)), ev.get((w, 11, n)), ev.get((w, 2, n))
                    if None in (s1, st, p2):
                        continue
                    hand.append(p2)
                    last = None
                    for ci in (2 * n, 2 * n + 1):
                        a, b, c = (ev.get((w, code, ci)) for code in (8, 9, 10))
                        if None in (a, b, c):
                            continue
                        if ci == 2 * n:
                            ph["start_to_load"].append(a - s1)
                        ph["tmem_load"].append(b - a)
                        ph["chunk_math"].append(c - b)
                        last = c
                    if last is not None:
                        ph["store_wait"].append(st - last)
                    if idx + 1 < len(ns):
                        nxt = ev.get((w, 1, ns[idx + 1]))
                        if nxt is not None:
                            ph["next_wait"].append(nxt - p2)
                if len(hand) == len(ws):
                    ph["warp_skew"].append(max(hand) - min(hand))
                    iss = ev.get((1, 5, 2 * n + x))
                    if iss is not None:
                        ph["issuer_delay"].append(iss - max(hand))
        times = list(ev.values())
        res = _stats(ph)
        res["blocks"] = len(steps)
        res["cycles_per_block"] = round((max(times) - min(times)) / max(len(steps), 1))
        out[slot] = res
    return out


def analyse(buf: np.ndarray) -> dict:
    """Backward: per traced CTA, phase statistics (median, p90) and cycles per block."""
    out = {}
    for slot in range(buf.shape[0]):
        ev = _events(buf, slot)
        if not ev:
            continue
        ph = {k: [] for k, _ in PHASES_BWD}
        blocks = set()
        for ws in GROUPS.values():
            for jb in sorted({k[2] for k in ev if k[0] in ws and k[1] == 1}):
                blocks.add(jb)
                hand = []
                for w in ws:
                    g = lambda c, o=jb: ev.get((w, c, o))
                    s1, p2, d3, d4, st = g(1), g(2), g(3), g(4), g(11)
                    if None in (s1, p2, d3, d4, st):
                        continue
                    hand.append(p2)
                    last_done = None
                    for ci in (2 * jb, 2 * jb + 1):
                        a, b, c = (ev.get((w, code, ci)) for code in (8, 9, 10))
                        if None in (a, b, c):
                            continue
                        if ci == 2 * jb:
                            ph["start_to_load"].append(a - s1)
                        ph["tmem_load"].append(b - a)
                        ph["chunk_math"].append(c - b)
                        last_done = c
                    if last_done is not None:
                        ph["store_wait"].append(st - last_done)
                    ph["dq_ready"].append(d3 - p2)
                    ph["dq_phase"].append(d4 - d3)
                    nxt = ev.get((w, 1, jb + 2))
                    if nxt is not None:
                        ph["next_wait"].append(nxt - d4)
                if len(hand) == len(ws):
                    ph["warp_skew"].append(max(hand) - min(hand))
                    iss = ev.get((1, 5, jb))
                    if iss is not None:
                        ph["issuer_delay"].append(iss - max(hand))
        times = list(ev.values())
        res = _stats(ph)
        res["blocks"] = len(blocks)
        res["cycles_per_block"] = round((max(times) - min(times)) / max(len(blocks), 1))
        out[slot] = res
    return out


def child(kernel: str, workload: str) -> int:
    import torch
    from hstu_pointwise_attention_b200 import ops, workloads as W
    w = W.zipf_bf16_fwd_bwd() if workload == "zipf" else W.long_bf16_fwd_bwd()
    bf = torch.bfloat16
    q, k, v, dout = (torch.from_numpy(a).cuda().to(bf) for a in (w.q, w.k, w.v, w.dout))
    ts = torch.from_numpy(w.timestamps).cuda()
    rp, rt = torch.from_numpy(w.rab_p).cuda(), torch.from_numpy(w.rab_t).cuda()
    kw = dict(max_seq_len=w.max_seq_len, time_bucket_sub_bits=w.time_bucket_sub_bits,
              alpha=w.alpha, silu_scale=w.silu_scale)

    def run():
        if kernel == "fwd":
            ops.attn_fwd(q, k, v, w.offsets, ts, rp, rt, **kw)
        else:
            ops.attn_bwd(q, k, v, w.offsets, ts, rp, rt, dout, **kw)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    ops.trace_clear(kernel)
    run()
    torch.cuda.synchronize()
    buf = ops.trace_read(kernel)
    print(json.dumps(analyse_fwd(buf) if kernel == "fwd" else analyse(buf)))
    return 0


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--no-build", action="store_true")
    ap.add_argument("--json", default=None, help="also write the result here")
    ap.add_argument("--kernel", default="bwd", choices=["bwd", "fwd"])
    ap.add_argument("--workload", default="long", choices=["long", "zipf"])
    ap.add_argument("--child", action="store_true", help=argparse.SUPPRESS)
    a = ap.parse_args()
    if a.child:
        return child(a.kernel, a.workload)
    from hstu_pointwise_attention_b200 import build
    if not a.no_build:
        build.build(trace=True)
    env = dict(os.environ, HSTU_LIB=build.TRACE_LIB)
    r = subprocess.run([sys.executable, "-m", "hstu_pointwise_attention_b200.trace",
                        "--child", "--kernel", a.kernel, "--workload", a.workload], env=env,
                       capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        return r.returncode
    res = json.loads(r.stdout.strip().splitlines()[-1])
    unit, one = ("key tiles", "key tile") if a.kernel == "fwd" else ("blocks", "block")
    for slot, ph in res.items():
        print(f"traced CTA {slot}: {ph['blocks']} {unit}, {ph['cycles_per_block']} cycles per {one}")
        for key, what in (PHASES_FWD if a.kernel == "fwd" else PHASES_BWD):
            v = ph.get(key)
            if v:
                print(f"  {key:14s} median {v[0]:6d}  p90 {v[1]:6d}   {what}")
    if a.json:
        with open(a.json, "w") as f:
            json.dump(res, f, indent=1)
    return 0


if __name__ == "__main__":
    sys.exit(main())
