"""hstu_attn_fwd_noalloc: the forward for callers that cannot allocate.

Some callers may not call cudaMalloc or any allocating routine -- code running
under a host framework's own memory manager, inside a callback where
allocation is forbidden, or on a latency budget where an allocation could
synchronise the device -- so they cannot provide hstu_attn_fwd's workspace.
The allocation-free entry point keeps its scratch in a fixed device array
inside the library instead.  These tests call it through the C ABI and check
its output against the workspace entry point's on two calls in a row (the
second call reuses the array the first one left behind), and check that a
problem too large for the array is refused before any launch.

The file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from hstu_pointwise_attention_b200 import workloads as W

from gpu_common import assert_close, gpu_fwd, kwargs_of, to_device, torch_dtype

pytestmark = pytest.mark.gpu


def _noalloc(w):
    from hstu_pointwise_attention_b200 import ops
    d = to_device(w)
    out = torch.full((w.total_tokens, w.num_heads, w.d_v), float("nan"), dtype=torch_dtype(w),
                     device="cuda")
    ops.attn_fwd_noalloc(d["q"], d["k"], d["v"], w.offsets, d["ts"], d["rab_p"], d["rab_t"],
                         out=out, **kwargs_of(w))
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


def test_noalloc_matches_workspace_forward_on_two_calls():
    first = W.make_attention("noalloc_a", [1, 37, 129, 300, 513], 2, 128, 128, 2, "bf16",
                             seed=41, with_grad=False)
    second = W.make_attention("noalloc_b", [260, 640, 77], 2, 128, 64, 2, "bf16", seed=42,
                              num_candidates=[60, 128, 77])
    for w in (first, second):
        assert_close(_noalloc(w), gpu_fwd(w), "bf16", f"{w.name} no-alloc vs workspace")


def test_noalloc_float32_simt_path_two_calls():
    w = W.tiny_f32_fwd()
    for _ in range(2):
        assert_close(_noalloc(w), gpu_fwd(w), "f32", "tiny f32 no-alloc vs workspace")


def test_noalloc_rejects_problem_larger_than_its_scratch():
    from hstu_pointwise_attention_b200 import ops
    # 2^22 tokens need 16 MiB of float timestamps, more than the 8 MiB array;
    # the call must refuse before touching the (tiny) buffers below.
    T = 1 << 22
    off = np.array([0, T], np.int64)
    q = torch.zeros((1, 2, 64), dtype=torch.bfloat16, device="cuda")
    ts = torch.zeros(1, dtype=torch.int64, device="cuda")
    rab = torch.zeros(8, dtype=torch.float32, device="cuda")
    p = ops.make_params(q, q, q, off, max_seq_len=T, num_pos_buckets=8, num_time_buckets=8,
                        time_bucket_sub_bits=1)
    rc = ops.LIB.hstu_attn_fwd_noalloc(ctypes.byref(p), off.ctypes.data, None, ts.data_ptr(),
                                       q.data_ptr(), q.data_ptr(), q.data_ptr(), rab.data_ptr(),
                                       rab.data_ptr(), q.data_ptr(), None)
    assert rc == 3, ops.STATUS.get(rc)
