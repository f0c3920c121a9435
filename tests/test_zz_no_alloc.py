"""hstu_attn_fwd_noalloc: the forward for callers that cannot allocate.

Some callers may not call cudaMalloc or any allocating routine -- code running
under a host framework's own memory manager, inside a callback where
allocation is forbidden, or on a latency budget where an allocation could
synchronise the device -- so they cannot provide hstu_attn_fwd's workspace.
The allocation-free entry point keeps its scratch in a fixed device array
inside the library instead.  These tests call it through the C ABI and check
its output against the workspace entry point's on two calls in a row (the
second call reuses the array the first one left behind).  The refusal of a
problem too large for the array is checked on the CPU, in test_abi_host.py:
the layout is computed before any CUDA call.

The file name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

from hstu_pointwise_attention_b200 import workloads as W

from gpu_common import assert_close, gpu_fwd, kwargs_of, oracle_fwd, to_device, torch_dtype

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
        got = _noalloc(w)
        assert_close(got, gpu_fwd(w), "bf16", f"{w.name} no-alloc vs workspace")
        assert_close(got, oracle_fwd(w), "bf16", f"{w.name} no-alloc vs oracle")


def test_noalloc_float32_simt_path_two_calls():
    w = W.tiny_f32_fwd()
    for _ in range(2):
        assert_close(_noalloc(w), gpu_fwd(w), "f32", "tiny f32 no-alloc vs workspace")
