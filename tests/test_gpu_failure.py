"""Device-side failure detection on the GPU without a fault: a bounded wait
that runs out is recorded in the workspace's error word and reported by
hstu_get_device_error, the kernel returns, and the same context and
workspace then run the attention path correctly."""
import numpy as np
import pytest
import torch

from hstu_pointwise_attention_b200 import ops
from hstu_pointwise_attention_b200 import workloads as W

from gpu_common import assert_close, kwargs_of, oracle_fwd, to_device

pytestmark = pytest.mark.gpu

HSTU_OK, HSTU_ERR_DEVICE_TIMEOUT = 0, 5


def test_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    w = W.make_attention("case", [1, 130, 257], 2, 128, 128, 2, "bf16", 11)
    d = to_device(w)
    kw = kwargs_of(w)
    pf = ops.make_params(d["q"], d["k"], d["v"], w.offsets,
                         num_pos_buckets=w.num_pos_buckets,
                         num_time_buckets=w.num_time_buckets, **kw)
    ws = torch.empty(ops.attn_workspace_size(pf, w.offsets, False), dtype=torch.uint8,
                     device="cuda")
    # a 2 ms wait on a barrier nothing arrives at
    assert ops.debug_wait_probe(ws, 2000) == HSTU_OK
    rc, word = ops.get_device_error(ws)
    assert rc == HSTU_ERR_DEVICE_TIMEOUT and (word & 1)
    # same stream, same workspace: the next call clears the word and is correct
    out = torch.full((w.total_tokens, w.num_heads, w.d_v), float("nan"), dtype=torch.bfloat16,
                     device="cuda")
    ops.attn_fwd(d["q"], d["k"], d["v"], w.offsets, d["ts"], d["rab_p"], d["rab_t"], out=out,
                 workspace=ws, **kw)
    rc, word = ops.get_device_error(ws)
    assert rc == HSTU_OK and word == 0
    got = out.float().cpu().numpy().astype(np.float64)
    assert_close(got, oracle_fwd(w), "bf16", "forward after a reported timeout")
