"""Host logic of the phase traces: the analysis of synthetic trace buffers
(backward and forward), and the product library's refusal when built
without the trace."""
import ctypes

import numpy as np

from hstu_pointwise_attention_b200 import ops
from hstu_pointwise_attention_b200.trace import analyse, analyse_fwd


def _entry(code, ordinal, clock):
    return np.uint64((code << 56) | (ordinal << 40) | clock)


def test_trace_analysis_phases():
    buf = np.zeros(ops.TRACE_SHAPE, dtype=np.uint64)
    n = np.zeros(ops.TRACE_SHAPE[:2], dtype=np.int64)

    def put(rec, code, ordinal, clock):
        buf[0, rec, n[0, rec]] = _entry(code, ordinal, clock)
        n[0, rec] += 1

    group0 = [4, 5, 6, 7, 12, 13, 14, 15]
    for i, w in enumerate(group0):
        base = 1000 + 3 * i
        put(w, 1, 0, base)                 # block 0 starts
        put(w, 8, 0, base + 20)            # chunk 0: load issued
        put(w, 9, 0, base + 20 + 250)      #          landed
        put(w, 10, 0, base + 270 + 1300)   #          math done
        put(w, 8, 1, base + 1600)          # chunk 1
        put(w, 9, 1, base + 1850)
        put(w, 10, 1, base + 3150)
        put(w, 11, 0, base + 3290)         # P^T stored
        put(w, 2, 0, base + 3300 + 10 * i)  # hand-over, 10 cycles apart per warp
        put(w, 3, 0, base + 5300 + 10 * i)  # dQ^T ready
        put(w, 4, 0, base + 6800 + 10 * i)  # reductions issued
        put(w, 1, 2, base + 7600 + 10 * i)  # block 2 starts
    last_hand = max(1000 + 3 * i + 3300 + 10 * i for i in range(8))
    put(1, 5, 0, last_hand + 850)           # issuer: dQ^T issued
    res = analyse(buf)[0]
    assert res["tmem_load"][0] == 250
    assert res["chunk_math"][0] == 1300
    assert res["start_to_load"][0] == 20
    assert res["store_wait"][0] == 140
    assert res["warp_skew"][0] == 7 * 13
    assert res["issuer_delay"][0] == 850
    assert res["dq_ready"][0] == 2000
    assert res["dq_phase"][0] == 1500
    assert res["next_wait"][0] == 800
    assert res["blocks"] == 2


def test_forward_trace_analysis_phases():
    buf = np.zeros(ops.TRACE_SHAPE, dtype=np.uint64)
    n = np.zeros(ops.TRACE_SHAPE[:2], dtype=np.int64)

    def put(rec, code, ordinal, clock):
        buf[0, rec, n[0, rec]] = _entry(code, ordinal, clock)
        n[0, rec] += 1

    group1 = [8, 9, 10, 11, 16, 17, 18, 19]   # query tile B (x = 1)
    for i, w in enumerate(group1):
        for step, base in ((3, 10000 + 5 * i), (4, 17000 + 5 * i)):
            put(w, 1, step, base)
            put(w, 8, 2 * step, base + 30)
            put(w, 9, 2 * step, base + 30 + 400)
            put(w, 10, 2 * step, base + 430 + 1500)
            put(w, 8, 2 * step + 1, base + 1960)
            put(w, 9, 2 * step + 1, base + 2360)
            put(w, 10, 2 * step + 1, base + 3860)
            put(w, 11, step, base + 4000)
            put(w, 2, step, base + 4010 + 10 * i)
    put(1, 5, 2 * 3 + 1, 10000 + 7 * 5 + 4010 + 70 + 600)   # O += P V of step 3, tile B
    res = analyse_fwd(buf)[0]
    assert res["tmem_load"][0] == 400
    assert res["chunk_math"][0] == 1500
    assert res["start_to_load"][0] == 30
    assert res["store_wait"][0] == 140
    assert res["warp_skew"][0] == 7 * 15
    assert res["issuer_delay"][0] == 600
    # each warp's hand-over at step 3 -> its start of step 4: 2990 - 10 i cycles
    assert res["next_wait"][0] == int(np.median([2990 - 10 * i for i in range(8)]))
    assert res["blocks"] == 2


def test_trace_entry_points_refuse_without_trace_build():
    # the in-tree library is built without -DHSTU_TRACE: no CUDA call is made
    lib = ops.load(ops.os.path.join(ops._HERE, "lib", "libhstu.so"))
    buf = np.zeros(8, dtype=np.uint64)
    for kernel in (0, 1):
        assert lib.hstu_debug_trace_read(kernel, buf.ctypes.data, ctypes.c_size_t(buf.nbytes)) == 2
        assert lib.hstu_debug_trace_clear(kernel) == 2
    assert lib.hstu_debug_trace_read(7, buf.ctypes.data, ctypes.c_size_t(buf.nbytes)) == 1
    assert lib.hstu_debug_trace_clear(7) == 1
