"""The C-ABI library loads without a GPU, exports every entry point that
include/hstu.h declares, and its host-side validation rejects bad arguments
before any CUDA call (so these run on a CPU-only machine).

The validation checks hand the library dummy pointers.  They run in a child
process started with CUDA_VISIBLE_DEVICES="" (see ``hidden``), so that even if
validation regressed and a call went on to launch, no GPU could be reached
with those pointers: the launch would fail for want of a device.
"""
import ctypes
import multiprocessing as mp
import os
import re

import numpy as np
import pytest

from hstu_pointwise_attention_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hidden():
    """A one-process pool whose worker sees no CUDA device."""
    old = os.environ.get("CUDA_VISIBLE_DEVICES")
    os.environ["CUDA_VISIBLE_DEVICES"] = ""
    try:
        pool = mp.get_context("spawn").Pool(1)
    finally:
        if old is None:
            del os.environ["CUDA_VISIBLE_DEVICES"]
        else:
            os.environ["CUDA_VISIBLE_DEVICES"] = old
    yield pool
    pool.close()
    pool.join()


def _no_device_visible():
    return os.environ.get("CUDA_VISIBLE_DEVICES") == ""


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hstu.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hstu_[a-z_]+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ("hstu_attn_fwd", "hstu_attn_bwd", "hstu_layer_fwd", "hstu_attn_workspace_size",
              "hstu_get_device_error", "hstu_debug_buckets"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(ops.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(ops.EXPORTED) <= set(declared_functions())


def declared_parameter_counts():
    """{function: number of parameters} from include/hstu.h."""
    src = open(os.path.join(ROOT, "include", "hstu.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(hstu_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", src, flags=re.S):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header():
    """Every function the binding declares argtypes for takes exactly as many
    arguments as include/hstu.h says (a short list would shift the stream)."""
    counts = declared_parameter_counts()
    checked = 0
    for name in ops.EXPORTED:
        at = getattr(ops.LIB, name).argtypes
        if at is None:
            continue
        assert len(at) == counts[name], (name, len(at), counts[name])
        checked += 1
    assert checked >= 15


def test_version_and_status_strings():
    assert "sm_100a" in ops.version()
    for code, name in ops.STATUS.items():
        assert ops.LIB.hstu_status_string(code).decode() == name


def _params(batch=2, H=2, d=64, msl=64, nb=32, s=2, mask=0):
    p = ops.AttnParams()
    p.batch, p.num_heads, p.d_qk, p.d_v, p.max_seq_len = batch, H, d, d, msl
    p.num_pos_buckets = p.num_time_buckets = nb
    p.time_bucket_sub_bits = s
    p.mask = mask
    p.dtype = ops.BF16
    for f in ("q", "k", "v", "o", "do", "dq", "dk", "dv"):
        setattr(p, f + "_row_stride", H * d)
    p.alpha, p.silu_scale = 0.125, 1.0 / msl
    return p


def _ws(p, off, bwd=0):
    n = ctypes.c_size_t(0)
    rc = ops.LIB.hstu_attn_workspace_size(ctypes.byref(p), off.ctypes.data, bwd, ctypes.byref(n))
    return rc, n.value


def test_workspace_size_grows_with_tokens_and_backward():
    p = _params()
    rc1, n1 = _ws(p, np.array([0, 10, 64], np.int64))
    rc2, n2 = _ws(p, np.array([0, 64, 128], np.int64))
    rc3, n3 = _ws(p, np.array([0, 64, 128], np.int64), bwd=1)
    assert rc1 == rc2 == rc3 == ops.HSTU_OK
    assert 0 < n1 <= n2 < n3
    # backward adds a float32 dQ accumulator of T * H * d_qk
    assert n3 - n2 >= 128 * 2 * 64 * 4


# ---- checks that hand the library dummy pointers: run in the hidden worker ----

_MUTATIONS = {
    "num_heads": ("num_heads", 0), "d_qk": ("d_qk", 0), "d_v": ("d_v", 300),
    "num_pos_buckets": ("num_pos_buckets", 0), "sub_bits": ("time_bucket_sub_bits", 9),
    "mask": ("mask", 7), "dtype": ("dtype", 5), "impl": ("impl", 9),
    "q_row_stride": ("q_row_stride", 10), "alpha": ("alpha", float("nan")),
}


def _invalid_argument_rc(field, off):
    assert _no_device_visible()
    p = _params(batch=len(off) - 1)
    if field is not None:
        setattr(p, *_MUTATIONS[field])
    o = np.array(off, np.int64)
    # Every pointer is a dummy non-null host address: the call must fail in
    # validation, before it could touch them.
    dummy = ctypes.c_void_p(16)
    return ops.LIB.hstu_attn_fwd(ctypes.byref(p), o.ctypes.data, None, dummy, dummy, dummy,
                                 dummy, dummy, dummy, dummy, dummy, 1 << 30, None)


@pytest.mark.parametrize("field, off", [(f, [0, 5]) for f in _MUTATIONS] + [
    (None, [1, 5]),            # offsets[0] != 0
    (None, [0, 5, 3]),         # decreasing
    (None, [0, 65]),           # longer than max_seq_len
])
def test_invalid_arguments_are_rejected_before_any_launch(hidden, field, off):
    rc = hidden.apply(_invalid_argument_rc, (field, off))
    assert rc == 1, ops.STATUS.get(rc)


def _mfalcon_candidate_rcs():
    assert _no_device_visible()
    p = _params(batch=1, mask=ops.MASK_MFALCON)
    o = np.array([0, 10], np.int64)
    dummy = ctypes.c_void_p(16)
    rcs = []
    for nc in (None, np.array([11], np.int32), np.array([-1], np.int32)):
        rcs.append(ops.LIB.hstu_attn_fwd(ctypes.byref(p), o.ctypes.data,
                                         None if nc is None else nc.ctypes.data, dummy, dummy,
                                         dummy, dummy, dummy, dummy, dummy, dummy, 1 << 30, None))
    return rcs


def test_mfalcon_requires_valid_candidate_counts(hidden):
    assert hidden.apply(_mfalcon_candidate_rcs) == [1, 1, 1]


def _workspace_rcs():
    assert _no_device_visible()
    p = _params(batch=1)
    o = np.array([0, 10], np.int64)
    rc, need = _ws(p, o)
    assert rc == 0
    dummy = ctypes.c_void_p(16)
    small = ops.LIB.hstu_attn_fwd(ctypes.byref(p), o.ctypes.data, None, dummy, dummy, dummy,
                                  dummy, dummy, dummy, dummy, ctypes.c_void_p(256), need - 1, None)
    skew = ops.LIB.hstu_attn_fwd(ctypes.byref(p), o.ctypes.data, None, dummy, dummy, dummy,
                                 dummy, dummy, dummy, dummy, ctypes.c_void_p(256 + 16), need, None)
    return small, skew


def test_workspace_too_small_or_misaligned_is_rejected(hidden):
    assert hidden.apply(_workspace_rcs) == (3, 3)


def _missing_pointer_rc():
    assert _no_device_visible()
    p = _params(batch=1)
    o = np.array([0, 10], np.int64)
    dummy = ctypes.c_void_p(16)
    return ops.LIB.hstu_attn_fwd(ctypes.byref(p), o.ctypes.data, None, dummy, None, dummy, dummy,
                                 dummy, dummy, dummy, ctypes.c_void_p(256), 1 << 30, None)


def test_missing_pointer_is_rejected(hidden):
    assert hidden.apply(_missing_pointer_rc) == 1


def _wait_probe_rcs():
    assert _no_device_visible()
    return [ops.LIB.hstu_debug_wait_probe(None, 1 << 20, 1000, None),       # no workspace
            ops.LIB.hstu_debug_wait_probe(256 + 16, 1 << 20, 1000, None),   # misaligned
            ops.LIB.hstu_debug_wait_probe(256, 8, 1000, None),              # too small
            ops.LIB.hstu_debug_wait_probe(256, 1 << 20, 0, None)]           # no limit


def test_wait_probe_rejects_bad_arguments_before_any_launch(hidden):
    assert hidden.apply(_wait_probe_rcs) == [3, 3, 3, 1]


def _noalloc_oversize_rc():
    assert _no_device_visible()
    # 2^22 tokens need 16 MiB of float timestamps, more than the 8 MiB array;
    # the call must refuse from the host-side layout, before any CUDA call.
    T = 1 << 22
    off = np.array([0, T], np.int64)
    p = _params(batch=1, H=2, d=64, msl=T, nb=8, s=1)
    dummy = ctypes.c_void_p(16)
    return ops.LIB.hstu_attn_fwd_noalloc(ctypes.byref(p), off.ctypes.data, None, dummy, dummy,
                                         dummy, dummy, dummy, dummy, dummy, None)


def test_noalloc_rejects_problem_larger_than_its_scratch_before_any_cuda_call(hidden):
    assert hidden.apply(_noalloc_oversize_rc) == 3


def test_layer_validation():
    lp = ops.LayerParams()
    lp.attn = _params(batch=1, H=2, d=64)
    lp.d_model = 100        # not a multiple of 8
    lp.ln_eps = 1e-5
    n = ctypes.c_size_t(0)
    o = np.array([0, 10], np.int64)
    assert ops.LIB.hstu_layer_workspace_size(ctypes.byref(lp), o.ctypes.data,
                                             ctypes.byref(n)) == 1
    lp.d_model = 128
    assert ops.LIB.hstu_layer_workspace_size(ctypes.byref(lp), o.ctypes.data,
                                             ctypes.byref(n)) == 0
    assert n.value > 10 * 4 * 128 * 2
    lp.attn.dtype = ops.F32
    assert ops.LIB.hstu_layer_workspace_size(ctypes.byref(lp), o.ctypes.data,
                                             ctypes.byref(n)) == 2
