"""The C ABI library loads, exports what include/ltxattn.h declares, and rejects bad
arguments on the host before any CUDA call (no GPU needed)."""
import ctypes

import pytest

from joint_audio_video_flash_b200 import build, ltxattn


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ltxattn.load()


def test_exports_every_declared_symbol(lib):
    declared = ltxattn.header_entry_points()
    assert len(declared) >= 5
    for name in ("ltxattn_create", "ltxattn_forward", "ltxattn_destroy"):
        assert name in declared
    for name in declared:
        assert hasattr(lib, name), name
    listed = [lib.ltxattn_entry_point_name(i).decode()
              for i in range(lib.ltxattn_num_entry_points())]
    assert sorted(listed) == sorted(declared)
    assert lib.ltxattn_entry_point_name(-1) is None
    assert lib.ltxattn_entry_point_name(len(listed)) is None


def test_status_strings(lib):
    names = [ltxattn.status_string(i) for i in range(8)]
    assert names[0] == "LTXATTN_OK"
    assert names[5] == "LTXATTN_ERR_DEVICE_TIMEOUT"
    assert names[7] == "LTXATTN_ERR_WORKSPACE_GUARD"
    assert len(set(names)) == 8
    assert ltxattn.status_string(99) == "LTXATTN_UNKNOWN_STATUS"


def test_debug_build_loads_and_exports_the_same_symbols():
    # the guard-word build (-DLTXATTN_DEBUG) is a drop-in for the release library
    path = build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in ltxattn.header_entry_points():
        assert hasattr(dbg, name), name
    dbg.ltxattn_status_string.restype = ctypes.c_char_p
    assert dbg.ltxattn_status_string(7) == b"LTXATTN_ERR_WORKSPACE_GUARD"


# fake, never dereferenced device addresses: validation fails before any CUDA call
Q, K, V, O = 1 << 20, 2 << 20, 3 << 20, 4 << 20


def fwd(lib, q=Q, k=K, v=V, o=O, q_len=128, kv_len=128, valid=128, batch=2, heads=4, d=64,
        scale=0.125, splits=None):
    args = [ctypes.c_void_p(q), ctypes.c_void_p(k), ctypes.c_void_p(v), ctypes.c_void_p(o),
            q_len, kv_len, valid, batch, heads, d, ctypes.c_float(scale)]
    if splits is None:
        return lib.ltxattn_forward(*args, None)
    return lib.ltxattn_forward_ex(*args, splits, None, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=0), ltxattn.ERR_INVALID_ARG),
    (dict(o=0), ltxattn.ERR_INVALID_ARG),
    (dict(q_len=0), ltxattn.ERR_INVALID_ARG),
    (dict(kv_len=0, valid=0), ltxattn.ERR_INVALID_ARG),
    (dict(valid=0), ltxattn.ERR_INVALID_ARG),
    (dict(valid=129), ltxattn.ERR_INVALID_ARG),
    (dict(batch=0), ltxattn.ERR_INVALID_ARG),
    (dict(heads=-1), ltxattn.ERR_INVALID_ARG),
    (dict(scale=0.0), ltxattn.ERR_INVALID_ARG),
    (dict(scale=-1.0), ltxattn.ERR_INVALID_ARG),
    (dict(scale=float("nan")), ltxattn.ERR_INVALID_ARG),
    (dict(scale=float("inf")), ltxattn.ERR_INVALID_ARG),
    (dict(d=96), ltxattn.ERR_UNSUPPORTED),
    (dict(d=256), ltxattn.ERR_UNSUPPORTED),
    (dict(q_len=(1 << 24) + 1), ltxattn.ERR_UNSUPPORTED),
    (dict(heads=1025), ltxattn.ERR_UNSUPPORTED),
    (dict(batch=1025), ltxattn.ERR_UNSUPPORTED),
    (dict(q=Q + 8), ltxattn.ERR_MISALIGNED),
    (dict(k=K + 2), ltxattn.ERR_MISALIGNED),
    (dict(o=O + 4), ltxattn.ERR_MISALIGNED),
    (dict(o=Q), ltxattn.ERR_INVALID_ARG),             # out aliases q
    (dict(o=K + 4096), ltxattn.ERR_INVALID_ARG),      # out overlaps k
    (dict(splits=-1), ltxattn.ERR_INVALID_ARG),
])
def test_host_validation(lib, kw, status):
    assert fwd(lib, **kw) == status


def test_validation_order_invalid_before_unsupported_before_misaligned(lib):
    assert fwd(lib, valid=0, d=96, q=Q + 2) == ltxattn.ERR_INVALID_ARG
    assert fwd(lib, d=96, q=Q + 2) == ltxattn.ERR_UNSUPPORTED


def test_valid_arguments_reach_cuda(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-only expectation: no CUDA device")
    # validation passes, then the first CUDA call fails without a device
    assert fwd(lib) in (ltxattn.ERR_CUDA, ltxattn.ERR_NOT_INITIALIZED)
    assert lib.ltxattn_create() == ltxattn.ERR_CUDA
    assert lib.ltxattn_selftest_wait_timeout(ctypes.c_ulonglong(10), None) == \
        ltxattn.ERR_INVALID_ARG


def na3d(lib, q=Q, k=K, v=V, o=O, batch=1, grid=(2, 8, 8), heads=2, d=64, win=(1, 3, 3),
         scale=0.125):
    return lib.ltxattn_na3d_forward(ctypes.c_void_p(q), ctypes.c_void_p(k), ctypes.c_void_p(v),
                                    ctypes.c_void_p(o), batch, *grid, heads, d, *win,
                                    ctypes.c_float(scale), None)


@pytest.mark.parametrize("kw,status", [
    (dict(v=0), ltxattn.ERR_INVALID_ARG),
    (dict(batch=0), ltxattn.ERR_INVALID_ARG),
    (dict(grid=(0, 8, 8)), ltxattn.ERR_INVALID_ARG),
    (dict(win=(2, 3, 3)), ltxattn.ERR_INVALID_ARG),       # even window
    (dict(win=(1, 3, 0)), ltxattn.ERR_INVALID_ARG),
    (dict(win=(3, 3, 3)), ltxattn.ERR_INVALID_ARG),       # window longer than its axis (t = 2)
    (dict(win=(1, 9, 3)), ltxattn.ERR_INVALID_ARG),
    (dict(scale=float("nan")), ltxattn.ERR_INVALID_ARG),
    (dict(d=96), ltxattn.ERR_UNSUPPORTED),
    (dict(grid=(2, 1 << 12, 1 << 12)), ltxattn.ERR_UNSUPPORTED),  # 2^25 tokens
    (dict(heads=1025), ltxattn.ERR_UNSUPPORTED),
    (dict(k=K + 8), ltxattn.ERR_MISALIGNED),
    (dict(o=V + 64), ltxattn.ERR_INVALID_ARG),             # out overlaps v
])
def test_na3d_host_validation(lib, kw, status):
    assert na3d(lib, **kw) == status


def qk(lib, q=Q, k=K, qo=O, ko=O + (1 << 20), wq=9 << 20, wk=10 << 20, cos=11 << 20,
       sin=12 << 20, batch=1, seq=16, heads=8, d=128, eps=1e-6):
    return lib.ltxattn_qk_norm_rope(*(ctypes.c_void_p(x) for x in (q, k, qo, ko, wq, wk)),
                                    ctypes.c_void_p(cos), ctypes.c_void_p(sin), batch, seq,
                                    heads, d, ctypes.c_float(eps), None)


@pytest.mark.parametrize("kw,status", [
    (dict(wq=0), ltxattn.ERR_INVALID_ARG),
    (dict(seq=0), ltxattn.ERR_INVALID_ARG),
    (dict(eps=-1.0), ltxattn.ERR_INVALID_ARG),
    (dict(eps=float("inf")), ltxattn.ERR_INVALID_ARG),
    (dict(heads=3, d=64), ltxattn.ERR_UNSUPPORTED),        # inner 192
    (dict(heads=4, d=36), ltxattn.ERR_UNSUPPORTED),        # head_dim not a multiple of 8
    (dict(heads=128, d=128), ltxattn.ERR_UNSUPPORTED),     # inner 16384
    (dict(cos=(11 << 20) + 4), ltxattn.ERR_MISALIGNED),
    (dict(ko=Q), ltxattn.ERR_INVALID_ARG),                 # k_out overlaps q
    (dict(qo=K), ltxattn.ERR_INVALID_ARG),                 # q_out overlaps k
])
def test_qk_norm_rope_host_validation(lib, kw, status):
    assert qk(lib, **kw) == status


def partial(lib, q=Q, k=K, v=V, o=O, lse=O + (1 << 24), q_len=128, kv_len=128, valid=128,
            batch=2, heads=4, d=64, scale=0.125):
    return lib.ltxattn_forward_partial(*(ctypes.c_void_p(x) for x in (q, k, v, o, lse)),
                                       q_len, kv_len, valid, batch, heads, d,
                                       ctypes.c_float(scale), None)


@pytest.mark.parametrize("kw,status", [
    (dict(lse=0), ltxattn.ERR_INVALID_ARG),
    (dict(valid=0), ltxattn.ERR_INVALID_ARG),
    (dict(d=96), ltxattn.ERR_UNSUPPORTED),
    (dict(lse=O + (1 << 24) + 4), ltxattn.ERR_MISALIGNED),
    (dict(o=K), ltxattn.ERR_INVALID_ARG),                  # o_part overlaps k
    (dict(lse=Q + 1024), ltxattn.ERR_INVALID_ARG),         # lse overlaps q
    (dict(lse=O + 4096), ltxattn.ERR_INVALID_ARG),         # lse overlaps o_part
])
def test_forward_partial_host_validation(lib, kw, status):
    assert partial(lib, **kw) == status


def comb(lib, o=O, lse=O + (1 << 24), out=Q, parts=2, q_len=100, batch=2, heads=4, d=64):
    return lib.ltxattn_combine(ctypes.c_void_p(o), ctypes.c_void_p(lse), ctypes.c_void_p(out),
                               parts, q_len, batch, heads, d, None)


@pytest.mark.parametrize("kw,status", [
    (dict(out=0), ltxattn.ERR_INVALID_ARG),
    (dict(parts=0), ltxattn.ERR_INVALID_ARG),
    (dict(q_len=0), ltxattn.ERR_INVALID_ARG),
    (dict(d=32), ltxattn.ERR_UNSUPPORTED),
    (dict(parts=65537), ltxattn.ERR_UNSUPPORTED),
    (dict(out=Q + 8), ltxattn.ERR_MISALIGNED),
    (dict(out=O + 1024), ltxattn.ERR_INVALID_ARG),         # out overlaps the partials
])
def test_combine_host_validation(lib, kw, status):
    assert comb(lib, **kw) == status


def test_new_calls_reach_cuda_with_valid_arguments(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-only expectation: no CUDA device")
    assert na3d(lib) in (ltxattn.ERR_CUDA, ltxattn.ERR_NOT_INITIALIZED)
    assert qk(lib) in (ltxattn.ERR_CUDA, ltxattn.ERR_NOT_INITIALIZED)
    assert qk(lib, qo=Q, ko=K) in (ltxattn.ERR_CUDA, ltxattn.ERR_NOT_INITIALIZED)  # in place
    assert partial(lib) in (ltxattn.ERR_CUDA, ltxattn.ERR_NOT_INITIALIZED)
    assert comb(lib) == ltxattn.ERR_CUDA


def group(lib, *calls):
    arr = (ltxattn._Call * max(len(calls), 1))()
    for i, c in enumerate(calls):
        d = dict(q=Q, k=K, v=V, out=O, q_len=128, kv_len=128, kv_valid_len=126, batch=2,
                 heads=4, head_dim=64, scale=0.125)
        d.update(c)
        arr[i] = ltxattn._Call(**d)
    return lib.ltxattn_forward_grouped(ctypes.cast(arr, ctypes.c_void_p), len(calls), None)


# a second call's tensors, 16 MiB further on
Q2, K2, V2, O2 = (x + (16 << 20) for x in (Q, K, V, O))
SECOND = dict(q=Q2, k=K2, v=V2, out=O2)


@pytest.mark.parametrize("calls,status", [
    ((), ltxattn.ERR_INVALID_ARG),                                    # no call
    (({"q": 0},), ltxattn.ERR_INVALID_ARG),                           # a call's own checks
    (({}, dict(SECOND, kv_valid_len=0)), ltxattn.ERR_INVALID_ARG),    # ... in any position
    (({}, dict(SECOND, head_dim=96)), ltxattn.ERR_UNSUPPORTED),
    (({}, dict(SECOND, k=K2 + 8)), ltxattn.ERR_MISALIGNED),
    (({}, dict(SECOND, out=O)), ltxattn.ERR_INVALID_ARG),             # two calls write one out
    (({}, dict(SECOND, out=Q + 4096)), ltxattn.ERR_INVALID_ARG),      # out over another's q
    (({}, dict(SECOND, q=O)), ltxattn.ERR_INVALID_ARG),               # another reads this out
    (({}, dict(SECOND, v=O + 1024)), ltxattn.ERR_INVALID_ARG),
])
def test_grouped_host_validation(lib, calls, status):
    assert group(lib, *calls) == status


def test_grouped_limits_and_shared_inputs(lib):
    import torch
    calls = [dict(q=Q + (i << 24), k=K + (i << 24), v=V + (i << 24), out=O + (i << 24))
             for i in range(65)]
    assert group(lib, *calls) == ltxattn.ERR_UNSUPPORTED             # above LTXATTN_MAX_GROUP
    if torch.cuda.is_available():
        return
    # two calls reading the same k and v (a2v and audio self share the audio keys): valid,
    # so the call gets as far as the context lookup
    assert group(lib, {}, dict(q=Q2, out=O2)) in (ltxattn.ERR_CUDA,
                                                   ltxattn.ERR_NOT_INITIALIZED)
