"""The C-ABI library loads, exports what include/kvp.h declares, and rejects bad
arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"KVP_API\s+[\w\s\*]*?\b(kvp_\w+)\s*\(", text))
    return names


def test_header_declares_the_boundary():
    assert {"kvp_workspace_bytes", "kvp_score", "kvp_select", "kvp_select_policy", "kvp_compact",
            "kvp_leverage", "kvp_select_adaptive", "kvp_compact_ragged", "kvp_workspace_status",
            "kvp_score_static", "kvp_score_static_status", "kvp_status_string",
            "kvp_last_cuda_error"} <= declared_symbols()


def test_binding_lists_every_declared_symbol():
    import token_eviction_b200 as m
    assert declared_symbols() == set(m.EXPORTED)


def test_library_exports_every_declared_symbol():
    import token_eviction_b200 as m
    lib = ctypes.CDLL(m.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} declared but not exported"


def test_status_strings():
    import token_eviction_b200 as m
    for code, name in m.STATUS_NAMES.items():
        assert m.kvp_status_string(code).startswith(name)
    assert "unknown" in m.kvp_status_string(99)


def test_workspace_bytes_positive_and_zero_for_bad_shapes():
    import token_eviction_b200 as m
    assert m.kvp_workspace_bytes((1, 32, 8, 128, 32768, 32, 2048)) > 0
    assert m.kvp_workspace_bytes((8, 28, 4, 128, 16384, 64, 1024)) > 0
    bad = [(1, 32, 7, 128, 1024, 32, 64),    # hq not a multiple of hkv
           (1, 32, 8, 96, 1024, 32, 64),     # unsupported head_dim
           (1, 32, 8, 128, 1024, 32, 16),    # B < w
           (1, 32, 8, 128, 1024, 32, 1025),  # B > L
           (1, 32, 8, 128, 16, 32, 32),      # w > L
           (1, 32, 1, 128, 4096, 32, 64),    # G * w > 512
           (0, 32, 8, 128, 1024, 32, 64)]
    for s in bad:
        assert m.kvp_workspace_bytes(s) == 0, s


def raw(m):
    return ctypes.CDLL(m.LIB_PATH)


def call_score(m, shape, q=16, k=16, v=16, score=16, ws=16, ws_bytes=1 << 30):
    lib = m._lib
    sh = m.make_shape(*shape)
    return lib.kvp_score(ctypes.byref(sh), q, k, v, score, None, None, ws, ws_bytes, None)


def test_host_side_argument_errors():
    import token_eviction_b200 as m
    ok_shape = (1, 32, 8, 128, 4096, 32, 256)
    assert call_score(m, ok_shape, q=None) == 1
    assert call_score(m, ok_shape, score=None) == 1
    assert m._lib.kvp_score(None, 16, 16, 16, 16, None, None, 16, 1 << 30, None) == 1
    assert call_score(m, (1, 32, 8, 100, 4096, 32, 256)) == 2
    assert call_score(m, ok_shape, k=24) == 3          # misaligned
    assert call_score(m, ok_shape, ws=None) == 4
    assert call_score(m, ok_shape, ws_bytes=8) == 4
    sh = m.make_shape(*ok_shape)
    assert m._lib.kvp_select(ctypes.byref(sh), 16, None, 16, 1 << 30, None) == 1
    assert m._lib.kvp_select(ctypes.byref(sh), 16, 20, 16, 1 << 30, None) == 3
    assert m._lib.kvp_select(ctypes.byref(sh), 16, 16, 16, 0, None) == 4
    assert m._lib.kvp_compact(ctypes.byref(sh), 16, 16, 16, 16, None, None) == 1
    assert m._lib.kvp_compact(ctypes.byref(sh), 16, 16, 16, 16, 8, None) == 3
    bad = m.make_shape(1, 32, 8, 128, 4096, 32, 8)
    assert m._lib.kvp_compact(ctypes.byref(bad), 16, 16, 16, 16, 16, None) == 2


def test_policy_select_rejects_bad_policies_on_the_host():
    import token_eviction_b200 as m
    sh = m.make_shape(1, 32, 8, 128, 4096, 32, 256)

    def call(sinks=0, kernel=1, mode=0, s1=16, s2=16, idx=16, shape=sh):
        pol = m.make_policy(sinks, kernel, mode)
        return m._lib.kvp_select_policy(ctypes.byref(shape), ctypes.byref(pol), s1, s2, idx, None)

    assert call(kernel=2) == 2                # even kernel
    assert call(kernel=0) == 2
    assert call(kernel=257) == 2
    assert call(mode=3) == 2
    assert call(mode=-1) == 2
    assert call(sinks=-1) == 2
    assert call(sinks=225) == 2               # sinks + w > B
    small = m.make_shape(1, 32, 8, 128, 64, 32, 64)
    assert call(sinks=33, shape=small) == 2   # sinks > L - w
    assert call(idx=None) == 1
    assert call(s1=None) == 1                 # product needs S1
    assert call(mode=1, s1=None) == 1
    assert call(mode=2, s2=None) == 1
    assert call(s1=24) == 3                   # misaligned
    assert m._lib.kvp_select_policy(ctypes.byref(sh), None, 16, 16, 16, None) == 1


def test_adaptive_calls_reject_bad_arguments_on_the_host():
    import token_eviction_b200 as m
    sh = m.make_shape(1, 32, 8, 128, 4096, 32, 256)
    lib = m._lib
    ws_bytes = lib.kvp_adaptive_workspace_bytes(ctypes.byref(sh))
    assert ws_bytes >= 8 * 4096 * 4
    assert lib.kvp_adaptive_workspace_bytes(ctypes.byref(m.make_shape(1, 32, 8, 100, 4096, 32, 256))) == 0
    sel = lib.kvp_select_adaptive
    assert sel(ctypes.byref(sh), ctypes.c_float(1.5), 16, 16, 16, 16, ws_bytes, None) == 2
    assert sel(ctypes.byref(sh), ctypes.c_float(float("nan")), 16, 16, 16, 16, ws_bytes, None) == 2
    assert sel(ctypes.byref(sh), ctypes.c_float(0.2), 16, None, 16, 16, ws_bytes, None) == 1
    assert sel(ctypes.byref(sh), ctypes.c_float(0.2), 16, 16, 16, 16, 8, None) == 4
    assert sel(ctypes.byref(sh), ctypes.c_float(0.2), 16, 16, 20, 16, ws_bytes, None) == 3
    assert lib.kvp_compact_ragged(ctypes.byref(sh), 16, 16, 16, None, 16, 16, None) == 1
    assert lib.kvp_compact_ragged(ctypes.byref(sh), 16, 16, 16, 16, 16, 8, None) == 3


def test_binding_validates_tensors_before_calling():
    import torch
    import token_eviction_b200 as m
    sh = m.make_shape(1, 4, 2, 64, 128, 16, 32)
    cpu = torch.zeros((1, 4, 16, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        m.kvp_score(sh, cpu, cpu, cpu, cpu)


def test_static_scratch_call_rejects_bad_arguments_on_the_host():
    """kvp_score_static checks its arguments, and that the shape's scratch fits the
    library's fixed array, before it touches the device."""
    import token_eviction_b200 as m
    f = m._lib.kvp_score_static
    f.argtypes = [ctypes.c_void_p] * 8
    f.restype = ctypes.c_int
    ok = m.make_shape(1, 32, 8, 128, 4096, 32, 256)
    assert f(ctypes.addressof(ok), None, 16, 16, 16, None, None, None) == 1          # NULL q_win
    bad = m.make_shape(1, 32, 8, 100, 4096, 32, 256)
    assert f(ctypes.addressof(bad), 16, 16, 16, 16, None, None, None) == 2          # d = 100
    assert f(ctypes.addressof(ok), 16, 24, 16, 16, None, None, None) == 3           # misaligned k
    big = m.make_shape(256, 32, 8, 128, 4096, 128, 256)
    assert m.kvp_workspace_bytes(big) > (2 << 20)
    assert f(ctypes.addressof(big), 16, 16, 16, 16, None, None, None) == 4          # over 2 MiB


def test_status_call_rejects_bad_workspace_on_the_host():
    import token_eviction_b200 as m
    assert m._lib.kvp_workspace_status(None, None) == 1      # KVP_ERR_NULL
    assert m._lib.kvp_workspace_status(24, None) == 3        # KVP_ERR_ALIGN


def test_static_call_names_the_cuda_error_behind_a_failure():
    """Without a device, kvp_score_static fails when it looks up its scratch array; the
    CUDA error must then be the one kvp_last_cuda_error() names."""
    import torch
    import token_eviction_b200 as m
    if torch.cuda.is_available():
        pytest.skip("needs a host without a usable CUDA device")
    ok = m.make_shape(1, 32, 8, 128, 4096, 32, 256)
    st = m._lib.kvp_score_static(ctypes.byref(ok), 16, 16, 16, 16, None, None, None)
    assert st == 5                                            # KVP_ERR_CUDA
    assert m.kvp_last_cuda_error() != "cudaSuccess"
    assert m._lib.kvp_score_static_status(None) == 5
