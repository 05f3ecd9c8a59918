"""A bounded device wait that runs out is reported, and the device stays usable.

Every wait inside kvp_score is bounded in time. This makes one run out on purpose: the
debug build of the library (device-side checks plus a fault-injection hook) is told
that every KV head has one more peer CTA than it really has, so each CTA's wait for its
head's peers can never be satisfied, and every wait gives up after 1 ms. The kernel then
records an error code in the workspace and returns early; kvp_workspace_status must read
KVP_ERR_TIMEOUT back. With the hook cleared, the next call on a fresh workspace must score
correctly and report KVP_OK. Nothing faults or hangs: the wait ends by its own limit.
"""
import ctypes
import importlib.util
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_utils import check_scores, to_dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KVP_ERR_TIMEOUT = 6


def checks_library():
    spec = importlib.util.spec_from_file_location(
        "kvp_build", os.path.join(ROOT, "token_eviction_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    lib = ctypes.CDLL(mod.build_checks())
    P = ctypes.c_void_p
    lib.kvp_score.argtypes = [P] * 8 + [ctypes.c_size_t, P]
    lib.kvp_score.restype = ctypes.c_int
    lib.kvp_workspace_bytes.argtypes = [P]
    lib.kvp_workspace_bytes.restype = ctypes.c_size_t
    lib.kvp_workspace_status.argtypes = [P, P]
    lib.kvp_workspace_status.restype = ctypes.c_int
    lib.kvp_debug_set_fault.argtypes = [ctypes.c_int, ctypes.c_ulonglong]
    lib.kvp_debug_set_fault.restype = None
    lib.kvp_debug_take_check.argtypes = [P]
    lib.kvp_debug_take_check.restype = ctypes.c_int
    return lib


def test_wait_that_runs_out_is_reported_and_next_call_is_clean():
    import token_eviction_b200 as m
    lib = checks_library()
    wl = synth.small("llama8b_32k", hq=8, hkv=2, seq_len=3000, window=32, budget=300)
    inp = synth.make_inputs(wl)
    sh = m.make_shape(*wl.shape_tuple())
    q, k, v = to_dev(inp.q_win), to_dev(inp.k), to_dev(inp.v)
    b, hkv, L = wl.batch, wl.hkv, wl.seq_len
    nbytes = lib.kvp_workspace_bytes(ctypes.byref(sh))
    stream = torch.cuda.current_stream().cuda_stream

    def score_into(ws, out):
        st = lib.kvp_score(ctypes.byref(sh), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                           None, None, ws.data_ptr(), nbytes, stream)
        assert st == 0, m.kvp_status_string(st)
        return lib.kvp_workspace_status(ws.data_ptr(), stream)

    try:
        lib.kvp_debug_set_fault(1, 1_000_000)          # a peer that never arrives; 1 ms waits
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        out = torch.zeros((b, hkv, L), dtype=torch.float32, device="cuda")
        assert score_into(ws, out) == KVP_ERR_TIMEOUT
    finally:
        lib.kvp_debug_set_fault(0, 0)
    torch.cuda.synchronize()                            # the context is still usable

    ws2 = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out2 = torch.empty((b, hkv, L), dtype=torch.float32, device="cuda")
    assert score_into(ws2, out2) == 0
    # the first workspace is cleared by the next call made with it
    assert score_into(ws, out) == 0
    _, _, ora = oracle.oracle_score(inp.q_win, inp.k, inp.v)
    check_scores(out2.cpu().numpy(), ora, "S")
    check_scores(out.cpu().numpy(), ora, "S")
    chk = np.zeros(4, dtype=np.int32)
    assert lib.kvp_debug_take_check(chk.ctypes.data) == 0
    assert chk[0] == 0, f"device-side bounds check {chk.tolist()}"
