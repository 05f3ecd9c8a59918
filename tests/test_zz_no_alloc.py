"""kvp_score_static: the scoring call without a caller-provided workspace.

Some callers cannot allocate device memory when they evict (a serving engine whose
memory pool owns the whole device, code that may not allocate after start-up); for
them the library keeps its scratch in a fixed array of its own. This checks, through
the C ABI, that two calls in a row give the same scores as kvp_score with a workspace,
and that a shape needing more scratch than the array holds is refused. The file sorts
last so that a failure here stops a -x run only after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from tests.parity_utils import check_scores, to_dev

pytestmark = pytest.mark.gpu

STATIC_BYTES = 2 << 20   # KVP_STATIC_SCRATCH_BYTES in include/kvp.h


def _lib():
    import token_eviction_b200 as m
    f = m._lib.kvp_score_static
    f.argtypes = [ctypes.POINTER(m.KvpShape)] + [ctypes.c_void_p] * 7
    f.restype = ctypes.c_int
    return m, f


@pytest.mark.parametrize("name,with_s1_s2", [("llama8b_32k", True), ("gqa7_batched", True), ("tiny", True),
                                             ("long_128k_b10", False), ("llama8b_32k", False)])
def test_static_scratch_matches_workspace_call(name, with_s1_s2):
    m, kvp_score_static = _lib()
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl)
    sh = m.make_shape(*wl.shape_tuple())
    assert m.kvp_workspace_bytes(sh) <= STATIC_BYTES
    q, k, v = to_dev(inp.q_win), to_dev(inp.k), to_dev(inp.v)
    b, hkv, L = wl.batch, wl.hkv, wl.seq_len
    ref = [torch.empty((b, hkv, L), dtype=torch.float32, device="cuda") for _ in range(3)]
    m.kvp_score(sh, q, k, v, *ref)
    stream = torch.cuda.current_stream().cuda_stream
    nout = 3 if with_s1_s2 else 1
    for _ in range(2):                     # two calls in a row reuse the same scratch
        out = [torch.full((b, hkv, L), float("nan"), dtype=torch.float32, device="cuda")
               for _ in range(nout)]
        ptrs = [t.data_ptr() for t in out] + [None] * (3 - nout)
        st = kvp_score_static(ctypes.byref(sh), q.data_ptr(), k.data_ptr(), v.data_ptr(), *ptrs, stream)
        assert st == 0, m.kvp_status_string(st)
        assert m._lib.kvp_score_static_status(stream) == 0
        torch.cuda.synchronize()
        for got, want, what in zip(out, ref, ("S", "S1", "S2")):
            check_scores(got.cpu().numpy(), want.cpu().numpy().astype(np.float64), what)


def test_static_scratch_refuses_oversized_shapes():
    m, kvp_score_static = _lib()
    sh = m.make_shape(256, 32, 8, 128, 4096, 128, 256)
    assert m.kvp_workspace_bytes(sh) > STATIC_BYTES
    t = torch.empty(16, dtype=torch.float32, device="cuda")
    st = kvp_score_static(ctypes.byref(sh), t.data_ptr(), t.data_ptr(), t.data_ptr(),
                          t.data_ptr(), None, None, None)
    assert st == 4   # KVP_ERR_WORKSPACE, before anything is launched
