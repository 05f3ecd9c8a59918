"""CPU oracle for prefill KV-cache token eviction (S1 * S2 scores, top-B select, gather).

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only users. The product path (the package
``token_eviction_b200``) never imports this module, and this module imports nothing
from it; the two share only the seeded input generator ``synth``.

The arithmetic lives in ``kvp_oracle.c``: the plain definition of the method in double
precision, following "Preserving Large Activations: The Key to KV Cache Pruning"
(SlimKV) Eq. 3 (S1), Eq. 4 (S2), Eq. 5 (S = S1 * S2) and Listing 1 (window_size,
max_capacity_prompt), with C = sqrt(d) read from the CurDKV rebuttal page's statement
of attention, softmax(Q K^T / C) V. This wrapper only marshals numpy arrays.

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed forms,
invariants, library routines and brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvp_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile ``kvp_oracle.c`` into ``liboracle.so`` (gcc -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _get():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i, p = ctypes.c_int, ctypes.c_void_p
        lib.oracle_score.argtypes = [i, i, i, i, i, i, p, p, p, p, p, p, p]
        lib.oracle_score.restype = i
        lib.oracle_select.argtypes = [i, i, i, i, p, p]
        lib.oracle_select.restype = i
        lib.oracle_compact.argtypes = [i, i, i, i, p, p, p, p, p]
        lib.oracle_compact.restype = i
        lib.oracle_select_policy.argtypes = [i, i, i, i, i, i, i, i, p, p, p, p]
        lib.oracle_select_policy.restype = i
        lib.oracle_leverage.argtypes = [i, i, i, i, p, p, p, p, p, p]
        lib.oracle_leverage.restype = i
        lib.oracle_select_adaptive.argtypes = [i, i, i, i, i, ctypes.c_double, p, p, p]
        lib.oracle_select_adaptive.restype = i
        _lib = lib
    return _lib


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 tensors are passed as uint16 bit patterns"
    return a


def oracle_score(q_win, k, v, want_lse: bool = False):
    """S1, S2, S [b, hkv, L] (float64) and optionally lse [b, hq, w].

    q_win [b, hq, w, d], k and v [b, hkv, L, d]: bf16 bit patterns (uint16).
    """
    q_win, k, v = _u16(q_win), _u16(k), _u16(v)
    b, hq, w, d = q_win.shape
    _, hkv, L, _ = k.shape
    assert k.shape == v.shape == (b, hkv, L, d)
    s1 = np.empty((b, hkv, L))
    s2 = np.empty((b, hkv, L))
    s = np.empty((b, hkv, L))
    lse = np.empty((b, hq, w)) if want_lse else None
    rc = _get().oracle_score(b, hq, hkv, d, L, w, q_win.ctypes.data, k.ctypes.data, v.ctypes.data,
                             s1.ctypes.data, s2.ctypes.data, s.ctypes.data,
                             None if lse is None else lse.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_score: bad shape")
    return (s1, s2, s, lse) if want_lse else (s1, s2, s)


def oracle_select(score, window: int, budget: int):
    """Kept positions [..., B] (int32, ascending) for scores [..., L] (any float dtype)."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    lead, L = score.shape[:-1], score.shape[-1]
    rows = int(np.prod(lead)) if lead else 1
    idx = np.empty(lead + (budget,), dtype=np.int32)
    rc = _get().oracle_select(rows, L, window, budget, score.ctypes.data, idx.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_select: bad window/budget")
    return idx


MODE_PRODUCT, MODE_S1, MODE_S2 = 0, 1, 2


def oracle_select_policy(s1, s2, window: int, budget: int, sinks: int = 0, kernel: int = 1,
                         mode: int = MODE_PRODUCT, fp32_key: bool = False, want_key: bool = False):
    """Kept positions [..., B] under a selection policy: sinks [0, s) always kept, S1
    max-pooled with an odd kernel over the positions before the window, ranked by
    pool(S1) * S2 (mode 0), pool(S1) (mode 1) or S2 (mode 2). ``fp32_key`` forms the key
    in single precision with subnormals flushed, as the CUDA path does."""
    s1 = np.ascontiguousarray(s1, dtype=np.float64)
    s2 = np.ascontiguousarray(s2, dtype=np.float64)
    assert s1.shape == s2.shape
    lead, L = s1.shape[:-1], s1.shape[-1]
    rows = int(np.prod(lead)) if lead else 1
    idx = np.empty(lead + (budget,), dtype=np.int32)
    key = np.full(s1.shape, np.nan) if want_key else None
    rc = _get().oracle_select_policy(rows, L, window, budget, sinks, kernel, mode, int(fp32_key),
                                     s1.ctypes.data, s2.ctypes.data, idx.ctypes.data,
                                     None if key is None else key.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_select_policy: bad policy")
    return (idx, key) if want_key else idx


def oracle_compact(k, v, idx):
    """k_out, v_out [..., B, d] gathered row by row (bit copies)."""
    k, v = _u16(k), _u16(v)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    L, d = k.shape[-2], k.shape[-1]
    B = idx.shape[-1]
    rows = int(np.prod(k.shape[:-2]))
    k_out = np.empty(k.shape[:-2] + (B, d), dtype=np.uint16)
    v_out = np.empty_like(k_out)
    rc = _get().oracle_compact(rows, L, d, B, k.ctypes.data, v.ctypes.data, idx.ctypes.data,
                               k_out.ctypes.data, v_out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_compact: index out of range")
    return k_out, v_out


def oracle_layer(q_win, k, v, window: int, budget: int):
    """The whole path for one layer: scores, kept positions, compacted K and V."""
    s1, s2, s = oracle_score(q_win, k, v)
    idx = oracle_select(s, window, budget)
    k_out, v_out = oracle_compact(k, v, idx)
    return {"s1": s1, "s2": s2, "score": s, "idx": idx, "k_out": k_out, "v_out": v_out}


def oracle_leverage(k, v, g, want_parts: bool = False):
    """CurDKV leverage scores [..., L] (float64): squared row norms of K G and V G, their
    product, normalised to sum 1 over each row's positions (CurDKV rebuttal page,
    "A clearer description of Algorithm 1", steps 1-4). k, v [..., L, d] and g [d, r]:
    bf16 bit patterns. With ``want_parts`` also returns the two squared norms."""
    k, v, g = _u16(k), _u16(v), _u16(g)
    assert k.shape == v.shape and g.ndim == 2 and g.shape[0] == k.shape[-1]
    lead, L, d = k.shape[:-2], k.shape[-2], k.shape[-1]
    r = g.shape[1]
    rows = int(np.prod(lead)) if lead else 1
    score = np.empty(lead + (L,))
    lk = np.empty(lead + (L,)) if want_parts else None
    lv = np.empty(lead + (L,)) if want_parts else None
    rc = _get().oracle_leverage(rows, L, d, r, k.ctypes.data, v.ctypes.data, g.ctypes.data,
                                None if lk is None else lk.ctypes.data,
                                None if lv is None else lv.ctypes.data, score.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_leverage: bad size")
    return (score, lk, lv) if want_parts else score


def oracle_select_adaptive(score, window: int, budget: int, alpha: float):
    """Adaptive per-head budgets (AdaKV, as the CurDKV rebuttal page describes it): score
    [b, hkv, L]. Returns (idx [b, hkv * B] int32: each head's kept positions, ascending,
    heads one after another; counts [b, hkv] int32, window included)."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    b, hkv, L = score.shape
    idx = np.empty((b, hkv * budget), dtype=np.int32)
    counts = np.empty((b, hkv), dtype=np.int32)
    rc = _get().oracle_select_adaptive(b, hkv, L, window, budget, float(alpha), score.ctypes.data,
                                       idx.ctypes.data, counts.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_select_adaptive: bad size or alpha")
    return idx, counts
