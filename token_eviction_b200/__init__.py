"""Prefill KV-cache token eviction (S1 * S2 scores) on NVIDIA B200: Python binding.

A thin ctypes layer over the C-ABI library ``libkvp.so`` (declared in
``include/kvp.h``). It only marshals arguments: every step of the path - the split-L
log-sum-exp pass, the scoring pass, the selection and the compaction - runs in the
library's CUDA kernels. PyTorch provides device memory and streams.

The functions carry the C names:

* ``kvp_workspace_bytes(shape)``
* ``kvp_score(shape, q_win, k, v, score, s1=None, s2=None, workspace=None, stream=None)``
* ``kvp_select(shape, score, idx, workspace=None, stream=None)``
* ``kvp_select_policy(shape, policy, s1, s2, idx, stream=None)``
* ``kvp_leverage(shape, k, v, g, score, workspace=None, stream=None)``
* ``kvp_select_adaptive(shape, alpha, score, idx, counts, workspace=None, stream=None)``
* ``kvp_compact_ragged(shape, k, v, idx, counts, k_out, v_out, stream=None)``
* ``kvp_compact(shape, k, v, idx, k_out, v_out, stream=None)``
* ``kvp_workspace_status(workspace, stream=None)``
* ``kvp_status_string(status)``

plus ``evict_layer``, which allocates the outputs and runs all three calls.

There is no fallback: if ``libkvp.so`` is missing or cannot be loaded, importing this
package raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# KVP_LIBRARY may point at another build of the same library (e.g. one compiled with
# device-side bounds checks); the default is the in-tree build.
LIB_PATH = os.environ.get("KVP_LIBRARY", os.path.join(_HERE, "libkvp.so"))

KVP_OK = 0
STATUS_NAMES = {0: "KVP_OK", 1: "KVP_ERR_NULL", 2: "KVP_ERR_SHAPE", 3: "KVP_ERR_ALIGN",
                4: "KVP_ERR_WORKSPACE", 5: "KVP_ERR_CUDA", 6: "KVP_ERR_TIMEOUT"}


class KvpShape(ctypes.Structure):
    """Mirror of ``kvp_shape``: budget counts every kept position, window included."""
    _fields_ = [("batch", ctypes.c_int32), ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("window", ctypes.c_int32), ("budget", ctypes.c_int32)]

    def __repr__(self):
        return ("KvpShape(batch=%d, hq=%d, hkv=%d, head_dim=%d, seq_len=%d, window=%d, budget=%d)"
                % (self.batch, self.hq, self.hkv, self.head_dim, self.seq_len, self.window, self.budget))


RANK_PRODUCT, RANK_S1, RANK_S2 = 0, 1, 2


class KvpPolicy(ctypes.Structure):
    """Mirror of ``kvp_policy``: sinks always kept, S1 max-pooling kernel, ranking mode."""
    _fields_ = [("sinks", ctypes.c_int32), ("pool_kernel", ctypes.c_int32), ("mode", ctypes.c_int32)]


def make_policy(sinks=0, pool_kernel=1, mode=RANK_PRODUCT) -> KvpPolicy:
    return KvpPolicy(int(sinks), int(pool_kernel), int(mode))


class KvpError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {kvp_status_string(status)}"
        if status == 5:
            msg += f" ({kvp_last_cuda_error()})"
        super().__init__(msg)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python token_eviction_b200/build.py` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P, S = ctypes.c_void_p, ctypes.POINTER(KvpShape)
    lib.kvp_workspace_bytes.argtypes = [S]
    lib.kvp_workspace_bytes.restype = ctypes.c_size_t
    lib.kvp_score.argtypes = [S, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.kvp_score.restype = ctypes.c_int
    lib.kvp_select.argtypes = [S, P, P, P, ctypes.c_size_t, P]
    lib.kvp_select.restype = ctypes.c_int
    lib.kvp_select_policy.argtypes = [S, ctypes.POINTER(KvpPolicy), P, P, P, P]
    lib.kvp_select_policy.restype = ctypes.c_int
    lib.kvp_leverage.argtypes = [S, P, P, P, ctypes.c_int32, P, P, ctypes.c_size_t, P]
    lib.kvp_leverage.restype = ctypes.c_int
    lib.kvp_adaptive_workspace_bytes.argtypes = [S]
    lib.kvp_adaptive_workspace_bytes.restype = ctypes.c_size_t
    lib.kvp_select_adaptive.argtypes = [S, ctypes.c_float, P, P, P, P, ctypes.c_size_t, P]
    lib.kvp_select_adaptive.restype = ctypes.c_int
    lib.kvp_compact_ragged.argtypes = [S, P, P, P, P, P, P, P]
    lib.kvp_compact_ragged.restype = ctypes.c_int
    lib.kvp_compact.argtypes = [S, P, P, P, P, P, P]
    lib.kvp_compact.restype = ctypes.c_int
    lib.kvp_status_string.argtypes = [ctypes.c_int]
    lib.kvp_status_string.restype = ctypes.c_char_p
    lib.kvp_last_cuda_error.argtypes = []
    lib.kvp_last_cuda_error.restype = ctypes.c_char_p
    lib.kvp_workspace_status.argtypes = [P, P]
    lib.kvp_workspace_status.restype = ctypes.c_int
    lib.kvp_score_static.argtypes = [S, P, P, P, P, P, P, P]
    lib.kvp_score_static.restype = ctypes.c_int
    lib.kvp_score_static_status.argtypes = [P]
    lib.kvp_score_static_status.restype = ctypes.c_int
    return lib


_lib = _load()

# Kernel launches one layer's kvp_score + kvp_select + kvp_compact makes: the fused
# scoring kernel (both passes over K), the selection and the gather. kvp_score also
# enqueues one small memset of its workspace counters.
KERNELS_PER_LAYER = 3

EXPORTED = ("kvp_workspace_bytes", "kvp_score", "kvp_select", "kvp_select_policy", "kvp_leverage",
            "kvp_adaptive_workspace_bytes", "kvp_select_adaptive", "kvp_compact_ragged", "kvp_compact",
            "kvp_workspace_status",
            "kvp_score_static", "kvp_score_static_status", "kvp_status_string", "kvp_last_cuda_error")


def make_shape(batch, hq, hkv, head_dim, seq_len, window, budget) -> KvpShape:
    return KvpShape(int(batch), int(hq), int(hkv), int(head_dim), int(seq_len), int(window),
                    int(budget))


def _as_shape(shape) -> KvpShape:
    if isinstance(shape, KvpShape):
        return shape
    if isinstance(shape, dict):
        return make_shape(**shape)
    return make_shape(*shape)


def kvp_status_string(status: int) -> str:
    return _lib.kvp_status_string(int(status)).decode()


def kvp_last_cuda_error() -> str:
    return _lib.kvp_last_cuda_error().decode()


def kvp_workspace_bytes(shape) -> int:
    return int(_lib.kvp_workspace_bytes(ctypes.byref(_as_shape(shape))))


def _ptr(t, name, dtype, shape=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def workspace_for(shape, device=None) -> torch.Tensor:
    n = kvp_workspace_bytes(shape)
    if n == 0:
        raise KvpError(2, "kvp_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def kvp_score(shape, q_win, k, v, score, s1=None, s2=None, workspace=None, stream=None):
    sh = _as_shape(shape)
    b, hq, hkv, d, L, w = sh.batch, sh.hq, sh.hkv, sh.head_dim, sh.seq_len, sh.window
    args = (_ptr(q_win, "q_win", torch.bfloat16, (b, hq, w, d)),
            _ptr(k, "k", torch.bfloat16, (b, hkv, L, d)),
            _ptr(v, "v", torch.bfloat16, (b, hkv, L, d)),
            _ptr(score, "score", torch.float32, (b, hkv, L)),
            _ptr(s1, "s1", torch.float32, (b, hkv, L), optional=True),
            _ptr(s2, "s2", torch.float32, (b, hkv, L), optional=True))
    if workspace is None:
        workspace = workspace_for(sh, k.device)
    st = _lib.kvp_score(ctypes.byref(sh), *args, workspace.data_ptr(), workspace.numel(),
                        _stream(stream))
    if st != KVP_OK:
        raise KvpError(st, "kvp_score")


def kvp_workspace_status(workspace, stream=None) -> int:
    """Device-side status of the last kvp_score on `workspace`: KVP_OK (0) or
    KVP_ERR_TIMEOUT (6) when one of its bounded waits gave up. Synchronises the stream."""
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    return int(_lib.kvp_workspace_status(workspace.data_ptr(), _stream(stream)))


def kvp_select(shape, score, idx, workspace=None, stream=None):
    sh = _as_shape(shape)
    b, hkv, L, B = sh.batch, sh.hkv, sh.seq_len, sh.budget
    ps = _ptr(score, "score", torch.float32, (b, hkv, L))
    pi = _ptr(idx, "idx", torch.int32, (b, hkv, B))
    if workspace is None:
        workspace = workspace_for(sh, score.device)
    st = _lib.kvp_select(ctypes.byref(sh), ps, pi, workspace.data_ptr(), workspace.numel(),
                         _stream(stream))
    if st != KVP_OK:
        raise KvpError(st, "kvp_select")


def kvp_select_policy(shape, policy, s1, s2, idx, stream=None):
    """Kept positions under `policy` (a KvpPolicy, or a dict of make_policy's arguments):
    sinks, then the best candidates by the policy's key, then the window; ascending."""
    sh = _as_shape(shape)
    pol = policy if isinstance(policy, KvpPolicy) else make_policy(**policy)
    b, hkv, L, B = sh.batch, sh.hkv, sh.seq_len, sh.budget
    p1 = _ptr(s1, "s1", torch.float32, (b, hkv, L), optional=pol.mode == RANK_S2)
    p2 = _ptr(s2, "s2", torch.float32, (b, hkv, L), optional=pol.mode == RANK_S1)
    pi = _ptr(idx, "idx", torch.int32, (b, hkv, B))
    st = _lib.kvp_select_policy(ctypes.byref(sh), ctypes.byref(pol), p1, p2, pi, _stream(stream))
    if st != KVP_OK:
        raise KvpError(st, "kvp_select_policy")


def kvp_leverage(shape, k, v, g, score, workspace=None, stream=None):
    """CurDKV leverage scores of every position: squared row norms of K G and V G, their
    product, normalised per KV head. g: [d, r] bf16 CUDA tensor, 1 <= r <= 32."""
    sh = _as_shape(shape)
    b, hkv, d, L = sh.batch, sh.hkv, sh.head_dim, sh.seq_len
    if not isinstance(g, torch.Tensor) or g.dim() != 2 or g.shape[0] != d:
        raise ValueError(f"g must be a [{d}, r] tensor")
    args = (_ptr(k, "k", torch.bfloat16, (b, hkv, L, d)),
            _ptr(v, "v", torch.bfloat16, (b, hkv, L, d)),
            _ptr(g, "g", torch.bfloat16, tuple(g.shape)))
    ps = _ptr(score, "score", torch.float32, (b, hkv, L))
    if workspace is None:
        workspace = workspace_for(sh, k.device)
    st = _lib.kvp_leverage(ctypes.byref(sh), *args, int(g.shape[1]), ps, workspace.data_ptr(),
                           workspace.numel(), _stream(stream))
    if st != KVP_OK:
        raise KvpError(st, "kvp_leverage")


def adaptive_workspace_for(shape, device=None) -> torch.Tensor:
    n = int(_lib.kvp_adaptive_workspace_bytes(ctypes.byref(_as_shape(shape))))
    if n == 0:
        raise KvpError(2, "kvp_adaptive_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def kvp_select_adaptive(shape, alpha, score, idx, counts, workspace=None, stream=None):
    """Adaptive per-head budgets (AdaKV with safeguard alpha): idx [b, hkv * B] packed
    head after head, counts [b, hkv]."""
    sh = _as_shape(shape)
    b, hkv, L, B = sh.batch, sh.hkv, sh.seq_len, sh.budget
    ps = _ptr(score, "score", torch.float32, (b, hkv, L))
    pi = _ptr(idx, "idx", torch.int32, (b, hkv * B))
    pc = _ptr(counts, "counts", torch.int32, (b, hkv))
    if workspace is None:
        workspace = adaptive_workspace_for(sh, score.device)
    st = _lib.kvp_select_adaptive(ctypes.byref(sh), float(alpha), ps, pi, pc, workspace.data_ptr(),
                                  workspace.numel(), _stream(stream))
    if st != KVP_OK:
        raise KvpError(st, "kvp_select_adaptive")


def kvp_compact_ragged(shape, k, v, idx, counts, k_out, v_out, stream=None):
    sh = _as_shape(shape)
    b, hkv, d, L, B = sh.batch, sh.hkv, sh.head_dim, sh.seq_len, sh.budget
    args = (_ptr(k, "k", torch.bfloat16, (b, hkv, L, d)),
            _ptr(v, "v", torch.bfloat16, (b, hkv, L, d)),
            _ptr(idx, "idx", torch.int32, (b, hkv * B)),
            _ptr(counts, "counts", torch.int32, (b, hkv)),
            _ptr(k_out, "k_out", torch.bfloat16, (b, hkv * B, d)),
            _ptr(v_out, "v_out", torch.bfloat16, (b, hkv * B, d)))
    st = _lib.kvp_compact_ragged(ctypes.byref(sh), *args, _stream(stream))
    if st != KVP_OK:
        raise KvpError(st, "kvp_compact_ragged")


def kvp_compact(shape, k, v, idx, k_out, v_out, stream=None):
    sh = _as_shape(shape)
    b, hkv, d, L, B = sh.batch, sh.hkv, sh.head_dim, sh.seq_len, sh.budget
    args = (_ptr(k, "k", torch.bfloat16, (b, hkv, L, d)),
            _ptr(v, "v", torch.bfloat16, (b, hkv, L, d)),
            _ptr(idx, "idx", torch.int32, (b, hkv, B)),
            _ptr(k_out, "k_out", torch.bfloat16, (b, hkv, B, d)),
            _ptr(v_out, "v_out", torch.bfloat16, (b, hkv, B, d)))
    st = _lib.kvp_compact(ctypes.byref(sh), *args, _stream(stream))
    if st != KVP_OK:
        raise KvpError(st, "kvp_compact")


class LayerBuffers:
    """Device outputs and workspace of one layer's eviction, reusable across calls."""

    def __init__(self, shape, device="cuda", want_s1_s2=False):
        sh = _as_shape(shape)
        self.shape = sh
        b, hkv, d, L, B = sh.batch, sh.hkv, sh.head_dim, sh.seq_len, sh.budget
        self.score = torch.empty((b, hkv, L), dtype=torch.float32, device=device)
        self.s1 = torch.empty_like(self.score) if want_s1_s2 else None
        self.s2 = torch.empty_like(self.score) if want_s1_s2 else None
        self.idx = torch.empty((b, hkv, B), dtype=torch.int32, device=device)
        self.k_out = torch.empty((b, hkv, B, d), dtype=torch.bfloat16, device=device)
        self.v_out = torch.empty_like(self.k_out)
        self.workspace = workspace_for(sh, device)


def evict_layer(q_win, k, v, window: int, budget: int, buffers: LayerBuffers | None = None,
                stream=None):
    """Score, select and compact one layer; returns the LayerBuffers holding the results.

    q_win [b, hq, w, d], k and v [b, hkv, L, d]: bf16 CUDA tensors.
    """
    b, hq, w, d = q_win.shape
    _, hkv, L, _ = k.shape
    if w != window:
        raise ValueError("q_win must hold exactly `window` queries per head")
    sh = make_shape(b, hq, hkv, d, L, window, budget)
    if buffers is None:
        buffers = LayerBuffers(sh, k.device)
    kvp_score(sh, q_win, k, v, buffers.score, buffers.s1, buffers.s2, buffers.workspace, stream)
    kvp_select(sh, buffers.score, buffers.idx, buffers.workspace, stream)
    kvp_compact(sh, k, v, buffers.idx, buffers.k_out, buffers.v_out, stream)
    return buffers
