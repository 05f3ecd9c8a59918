"""Seeded synthetic inputs for the prefill KV-cache eviction workloads.

This module draws random tensors with the shapes and value structure of the workloads
the eviction path is measured on (Llama-3.1-8B-shaped layers at 32K and 128K context,
a batched GQA-7 layer, and a tiny case), and nothing else: it holds none of the
eviction method's arithmetic. Both the CUDA path's tests and the CPU oracle take its
output as plain input data, so it is the one piece of code the two sides share.

The random numbers come from ``synth.c`` (a counter-based splitmix64 hash and a
Box-Muller normal, rounded to bf16 round-to-nearest-even). Every tensor is a function
of (seed, stream id, flat index) only, so any slice can be regenerated independently.

Structure recipes (all bf16, all ~N(0,1) before structure is applied):

* ``tiny``: b1, 4 query / 2 KV heads, d64, L512, w16, B128; 2 V channels per KV head
  scaled x20.
* ``llama8b_32k``: b1, 32/8 heads, d128, L32768, w32, B2048; 4 of 128 channels per KV
  head scaled x20 in both K and V; K then rotated RoPE-style (rotate-half pairs,
  base 500000, angle = position x base^(-2c/d)). Q is plain N(0,1).
* ``llama8b_32k_x32``: the same layer shape, 32 layers with independent seeds, B128.
* ``long_128k_b70`` / ``long_128k_b10``: b1, 32/8 heads, d128, L131072, w32,
  B = floor(0.7 L) / floor(0.1 L); 4 outlier K/V channels x20, no rotation; 16 planted
  needle keys per KV head at seeded positions j < L-w, each k_j = a sqrt(d) q / |q|^2
  for a seeded window query q of that head's group, so its logit for q is a, with
  a = max(24, 7 sigma_q). sigma_q = sqrt(sum_c q_c^2 s_c^2 / d) is the standard
  deviation of q's logit against an ordinary key (channel scales s_c), so the needle
  tops q's softmax row even when q leans on the x20 outlier channels.
* ``gqa7_batched``: b8, 28/4 heads, d128, L16384, w64, B1024; a seed per sequence;
  4 outlier channels x20 in V only.

Seeds: workload number c (1..5), layer l, sequence s -> seed = 1000 c + 100 s + l.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

# stream ids (part of the generator's key)
STREAM_Q, STREAM_K, STREAM_V, STREAM_OUTLIER, STREAM_NEEDLE = 1, 2, 3, 4, 5


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``libsynth.so`` beside it (gcc, OpenMP)."""
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
        lib.synth_normal_bf16.argtypes = [
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64, ctypes.c_uint64,
            ctypes.c_int64, ctypes.c_void_p, ctypes.c_double]
        lib.synth_normal_bf16.restype = None
        lib.synth_draw_u64.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                       ctypes.c_int64, ctypes.c_void_p]
        lib.synth_draw_u64.restype = None
        lib.synth_round_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        lib.synth_round_bf16.restype = None
        _lib = lib
    return _lib


def draw_u64(seed: int, stream: int, first: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _get().synth_draw_u64(seed, stream, first, n, out.ctypes.data)
    return out


def normal_bf16(rows: int, d: int, seed: int, stream: int, rows_per_head: int | None = None,
                scale: np.ndarray | None = None, rope_base: float = 0.0) -> np.ndarray:
    """bf16 bits [rows, d] of seeded N(0,1), optional per-head channel scale and rotation."""
    out = np.empty((rows, d), dtype=np.uint16)
    rph = rows if rows_per_head is None else rows_per_head
    sc = None
    if scale is not None:
        scale = np.ascontiguousarray(scale, dtype=np.float32)
        assert scale.size == (rows // rph) * d
        sc = scale.ctypes.data
    _get().synth_normal_bf16(out.ctypes.data, rows, d, seed, stream, rph, sc, float(rope_base))
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _get().synth_round_bf16(x.ctypes.data, x.size, out.ctypes.data)
    return out


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _pick_distinct(seed: int, stream: int, first: int, count: int, upper: int) -> list[int]:
    """`count` distinct integers in [0, upper), drawn in order from the hash stream."""
    out: list[int] = []
    e = first
    while len(out) < count:
        v = int(draw_u64(seed, stream, e, 1)[0] % np.uint64(upper))
        e += 1
        if v not in out:
            out.append(v)
    return out


@dataclass(frozen=True)
class Workload:
    name: str
    number: int            # workload number used in the seed (1..5)
    batch: int
    hq: int
    hkv: int
    head_dim: int
    seq_len: int
    window: int
    budget: int
    layers: int = 1
    k_outliers: int = 0    # outlier channels per KV head in K
    v_outliers: int = 0    # outlier channels per KV head in V
    outlier_scale: float = 20.0
    rope_base: float = 0.0
    needles: int = 0       # planted needle keys per KV head
    needle_logit: float = 24.0   # floor of a needle's logit for its query
    needle_sigmas: float = 7.0   # ... and at least this many sigma_q

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    def shape_tuple(self):
        return (self.batch, self.hq, self.hkv, self.head_dim, self.seq_len, self.window, self.budget)

    def bytes_per_layer(self) -> dict:
        """Algorithmic HBM bytes of one layer's score + select + compact."""
        b, hq, hkv, d, L, w, B = self.shape_tuple()
        kv = 2 * b * hkv * L * d * 2
        q = b * hq * w * d * 2
        s = b * hkv * L * 4
        idx = b * hkv * B * 4
        comp = 2 * 2 * b * hkv * B * d * 2  # read + write of kept K and V rows
        return {"score": kv + q + s, "select": s + idx, "compact": comp + idx,
                "total": kv + q + s + s + idx + idx + comp}


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 4, 2, 64, 512, 16, 128, v_outliers=2),
    "llama8b_32k": Workload("llama8b_32k", 2, 1, 32, 8, 128, 32768, 32, 2048,
                            k_outliers=4, v_outliers=4, rope_base=500000.0),
    "llama8b_32k_x32": Workload("llama8b_32k_x32", 3, 1, 32, 8, 128, 32768, 32, 128, layers=32,
                                k_outliers=4, v_outliers=4, rope_base=500000.0),
    "long_128k_b70": Workload("long_128k_b70", 4, 1, 32, 8, 128, 131072, 32, int(0.7 * 131072),
                              k_outliers=4, v_outliers=4, needles=16),
    "long_128k_b10": Workload("long_128k_b10", 4, 1, 32, 8, 128, 131072, 32, int(0.1 * 131072),
                              k_outliers=4, v_outliers=4, needles=16),
    "gqa7_batched": Workload("gqa7_batched", 5, 8, 28, 4, 128, 16384, 64, 1024, v_outliers=4),
}


def seed_of(wl: Workload, layer: int = 0, seq: int = 0) -> int:
    return 1000 * wl.number + 100 * seq + layer


@dataclass
class Inputs:
    """One layer's inputs as bf16 bit patterns (uint16), row-major, d innermost."""
    workload: Workload
    layer: int
    q_win: np.ndarray      # [b, hq, w, d]
    k: np.ndarray          # [b, hkv, L, d]
    v: np.ndarray          # [b, hkv, L, d]
    needle_pos: np.ndarray = field(default_factory=lambda: np.zeros((0, 0, 0), np.int64))  # [b, hkv, n]
    k_outlier_channels: np.ndarray | None = None  # [b, hkv, n]
    v_outlier_channels: np.ndarray | None = None


def _channel_scale(wl: Workload, seed: int, stream_first: int, count: int):
    hkv, d = wl.hkv, wl.head_dim
    scale = np.ones((hkv, d), dtype=np.float32)
    chans = np.zeros((hkv, count), dtype=np.int64)
    for h in range(hkv):
        c = _pick_distinct(seed, STREAM_OUTLIER, stream_first + 4096 * h, count, d)
        chans[h] = c
        scale[h, c] = wl.outlier_scale
    return scale, chans


def make_sequence(wl: Workload, layer: int = 0, seq: int = 0):
    """Tensors of one sequence (batch index `seq`): q_win [hq,w,d], k, v [hkv,L,d]."""
    seed = seed_of(wl, layer, seq)
    hq, hkv, d, L, w = wl.hq, wl.hkv, wl.head_dim, wl.seq_len, wl.window
    q = normal_bf16(hq * w, d, seed, STREAM_Q).reshape(hq, w, d)
    kscale = vscale = None
    kch = vch = None
    if wl.k_outliers:
        kscale, kch = _channel_scale(wl, seed, 0, wl.k_outliers)
    if wl.v_outliers:
        vscale, vch = _channel_scale(wl, seed, 1 << 20, wl.v_outliers)
    k = normal_bf16(hkv * L, d, seed, STREAM_K, rows_per_head=L, scale=kscale,
                    rope_base=wl.rope_base).reshape(hkv, L, d)
    v = normal_bf16(hkv * L, d, seed, STREAM_V, rows_per_head=L, scale=vscale).reshape(hkv, L, d)
    needle_pos = np.zeros((hkv, wl.needles), dtype=np.int64)
    if wl.needles:
        G = wl.group
        qf = bf16_to_f64(q)
        ks = np.ones((hkv, d)) if kscale is None else kscale.astype(np.float64)
        for h in range(hkv):
            pos = _pick_distinct(seed, STREAM_NEEDLE, 4096 * h, wl.needles, L - w)
            needle_pos[h] = sorted(pos)
            for t, j in enumerate(pos):
                r = int(draw_u64(seed, STREAM_NEEDLE, (1 << 24) + 64 * h + t, 1)[0] % np.uint64(G * w))
                g, i = divmod(r, w)
                qv = qf[h * G + g, i]
                sigma_q = math.sqrt(float(np.sum((qv * ks[h]) ** 2)) / d)
                a = max(wl.needle_logit, wl.needle_sigmas * sigma_q)
                k[h, j] = round_bf16(a * math.sqrt(d) * qv / float(qv @ qv))
    return q, k, v, needle_pos, kch, vch


def make_inputs(wl: Workload | str, layer: int = 0) -> Inputs:
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    parts = [make_sequence(wl, layer, s) for s in range(wl.batch)]
    if wl.batch == 1:
        q, k, v, npos, kch, vch = parts[0]
        return Inputs(wl, layer, q[None], k[None], v[None], npos[None],
                      None if kch is None else kch[None], None if vch is None else vch[None])
    stack = lambda i: np.stack([p[i] for p in parts])
    return Inputs(wl, layer, stack(0), stack(1), stack(2), stack(3),
                  None if parts[0][4] is None else stack(4), None if parts[0][5] is None else stack(5))


def small(name: str, **overrides) -> Workload:
    """A scaled-down copy of a workload (same structure, smaller sizes) for quick checks."""
    return replace(WORKLOADS[name], **overrides)
