"""Parity of the adaptive per-head budgets (kvp_select_adaptive) and the ragged compaction
(kvp_compact_ragged) with the CPU oracle.

AdaKV's shared budget with a safeguard floor alpha, as the CurDKV rebuttal page describes
it ("On the sensitivity of the safeguard parameter (alpha)", Tables 5-6; alpha = 0.20 is
AdaKV's default). Given the same fp32 scores both sides rank identically, so the kept
positions and the per-head counts must match exactly; the gathered rows bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_utils import to_bits, to_dev

pytestmark = pytest.mark.gpu


def kvp():
    import token_eviction_b200 as m
    return m


def gpu_adaptive(score, w, B, alpha, d=128):
    m = kvp()
    b, hkv, L = score.shape
    sh = m.make_shape(b, hkv, hkv, d, L, w, B)
    idx = torch.full((b, hkv * B), -1, dtype=torch.int32, device="cuda")
    counts = torch.full((b, hkv), -1, dtype=torch.int32, device="cuda")
    m.kvp_select_adaptive(sh, alpha, torch.from_numpy(np.ascontiguousarray(score, np.float32)).cuda(),
                          idx, counts)
    torch.cuda.synchronize()
    return sh, idx, counts


def structured_scores(b, hkv, L, seed):
    rng = np.random.default_rng(seed)
    s = (rng.random((b, hkv, L)) ** 3 * rng.uniform(0.2, 5.0, (b, hkv, 1))).astype(np.float32)
    s[:, :, 5:60] = np.round(s[:, :, 5:60], 1)            # ties within and across heads
    s[:, -1, :] = np.float32(0.5)                          # one head of equal scores
    return s


@pytest.mark.parametrize("b,hkv,L,w,B", [(2, 3, 300, 8, 60), (1, 8, 5000, 32, 600),
                                         (3, 5, 129, 1, 20), (1, 8, 50000, 16, 3000)])
@pytest.mark.parametrize("alpha", [0.0, 0.2, 0.5, 1.0])
def test_adaptive_exact_on_shared_fp32(b, hkv, L, w, B, alpha):
    s = structured_scores(b, hkv, L, seed=L + B)
    _, idx, counts = gpu_adaptive(s, w, B, alpha)
    want_idx, want_counts = oracle.oracle_select_adaptive(s, w, B, alpha)
    np.testing.assert_array_equal(counts.cpu().numpy(), want_counts)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)


@pytest.mark.parametrize("budget", [256, 2048])
def test_adaptive_on_the_32k_layer(budget):
    """The 32K layer's GPU scores (kvp_score) with AdaKV's alpha = 0.20: exact against the
    oracle on the same fp32 scores, then the ragged compaction against numpy indexing."""
    m = kvp()
    wl = synth.WORKLOADS["llama8b_32k"]
    inp = synth.make_inputs(wl)
    q, k, v = to_dev(inp.q_win), to_dev(inp.k), to_dev(inp.v)
    b, hkv, L, d = wl.batch, wl.hkv, wl.seq_len, wl.head_dim
    sh = m.make_shape(b, wl.hq, hkv, d, L, wl.window, budget)
    score = torch.empty((b, hkv, L), dtype=torch.float32, device="cuda")
    m.kvp_score(sh, q, k, v, score)
    idx = torch.empty((b, hkv * budget), dtype=torch.int32, device="cuda")
    counts = torch.empty((b, hkv), dtype=torch.int32, device="cuda")
    m.kvp_select_adaptive(sh, 0.2, score, idx, counts)
    k_out = torch.empty((b, hkv * budget, d), dtype=torch.bfloat16, device="cuda")
    v_out = torch.empty_like(k_out)
    m.kvp_compact_ragged(sh, k, v, idx, counts, k_out, v_out)
    torch.cuda.synchronize()
    want_idx, want_counts = oracle.oracle_select_adaptive(score.cpu().numpy(), wl.window, budget, 0.2)
    gi, gc = idx.cpu().numpy(), counts.cpu().numpy()
    np.testing.assert_array_equal(gc, want_counts)
    np.testing.assert_array_equal(gi, want_idx)
    assert (gc.sum(1) == hkv * budget).all()
    heads = np.repeat(np.arange(hkv), gc[0])
    np.testing.assert_array_equal(to_bits(k_out)[0], inp.k[0, heads, gi[0]])
    np.testing.assert_array_equal(to_bits(v_out)[0], inp.v[0, heads, gi[0]])


def test_ragged_compaction_bit_exact_with_uneven_counts():
    m = kvp()
    rng = np.random.default_rng(9)
    b, hkv, L, d, B = 2, 4, 700, 64, 90
    k = rng.integers(0, 1 << 16, (b, hkv, L, d), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, (b, hkv, L, d), dtype=np.uint16)
    counts = np.array([[30, 150, 0, 180], [90, 90, 90, 90]], dtype=np.int32)
    idx = np.empty((b, hkv * B), dtype=np.int32)
    for bi in range(b):
        o = 0
        for h in range(hkv):
            c = counts[bi, h]
            idx[bi, o:o + c] = np.sort(rng.choice(L, c, replace=False))
            o += c
    idx[1, 5] = L + 3                                      # out of range: a zero row
    sh = m.make_shape(b, hkv, hkv, d, L, 16, B)
    k_out = torch.empty((b, hkv * B, d), dtype=torch.bfloat16, device="cuda")
    v_out = torch.empty_like(k_out)
    m.kvp_compact_ragged(sh, to_dev(k), to_dev(v), torch.from_numpy(idx).cuda(),
                         torch.from_numpy(counts).cuda(), k_out, v_out)
    torch.cuda.synchronize()
    for bi in range(b):
        heads = np.repeat(np.arange(hkv), counts[bi])
        j = np.clip(idx[bi], 0, L - 1)
        ek, ev = k[bi, heads, j].copy(), v[bi, heads, j].copy()
        bad = idx[bi] >= L
        ek[bad] = 0
        ev[bad] = 0
        np.testing.assert_array_equal(to_bits(k_out)[bi], ek)
        np.testing.assert_array_equal(to_bits(v_out)[bi], ev)
