"""Parity of the CurDKV leverage scores (kvp_leverage) with the CPU oracle.

CurDKV rebuttal page, "A clearer description of Algorithm 1", steps 1-6: project K and V
with a Gaussian G (d x r, r = 20 on the page), take squared row norms, combine them by
product, normalise per KV head, keep the first s positions (sinks) and the top scores.

Tolerance, from the arithmetic: each projected value K_j . G_c is an fp32 sum of d exact
bf16 products, so its error is at most about d * 2^-24 * sum_t |k_t g_t|: small against
the typical |K_j . G_c| (~ sqrt(d) sigma_k sigma_g) but not against a value that cancels to
near zero. A score is a product of two sums of r such squares, so where it is at least
1e-6 of its head's largest (no sum of squares can have cancelled that far) the bound is
1e-3 relative; below that floor the GPU value must be within 1e-9 of the head's largest.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_utils import REL, to_dev

pytestmark = pytest.mark.gpu


def kvp():
    import token_eviction_b200 as m
    return m


LEV_FLOOR = 1e-6
LEV_ABS = 1e-9


def check_scores(gpu, ora, what):
    gpu = gpu.astype(np.float64)
    mx = ora.max(-1, keepdims=True)
    big = ora >= LEV_FLOOR * mx
    err = np.abs(gpu - ora)
    bad = (big & (err > REL * ora)) | (~big & (err > LEV_ABS * np.broadcast_to(mx, gpu.shape)))
    if bad.any():
        pos = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} values outside the bound; first "
                             f"{[(tuple(p), gpu[tuple(p)], ora[tuple(p)]) for p in pos]}")
    assert np.isfinite(gpu).all(), f"{what}: non-finite values"


def lev_inputs(b, hkv, L, d, r, seed):
    k = synth.normal_bf16(b * hkv * L, d, seed, 1).reshape(b, hkv, L, d)
    v = synth.normal_bf16(b * hkv * L, d, seed, 2).reshape(b, hkv, L, d)
    g = synth.normal_bf16(d, r, seed, 3)
    return k, v, g


def gpu_leverage(k, v, g, w=16, B=None):
    m = kvp()
    b, hkv, L, d = k.shape
    B = B or max(w, L // 4)
    sh = m.make_shape(b, hkv, hkv, d, L, w, B)
    score = torch.full((b, hkv, L), -1.0, dtype=torch.float32, device="cuda")
    ws = m.workspace_for(sh)
    m.kvp_leverage(sh, to_dev(k), to_dev(v), to_dev(g), score, ws)
    assert m.kvp_workspace_status(ws) == 0
    torch.cuda.synchronize()
    return sh, score


@pytest.mark.parametrize("b,hkv,L,d,r", [
    (1, 1, 128, 128, 20),        # one tile
    (1, 2, 1000, 128, 20),       # ragged tail, two heads
    (2, 3, 777, 64, 20),         # d = 64, heads crossing CTA runs
    (1, 4, 5000, 128, 1),        # rank-one projection
    (1, 2, 3000, 128, 32),       # the largest r
    (3, 5, 70, 64, 7),           # shorter than a tile, many heads
])
def test_leverage_small(b, hkv, L, d, r):
    k, v, g = lev_inputs(b, hkv, L, d, r, seed=L + r)
    _, score = gpu_leverage(k, v, g)
    got = score.cpu().numpy()
    ora = oracle.oracle_leverage(k, v, g)
    check_scores(got, ora, "leverage")
    np.testing.assert_allclose(got.astype(np.float64).sum(-1), 1.0, rtol=1e-4)


def test_leverage_32k_layer_and_curdkv_selection():
    """The 32K layer's K and V with r = 20: scores against the oracle, then CurDKV's
    selection (sinks kept, the top scores) against the oracle's, up to near ties."""
    m = kvp()
    wl = synth.WORKLOADS["llama8b_32k"]
    inp = synth.make_inputs(wl)
    g = synth.normal_bf16(wl.head_dim, 20, 99, 3)
    sh, score = gpu_leverage(inp.k, inp.v, g, w=wl.window, B=wl.budget)
    got = score.cpu().numpy()
    ora = oracle.oracle_leverage(inp.k, inp.v, g)
    check_scores(got, ora, "leverage")
    sinks = 4
    idx = torch.empty((wl.batch, wl.hkv, wl.budget), dtype=torch.int32, device="cuda")
    m.kvp_select_policy(sh, m.make_policy(sinks, 1, m.RANK_S1), score, None, idx)
    torch.cuda.synchronize()
    gi = idx.cpu().numpy()
    # exact against the oracle's selection on the same fp32 scores
    ones = np.ones_like(got)
    want = oracle.oracle_select_policy(got, ones, wl.window, wl.budget, sinks, 1, oracle.MODE_S1,
                                       fp32_key=True)
    np.testing.assert_array_equal(gi, want)
    # and up to near ties against the float64 scores
    ora_idx = oracle.oracle_select_policy(ora, np.ones_like(ora), wl.window, wl.budget, sinks, 1,
                                          oracle.MODE_S1)
    L, w, B = wl.seq_len, wl.window, wl.budget
    for r_ in range(gi.shape[1]):
        diff = np.setxor1d(gi[0, r_], ora_idx[0, r_])
        if diff.size:
            thr = np.sort(ora[0, r_, sinks:L - w])[::-1][B - w - sinks - 1]
            assert np.all(np.abs(ora[0, r_, diff] - thr) <= REL * thr)


def test_leverage_repeat_calls_agree_bit_for_bit():
    k, v, g = lev_inputs(1, 3, 4000, 128, 20, seed=5)
    _, a = gpu_leverage(k, v, g)
    _, b = gpu_leverage(k, v, g)
    assert torch.equal(a, b)


def test_leverage_zero_head_scores_zero():
    """A KV head whose keys are all zero has every product 0: its scores are 0, not NaN."""
    k, v, g = lev_inputs(1, 2, 600, 64, 20, seed=6)
    k[0, 1] = 0
    _, score = gpu_leverage(k, v, g)
    got = score.cpu().numpy()
    assert (got[0, 1] == 0).all()
    check_scores(got[:, :1], oracle.oracle_leverage(k, v, g)[:, :1], "leverage")
