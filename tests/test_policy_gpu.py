"""Parity of the policy selection (kvp_select_policy) with the oracle's policy selection.

Policies: attention sinks kept first (CurDKV rebuttal page, "how our method processes the
KV cache", step 5), ranking by S1 alone or S2 alone (the SlimKV page's review of the
Section 4.6 ablation), S1 max-pooled with a "kernel size" (same review; read as SnapKV-style
1-D max pooling), and the 256-token budget of the SlimKV page's Table 1.

Given the same fp32 S1 and S2, both sides form the key in fp32 and the kept sets must be
identical (oracle_select_policy with fp32_key=True). Against the float64 oracle end to end,
kept sets may differ only at near ties of the oracle's key.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_utils import REL, check_idx_valid, to_dev

pytestmark = pytest.mark.gpu


def kvp():
    import token_eviction_b200 as m
    return m


def gpu_policy(s1, s2, w, B, sinks=0, kernel=1, mode=0):
    """s1, s2: float32 [R, L] (or [b, hkv, L]); returns idx [.., B] from the CUDA path."""
    m = kvp()
    s1 = np.ascontiguousarray(s1, dtype=np.float32)
    s2 = np.ascontiguousarray(s2, dtype=np.float32)
    if s1.ndim == 2:
        s1, s2 = s1[None], s2[None]
    b, h, L = s1.shape
    sh = m.make_shape(b, h, h, 128, L, w, B)
    idx = torch.full((b, h, B), -1, dtype=torch.int32, device="cuda")
    m.kvp_select_policy(sh, m.make_policy(sinks, kernel, mode), torch.from_numpy(s1).cuda(),
                        torch.from_numpy(s2).cuda(), idx)
    torch.cuda.synchronize()
    return idx.cpu().numpy()


def check_policy_valid(idx, L, w, B, sinks):
    check_idx_valid(idx, L, w, B)
    rows = idx.reshape(-1, B)
    assert (rows[:, :sinks] == np.arange(sinks)).all(), "sinks not kept"


def check_policy_near_ties(gpu_idx, ora_idx, ora_key, w, B, sinks):
    """Kept sets equal except positions whose oracle key is within REL of the threshold
    key (the (B - w - s)-th largest candidate key)."""
    L = ora_key.shape[-1]
    g, o = gpu_idx.reshape(-1, B), ora_idx.reshape(-1, B)
    key = ora_key.reshape(-1, L)
    kk = B - w - sinks
    for r in range(g.shape[0]):
        diff = np.setxor1d(g[r], o[r])
        if diff.size == 0:
            continue
        cand = np.sort(key[r, sinks:L - w])[::-1]
        thr = cand[kk - 1]
        assert np.all(np.abs(key[r, diff] - thr) <= REL * thr), \
            f"row {r}: kept sets differ away from the threshold ({diff[:8]})"


def rows_with_structure(L, seed):
    """S1-like and S2-like fp32 rows: smooth positive values, a block of exact ties, zeros
    and subnormals, a planted spike, all-equal values."""
    rng = np.random.default_rng(seed)
    s1 = (rng.random((5, L)) ** 4 * 1e-2).astype(np.float32)
    s2 = (rng.random((5, L)) * 4 + 0.5).astype(np.float32)
    s1[1, : L // 3] = np.float32(2e-4)                      # exact ties
    s2[1, : L // 3] = np.float32(1.5)
    s1[2, ::5] = 0.0
    s1[2, 1::9] = np.float32(1e-40)                         # subnormal S1
    s2[2, 2::11] = np.float32(1e-39)                        # subnormal S2
    s1[3, L // 2] = np.float32(1.0)                         # a planted spike
    s1[4] = np.float32(3e-3)                                # every value equal
    s2[4] = np.float32(2.0)
    return s1, s2


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("kernel", [1, 7, 31])
@pytest.mark.parametrize("sinks", [0, 4])
def test_policy_exact_on_shared_fp32(mode, kernel, sinks):
    L, w, B = 3000, 24, 300
    s1, s2 = rows_with_structure(L, seed=kernel * 10 + mode)
    got = gpu_policy(s1, s2, w, B, sinks, kernel, mode)
    want = oracle.oracle_select_policy(s1, s2, w, B, sinks, kernel, mode, fp32_key=True)
    np.testing.assert_array_equal(got[0], want)
    check_policy_valid(got, L, w, B, sinks)


@pytest.mark.parametrize("L,w,B,sinks,kernel", [
    (70, 3, 9, 2, 5),            # tiny, ragged
    (64, 16, 20, 4, 3),          # no candidates left to choose from: B = w + sinks
    (64, 16, 64, 4, 3),          # B = L: everything kept
    (100, 10, 100, 90, 1),       # sinks = L - w
    (350000, 16, 1000, 3, 5),    # candidates beyond the shared-memory slices
    (131072, 32, 91750, 4, 7),   # B = 0.7 L
])
def test_policy_edges(L, w, B, sinks, kernel):
    s1, s2 = rows_with_structure(L, seed=L)
    for mode in (0, 1, 2):
        got = gpu_policy(s1[:3], s2[:3], w, B, sinks, kernel, mode)
        want = oracle.oracle_select_policy(s1[:3], s2[:3], w, B, sinks, kernel, mode, fp32_key=True)
        np.testing.assert_array_equal(got[0], want)
        check_policy_valid(got, L, w, B, sinks)


def test_policy_plain_equals_kvp_select():
    """sinks 0, kernel 1, product mode ranks by S1 * S2 = S: the same kept set as kvp_select
    on the score that kvp_score writes."""
    m = kvp()
    wl = synth.small("llama8b_32k", hq=8, hkv=2, seq_len=5000, window=32, budget=400)
    inp = synth.make_inputs(wl)
    q, k, v = to_dev(inp.q_win), to_dev(inp.k), to_dev(inp.v)
    sh = m.make_shape(*wl.shape_tuple())
    b, h, L, B = wl.batch, wl.hkv, wl.seq_len, wl.budget
    score = torch.empty((b, h, L), dtype=torch.float32, device="cuda")
    s1, s2 = torch.empty_like(score), torch.empty_like(score)
    m.kvp_score(sh, q, k, v, score, s1, s2)
    idx_plain = torch.empty((b, h, B), dtype=torch.int32, device="cuda")
    idx_pol = torch.empty_like(idx_plain)
    m.kvp_select(sh, score, idx_plain)
    m.kvp_select_policy(sh, m.make_policy(), s1, s2, idx_pol)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx_pol.cpu().numpy(), idx_plain.cpu().numpy())


@pytest.mark.parametrize("budget", [256, 2048])
def test_policies_on_the_32k_layer(budget):
    """The 32K layer's GPU S1 and S2 (kvp_score), every mode with sinks and pooling, at the
    SlimKV page's budgets 256 and 2048: exact against the oracle on the same fp32 inputs."""
    m = kvp()
    wl = synth.WORKLOADS["llama8b_32k"]
    inp = synth.make_inputs(wl)
    q, k, v = to_dev(inp.q_win), to_dev(inp.k), to_dev(inp.v)
    sh = m.make_shape(wl.batch, wl.hq, wl.hkv, wl.head_dim, wl.seq_len, wl.window, budget)
    b, h, L = wl.batch, wl.hkv, wl.seq_len
    score = torch.empty((b, h, L), dtype=torch.float32, device="cuda")
    s1, s2 = torch.empty_like(score), torch.empty_like(score)
    m.kvp_score(sh, q, k, v, score, s1, s2)
    torch.cuda.synchronize()
    s1h, s2h = s1.cpu().numpy(), s2.cpu().numpy()
    for sinks, kernel, mode in [(4, 7, 0), (4, 1, 1), (0, 1, 2), (16, 13, 1)]:
        idx = torch.empty((b, h, budget), dtype=torch.int32, device="cuda")
        m.kvp_select_policy(sh, m.make_policy(sinks, kernel, mode), s1, s2, idx)
        torch.cuda.synchronize()
        got = idx.cpu().numpy()
        want = oracle.oracle_select_policy(s1h, s2h, wl.window, budget, sinks, kernel, mode, fp32_key=True)
        np.testing.assert_array_equal(got, want)
        check_policy_valid(got, L, wl.window, budget, sinks)


def test_policy_end_to_end_against_float64_oracle():
    """kvp_score then kvp_select_policy against the float64 oracle (S1, S2 and the key in
    double): kept sets agree up to near ties of the oracle's key."""
    m = kvp()
    wl = synth.small("llama8b_32k", hq=8, hkv=2, seq_len=6000, window=32, budget=500)
    inp = synth.make_inputs(wl)
    q, k, v = to_dev(inp.q_win), to_dev(inp.k), to_dev(inp.v)
    sh = m.make_shape(*wl.shape_tuple())
    b, h, L, w, B = wl.batch, wl.hkv, wl.seq_len, wl.window, wl.budget
    score = torch.empty((b, h, L), dtype=torch.float32, device="cuda")
    s1, s2 = torch.empty_like(score), torch.empty_like(score)
    m.kvp_score(sh, q, k, v, score, s1, s2)
    ora_s1, ora_s2, _ = oracle.oracle_score(inp.q_win, inp.k, inp.v)
    for sinks, kernel, mode in [(4, 7, 0), (0, 5, 1), (8, 1, 2)]:
        idx = torch.empty((b, h, B), dtype=torch.int32, device="cuda")
        m.kvp_select_policy(sh, m.make_policy(sinks, kernel, mode), s1, s2, idx)
        torch.cuda.synchronize()
        ora_idx, ora_key = oracle.oracle_select_policy(ora_s1, ora_s2, w, B, sinks, kernel, mode,
                                                       want_key=True)
        got = idx.cpu().numpy()
        check_policy_valid(got, L, w, B, sinks)
        check_policy_near_ties(got, ora_idx, ora_key, w, B, sinks)
