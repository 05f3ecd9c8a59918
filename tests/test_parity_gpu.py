"""Parity of the CUDA path (through the C ABI) with the CPU oracle, element by element.

Small shapes span several 128-key tiles with ragged tails; the full-size workloads run
in the same launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_utils import (check_idx_near_ties, check_idx_valid, check_scores, to_bits,
                                to_dev)

pytestmark = pytest.mark.gpu


def kvp():
    import token_eviction_b200 as m
    return m


def run_gpu(inp, budget=None, want_s1_s2=True):
    m = kvp()
    wl = inp.workload
    B = wl.budget if budget is None else budget
    q, k, v = to_dev(inp.q_win), to_dev(inp.k), to_dev(inp.v)
    sh = m.make_shape(wl.batch, wl.hq, wl.hkv, wl.head_dim, wl.seq_len, wl.window, B)
    buf = m.LayerBuffers(sh, "cuda", want_s1_s2=want_s1_s2)
    m.evict_layer(q, k, v, wl.window, B, buffers=buf)
    torch.cuda.synchronize()
    out = {"score": buf.score.cpu().numpy(), "idx": buf.idx.cpu().numpy(),
           "k_out": to_bits(buf.k_out), "v_out": to_bits(buf.v_out)}
    if want_s1_s2:
        out["s1"] = buf.s1.cpu().numpy()
        out["s2"] = buf.s2.cpu().numpy()
    return out


def check_layer(inp, gpu, ora_s1, ora_s2, ora_s, budget=None):
    wl = inp.workload
    B = wl.budget if budget is None else budget
    w, L, G = wl.window, wl.seq_len, wl.group
    if "s2" in gpu:
        np.testing.assert_array_equal(gpu["s2"].astype(np.float64), ora_s2)
        check_scores(gpu["s1"], ora_s1, "S1")
        np.testing.assert_allclose(gpu["s1"].astype(np.float64).sum(-1), G * w, rtol=1e-4)
    check_scores(gpu["score"], ora_s, "S")
    check_idx_valid(gpu["idx"], L, w, B)
    # the selection, given the GPU's own fp32 scores, is exact
    np.testing.assert_array_equal(gpu["idx"], oracle.oracle_select(gpu["score"], w, B))
    # against the oracle's float64 scores: equal up to near ties
    ora_idx = oracle.oracle_select(ora_s, w, B)
    check_idx_near_ties(gpu["idx"], ora_idx, ora_s, w, B)
    # compaction given the GPU indices: bit-exact
    ko, vo = oracle.oracle_compact(inp.k, inp.v, gpu["idx"])
    np.testing.assert_array_equal(gpu["k_out"], ko)
    np.testing.assert_array_equal(gpu["v_out"], vo)


SMALL = {
    "tiny": synth.WORKLOADS["tiny"],
    "ragged_d128_g4": synth.small("llama8b_32k", hq=8, hkv=2, seq_len=1000, window=32, budget=300),
    "ragged_d64_b2": synth.small("tiny", batch=2, hq=6, hkv=3, seq_len=777, window=16, budget=100),
    "gqa7_small": synth.small("gqa7_batched", batch=2, hq=14, hkv=2, seq_len=1500, window=64, budget=200),
    "single_query": synth.small("tiny", hq=2, hkv=2, seq_len=300, window=1, budget=50),
    "identity": synth.small("tiny", seq_len=200, window=8, budget=200),
    "window_only": synth.small("tiny", seq_len=200, window=8, budget=8),
    "short": synth.small("tiny", seq_len=50, window=10, budget=20),
    "window_is_all": synth.small("tiny", seq_len=16, window=16, budget=16),
    "one_tile_edge": synth.small("llama8b_32k", hq=4, hkv=1, seq_len=129, window=32, budget=64),
    # more than 256 query rows per KV head: accumulators split across two TMEM stages
    "split_ragged_g5": synth.small("llama8b_32k", hq=10, hkv=2, seq_len=900, window=56, budget=150),
    "split_wide_window": synth.small("tiny", hq=2, hkv=2, head_dim=128, seq_len=700, window=300, budget=400),
    # one 256-column accumulator stage per epilogue group (128 < G w <= 256)
    "wide_stage_g8": synth.small("llama8b_32k", hq=8, hkv=1, seq_len=1100, window=32, budget=200),
    "wide_stage_g7": synth.small("llama8b_32k", hq=14, hkv=2, seq_len=777, window=32, budget=150),
    # d = 64 with every tile split across both groups (G w > 256)
    "split_d64": synth.small("tiny", hq=6, hkv=1, seq_len=900, window=48, budget=200),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_parity(name):
    inp = synth.make_inputs(SMALL[name])
    ora = oracle.oracle_score(inp.q_win, inp.k, inp.v)
    gpu = run_gpu(inp)
    check_layer(inp, gpu, *ora)


def test_llama8b_32k_layer():
    inp = synth.make_inputs("llama8b_32k")
    ora = oracle.oracle_score(inp.q_win, inp.k, inp.v)
    gpu = run_gpu(inp)
    check_layer(inp, gpu, *ora)


def test_llama8b_32k_all_layers_tight_budget():
    wl = synth.WORKLOADS["llama8b_32k_x32"]
    for layer in range(wl.layers):
        inp = synth.make_inputs(wl, layer)
        ora = oracle.oracle_score(inp.q_win, inp.k, inp.v)
        gpu = run_gpu(inp, want_s1_s2=False)
        check_layer(inp, gpu, *ora)


def test_long_128k_both_budgets_keep_needles():
    wl70 = synth.WORKLOADS["long_128k_b70"]
    inp = synth.make_inputs(wl70)
    ora = oracle.oracle_score(inp.q_win, inp.k, inp.v)
    for B in (synth.WORKLOADS["long_128k_b70"].budget, synth.WORKLOADS["long_128k_b10"].budget):
        gpu = run_gpu(inp, budget=B)
        check_layer(inp, gpu, *ora, budget=B)
        for h in range(wl70.hkv):
            assert np.isin(inp.needle_pos[0, h], gpu["idx"][0, h]).all(), f"needle lost in head {h}"


def test_gqa7_batched():
    inp = synth.make_inputs("gqa7_batched")
    ora = oracle.oracle_score(inp.q_win, inp.k, inp.v)
    gpu = run_gpu(inp)
    check_layer(inp, gpu, *ora)


@pytest.mark.parametrize("L,w,B", [(131072, 32, 91750), (131072, 32, 13107), (32768, 32, 2048),
                                   (32768, 32, 128), (5000, 7, 4000), (4096, 64, 65), (70, 3, 9),
                                   (350000, 16, 1000)])
def test_select_exact_with_ties(L, w, B):
    """Selection alone, on fp32 scores both sides share: the kept sets must be identical.
    Rows: a large block of exact ties, zeros (and negative zeros), all-equal scores."""
    m = kvp()
    rng = np.random.default_rng(L + B)
    score = rng.random((3, L), dtype=np.float32) * np.float32(1e-3)
    score[0, : L // 2] = np.float32(5e-4)          # a large block of exact ties
    score[1, ::3] = 0.0
    score[1, 1::7] = -0.0
    score[2] = np.float32(1.0)                      # every score equal
    score = score.reshape(1, 3, L)
    sh = m.make_shape(1, 3, 3, 128, L, w, B)
    s_dev = torch.from_numpy(score).cuda()
    idx = torch.empty((1, 3, B), dtype=torch.int32, device="cuda")
    m.kvp_select(sh, s_dev, idx)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx.cpu().numpy(), oracle.oracle_select(score, w, B))


def test_compact_bit_exact_and_out_of_range_rows():
    m = kvp()
    rng = np.random.default_rng(3)
    b, hkv, L, d, B = 2, 3, 700, 128, 90
    k = rng.integers(0, 65536, (b, hkv, L, d), dtype=np.uint16)
    v = rng.integers(0, 65536, (b, hkv, L, d), dtype=np.uint16)
    idx = rng.integers(0, L, (b, hkv, B)).astype(np.int32)
    idx[0, 0, 5] = -1
    idx[1, 2, 7] = L
    sh = m.make_shape(b, hkv, hkv, d, L, 1, B)
    ko = torch.empty((b, hkv, B, d), dtype=torch.bfloat16, device="cuda")
    vo = torch.empty_like(ko)
    m.kvp_compact(sh, to_dev(k), to_dev(v), torch.from_numpy(idx).cuda(), ko, vo)
    torch.cuda.synchronize()
    safe = np.clip(idx, 0, L - 1)
    ek, ev = oracle.oracle_compact(k, v, safe)
    ek[0, 0, 5] = 0
    ev[0, 0, 5] = 0
    ek[1, 2, 7] = 0
    ev[1, 2, 7] = 0
    np.testing.assert_array_equal(to_bits(ko), ek)
    np.testing.assert_array_equal(to_bits(vo), ev)


def test_identical_keys_closed_form_on_gpu():
    m = kvp()
    b, hq, hkv, d, L, w = 1, 8, 2, 128, 1000, 32
    G = hq // hkv
    rng = np.random.default_rng(1)
    q = synth.round_bf16(rng.standard_normal((b, hq, w, d)))
    row = synth.round_bf16(rng.standard_normal(d))
    k = np.broadcast_to(row, (b, hkv, L, d)).copy()
    v = synth.round_bf16(rng.standard_normal((b, hkv, L, d)))
    sh = m.make_shape(b, hq, hkv, d, L, w, 64)
    buf = m.LayerBuffers(sh, "cuda", want_s1_s2=True)
    m.kvp_score(sh, to_dev(q), to_dev(k), to_dev(v), buf.score, buf.s1, buf.s2, buf.workspace)
    torch.cuda.synchronize()
    pos = np.arange(L - w, L)
    expect = np.array([G * np.sum(1.0 / (pos[pos >= j] + 1)) for j in range(L)])
    np.testing.assert_allclose(buf.s1.cpu().numpy()[0, 0], expect, rtol=1e-3)


def test_repeat_calls_are_deterministic():
    inp = synth.make_inputs(SMALL["ragged_d128_g4"])
    a = run_gpu(inp)
    b = run_gpu(inp)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])
