"""The seeded input generator produces the structure the workloads are described by.

These are checks of the synthetic inputs themselves (no eviction arithmetic): fixed
seeds give fixed bits, the bulk is N(0, 1), outlier channels carry the stated scale,
keys are rotated pairwise without changing the pair norms, and every planted needle
reaches at least the stated logit for one of its head's window queries.
"""
import math

import numpy as np

import synth


def test_same_seed_same_bits_other_layer_other_bits():
    a = synth.make_inputs("tiny", layer=0)
    b = synth.make_inputs("tiny", layer=0)
    c = synth.make_inputs("tiny", layer=1)
    for x, y in ((a.q_win, b.q_win), (a.k, b.k), (a.v, b.v)):
        np.testing.assert_array_equal(x, y)
    assert not np.array_equal(a.k, c.k)


def test_bulk_is_standard_normal_and_outlier_channels_are_scaled():
    inp = synth.make_inputs("tiny")
    wl = inp.workload
    k = synth.bf16_to_f64(inp.k)
    assert abs(k.mean()) < 0.02 and abs(k.std() - 1.0) < 0.02
    v = synth.bf16_to_f64(inp.v)[0]                      # [hkv, L, d]
    out = inp.v_outlier_channels[0]                      # [hkv, v_outliers]
    for h in range(wl.hkv):
        mask = np.zeros(wl.head_dim, dtype=bool)
        mask[out[h]] = True
        assert mask.sum() == wl.v_outliers
        assert abs(v[h][:, mask].std() / wl.outlier_scale - 1.0) < 0.1
        assert abs(v[h][:, ~mask].std() - 1.0) < 0.05


def test_rotation_keeps_pair_norms_and_leaves_position_zero_alone():
    rows, d, seed = 64, 128, 77
    plain = synth.bf16_to_f64(synth.normal_bf16(rows, d, seed, synth.STREAM_K, rows_per_head=rows))
    rot = synth.bf16_to_f64(synth.normal_bf16(rows, d, seed, synth.STREAM_K, rows_per_head=rows,
                                              rope_base=500000.0))
    np.testing.assert_array_equal(rot[0], plain[0])      # angle 0 at position 0
    h = d // 2
    n_plain = np.hypot(plain[:, :h], plain[:, h:])
    n_rot = np.hypot(rot[:, :h], rot[:, h:])
    np.testing.assert_allclose(n_rot, n_plain, rtol=1e-2, atol=1e-2)   # bf16 rounding
    assert not np.array_equal(rot[1:], plain[1:])


def test_every_needle_tops_the_stated_logit_for_a_window_query():
    wl = synth.small("long_128k_b70", seq_len=4096, budget=2867)
    inp = synth.make_inputs(wl)
    q = synth.bf16_to_f64(inp.q_win)[0]                  # [hq, w, d]
    k = synth.bf16_to_f64(inp.k)[0]                      # [hkv, L, d]
    G, d = wl.group, wl.head_dim
    assert inp.needle_pos.shape == (1, wl.hkv, wl.needles)
    for h in range(wl.hkv):
        qs = q[h * G:(h + 1) * G].reshape(-1, d)          # the head's G w window queries
        for j in inp.needle_pos[0, h]:
            assert 0 <= j < wl.seq_len - wl.window
            best = float(np.max(qs @ k[h, j])) / math.sqrt(d)
            assert best >= wl.needle_logit * 0.98, (h, int(j), best)
