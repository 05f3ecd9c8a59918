"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test fixes a result by mathematics or by a library routine, so that a plausible
slip in the oracle (a dropped term, a wrong scale, a wrong causal index, a wrong GQA
head mapping, a transposed operand, a wrong tie rule) fails at least one of them:

* the softmax rows of Eq. 3 each sum to 1, so sum_j S1[j] = G w;
* identical keys make every visible logit equal, giving S1 in closed form (harmonic
  sums that depend on the causal mask inside the window);
* a single planted key along one axis gives each softmax row in closed form, with
  per-query-head amplitudes that expose the GQA mapping and the scale C = sqrt(d);
* G = 1, w = 1 reduces Eq. 3 to one softmax row, compared with torch.softmax (fp64)
  and the log-sum-exp with scipy;
* planted |V| values give Eq. 4 exactly;
* selection against numpy's stable lexsort, compaction against numpy indexing;
* brute force with math.fsum on tiny inputs;
* adding one vector to every key shifts each query row's logits by a constant and
  leaves S1 unchanged (a softmax over the wrong axis fails this);
* permuting the positions before the window permutes S1, S2 and S with them (a causal
  bound measured from the wrong origin fails this).

All run on the CPU (no GPU mark).
"""
import math

import numpy as np
import pytest

import oracle
import synth


def bf16(x):
    return synth.round_bf16(np.asarray(x, dtype=np.float64))


def f64(bits):
    return synth.bf16_to_f64(bits)


def rand_inputs(b, hq, hkv, d, L, w, seed=7):
    rng = np.random.default_rng(seed)
    q = bf16(rng.standard_normal((b, hq, w, d)))
    k = bf16(rng.standard_normal((b, hkv, L, d)))
    v = bf16(rng.standard_normal((b, hkv, L, d)))
    return q, k, v


@pytest.mark.parametrize("b,hq,hkv,d,L,w", [(1, 4, 2, 64, 96, 8), (2, 6, 2, 32, 50, 7), (1, 2, 2, 16, 9, 9)])
def test_s1_total_is_g_times_w(b, hq, hkv, d, L, w):
    q, k, v = rand_inputs(b, hq, hkv, d, L, w)
    s1, s2, s = oracle.oracle_score(q, k, v)
    G = hq // hkv
    np.testing.assert_allclose(s1.sum(-1), G * w, rtol=1e-12)
    assert (s1 >= 0).all()


def test_identical_keys_closed_form():
    b, hq, hkv, d, L, w = 1, 6, 2, 64, 40, 6
    G = hq // hkv
    rng = np.random.default_rng(3)
    q = bf16(rng.standard_normal((b, hq, w, d)))
    row = bf16(rng.standard_normal(d))
    k = np.broadcast_to(row, (b, hkv, L, d)).copy()
    v = bf16(rng.standard_normal((b, hkv, L, d)))
    s1, _, _ = oracle.oracle_score(q, k, v)
    pos = [L - w + i for i in range(w)]
    expect = np.empty(L)
    for j in range(L):
        # row i sees p_i + 1 equal logits, so each visible key gets 1 / (p_i + 1)
        expect[j] = G * sum(1.0 / (p + 1) for p in pos if j <= p)
    for h in range(hkv):
        np.testing.assert_allclose(s1[0, h], expect, rtol=1e-12)


def test_planted_key_closed_form_gqa_mapping_and_scale():
    b, hq, hkv, d, L, w = 1, 6, 3, 64, 30, 4
    G = hq // hkv
    amp = [2.0, 4.0, 8.0, 16.0, 3.0, 6.0]   # one amplitude per query head, exact in bf16
    planted = [5, 11, 27]                   # the key position planted in each KV head
    q = np.zeros((b, hq, w, d))
    for hqi in range(hq):
        q[0, hqi, :, 0] = amp[hqi]
    k = np.zeros((b, hkv, L, d))
    for h in range(hkv):
        k[0, h, planted[h], 0] = 1.0
    v = np.ones((b, hkv, L, d))
    s1, s2, s = oracle.oracle_score(bf16(q), bf16(k), bf16(v))
    C = math.sqrt(d)
    for h in range(hkv):
        jstar = planted[h]
        expect = np.zeros(L)
        for g in range(G):
            x = amp[h * G + g] / C          # query head h*G+g belongs to KV head h
            for i in range(w):
                p = L - w + i
                if jstar <= p:
                    den = math.exp(x) + p   # one key at logit x, p keys at logit 0
                    for j in range(p + 1):
                        expect[j] += (math.exp(x) if j == jstar else 1.0) / den
                else:
                    for j in range(p + 1):
                        expect[j] += 1.0 / (p + 1)
        np.testing.assert_allclose(s1[0, h], expect, rtol=1e-12)
        np.testing.assert_array_equal(s2[0, h], 1.0)
        np.testing.assert_allclose(s[0, h], expect, rtol=1e-12)


def test_single_query_reduces_to_library_softmax():
    import torch
    from scipy.special import logsumexp
    b, hq, hkv, d, L, w = 2, 3, 3, 128, 257, 1
    q, k, v = rand_inputs(b, hq, hkv, d, L, w, seed=11)
    s1, s2, s, lse = oracle.oracle_score(q, k, v, want_lse=True)
    qf, kf = f64(q), f64(k)
    for bi in range(b):
        for h in range(hkv):
            logits = torch.from_numpy(kf[bi, h] @ qf[bi, h, 0]) / math.sqrt(d)
            ref = torch.softmax(logits, dim=0).numpy()
            np.testing.assert_allclose(s1[bi, h], ref, rtol=1e-12, atol=1e-300)
            np.testing.assert_allclose(lse[bi, h, 0], logsumexp(logits.numpy()), rtol=1e-13)


def test_s2_planted_abs_max():
    b, hkv, L, d = 1, 2, 20, 16
    rng = np.random.default_rng(5)
    v = rng.uniform(-0.5, 0.5, (b, hkv, L, d))
    expect = np.empty((b, hkv, L))
    for h in range(hkv):
        for j in range(L):
            val = (j + 1) * (0.25 if h == 0 else 0.75)
            sign = -1.0 if (j + h) % 2 else 1.0       # negative planted values: |.| matters
            v[0, h, j, (3 * j + h) % d] = sign * val
            expect[0, h, j] = max(val, 0.5) if val < 0.5 else val
    vb = bf16(v)
    # bf16 rounding of the planted values is exact (multiples of 1/4 below 256)
    q = bf16(rng.standard_normal((b, 2 * hkv, 2, d)))
    k = bf16(rng.standard_normal((b, hkv, L, d)))
    _, s2, _ = oracle.oracle_score(q, k, vb)
    ref = np.abs(f64(vb)).max(-1)                 # library max as a second witness
    np.testing.assert_array_equal(s2, ref)
    big = expect >= 0.5
    np.testing.assert_array_equal(s2[big], expect[big])


def brute_force(q, k, v):
    b, hq, w, d = q.shape
    _, hkv, L, _ = k.shape
    G = hq // hkv
    qf, kf, vf = f64(q), f64(k), f64(v)
    s1 = np.zeros((b, hkv, L))
    for bi in range(b):
        for h in range(hkv):
            for g in range(G):
                for i in range(w):
                    p = L - w + i
                    lg = [math.fsum(qf[bi, h * G + g, i, c] * kf[bi, h, j, c] for c in range(d)) / math.sqrt(d)
                          for j in range(p + 1)]
                    m = max(lg)
                    den = math.fsum(math.exp(x - m) for x in lg)
                    for j in range(p + 1):
                        s1[bi, h, j] += math.exp(lg[j] - m) / den
    s2 = np.abs(vf).max(-1)
    return s1, s2, s1 * s2


def test_brute_force_tiny():
    q, k, v = rand_inputs(2, 4, 2, 8, 24, 5, seed=21)
    s1, s2, s = oracle.oracle_score(q, k, v)
    r1, r2, r = brute_force(q, k, v)
    np.testing.assert_allclose(s1, r1, rtol=1e-12)
    np.testing.assert_array_equal(s2, r2)
    np.testing.assert_allclose(s, r, rtol=1e-12)


def library_select(score, w, B):
    L = score.shape[-1]
    out = []
    for row in score.reshape(-1, L):
        n = L - w
        order = np.lexsort((np.arange(n), -row[:n]))   # by -score, then by position
        keep = np.sort(np.concatenate([order[:B - w], np.arange(n, L)]))
        out.append(keep)
    return np.array(out, dtype=np.int32).reshape(score.shape[:-1] + (B,))


@pytest.mark.parametrize("L,w,B", [(100, 8, 30), (64, 1, 1), (64, 4, 64), (50, 50, 50), (33, 5, 5)])
def test_select_matches_library_sort(L, w, B):
    rng = np.random.default_rng(L + w + B)
    score = rng.random((3, 2, L))
    score[0, 0, 10:20] = 0.5                      # a block of exact ties
    idx = oracle.oracle_select(score, w, B)
    np.testing.assert_array_equal(idx, library_select(score, w, B))
    assert idx.shape == (3, 2, B)
    assert (np.diff(idx, axis=-1) > 0).all()      # strictly ascending
    assert (idx[..., B - w:] == np.arange(L - w, L)).all()


def test_select_ties_go_to_lower_position():
    L, w, B = 40, 4, 14
    score = np.full((1, L), 2.0)
    idx = oracle.oracle_select(score, w, B)
    np.testing.assert_array_equal(idx[0], np.r_[np.arange(B - w), np.arange(L - w, L)])


def test_compact_matches_library_indexing():
    rng = np.random.default_rng(9)
    k = rng.integers(0, 65536, (2, 3, 50, 16), dtype=np.uint16)
    v = rng.integers(0, 65536, (2, 3, 50, 16), dtype=np.uint16)
    idx = np.sort(rng.permuted(np.tile(np.arange(50), (6, 1)), axis=1)[:, :12], axis=1).reshape(2, 3, 12).astype(np.int32)
    ko, vo = oracle.oracle_compact(k, v, idx)
    np.testing.assert_array_equal(ko, np.take_along_axis(k, idx[..., None].astype(np.int64), axis=2))
    np.testing.assert_array_equal(vo, np.take_along_axis(v, idx[..., None].astype(np.int64), axis=2))


def test_planted_needle_and_value_outlier_are_kept():
    b, hq, hkv, d, L, w, B = 1, 4, 2, 64, 300, 8, 20
    q, k, v = rand_inputs(b, hq, hkv, d, L, w, seed=13)
    qf = f64(q)
    needle, outlier = 37, 201
    for h in range(hkv):
        qq = qf[0, h * 2 + 1, 3]
        k[0, h, needle] = bf16(24 * math.sqrt(d) * qq / (qq @ qq))   # logit 24 for that query
        v[0, h, outlier] = bf16(f64(v[0, h, outlier]) * 1000)
    out = oracle.oracle_layer(q, k, v, w, B)
    for h in range(hkv):
        assert needle in out["idx"][0, h]
        assert outlier in out["idx"][0, h]
    assert out["idx"].shape == (1, 2, B)


def test_identity_when_budget_is_context():
    q, k, v = rand_inputs(1, 2, 1, 16, 33, 3)
    out = oracle.oracle_layer(q, k, v, 3, 33)
    np.testing.assert_array_equal(out["idx"][0, 0], np.arange(33))
    np.testing.assert_array_equal(out["k_out"], k)


def test_bad_shapes_raise():
    q, k, v = rand_inputs(1, 2, 1, 16, 10, 3)
    with pytest.raises(ValueError):
        oracle.oracle_select(np.zeros((1, 10)), 3, 2)      # B < w
    with pytest.raises(ValueError):
        oracle.oracle_select(np.zeros((1, 10)), 3, 11)     # B > L
    with pytest.raises(ValueError):
        oracle.oracle_compact(k, v, np.array([[[0, 10]]], dtype=np.int32))


def test_adding_one_vector_to_every_key_leaves_s1_unchanged():
    # q . (k + u) = q . k + q . u shifts every logit of a query row by the same amount,
    # so each softmax row, and S1, is unchanged. Small integers keep K and K + u exact
    # in bf16, so the logits are exact in double on both sides.
    b, hq, hkv, d, L, w = 1, 6, 3, 32, 40, 5
    rng = np.random.default_rng(31)
    q = bf16(rng.integers(-2, 3, (b, hq, w, d)) / 4.0)
    k = rng.integers(-3, 4, (b, hkv, L, d)).astype(np.float64)
    u = rng.integers(-3, 4, (1, hkv, 1, d)).astype(np.float64)
    v = bf16(rng.standard_normal((b, hkv, L, d)))
    s1a, s2a, _ = oracle.oracle_score(q, bf16(k), v)
    s1b, s2b, _ = oracle.oracle_score(q, bf16(k + u), v)
    np.testing.assert_allclose(s1b, s1a, rtol=1e-10)
    np.testing.assert_array_equal(s2b, s2a)


def test_permuting_keys_before_the_window_permutes_the_scores():
    # Every window query sees every position before the window, so moving a (K, V) row
    # there moves its S1, S2 and S with it; window positions stay put.
    b, hq, hkv, d, L, w = 2, 4, 2, 16, 37, 6
    q, k, v = rand_inputs(b, hq, hkv, d, L, w, seed=41)
    n = L - w
    perm = np.random.default_rng(42).permutation(n)
    kp, vp = k.copy(), v.copy()
    kp[:, :, :n] = k[:, :, perm]
    vp[:, :, :n] = v[:, :, perm]
    s1, s2, s = oracle.oracle_score(q, k, v)
    s1p, s2p, sp = oracle.oracle_score(q, kp, vp)
    np.testing.assert_allclose(s1p[..., :n], s1[..., perm], rtol=1e-10)
    np.testing.assert_array_equal(s2p[..., :n], s2[..., perm])
    np.testing.assert_allclose(sp[..., :n], s[..., perm], rtol=1e-10)
    np.testing.assert_allclose(s1p[..., n:], s1[..., n:], rtol=1e-10)


# ---- selection policies: sinks, score modes, pooling kernel ---------------------------------

def _library_policy_select(key, w, B, sinks):
    """Kept set by numpy alone: [0, s), the B - w - s largest keys of [s, L - w) (stable on
    position), the window."""
    L = key.shape[-1]
    n = L - w
    cand = np.arange(sinks, n)
    order = np.lexsort((cand, -key[sinks:n]))
    chosen = cand[order[: B - w - sinks]]
    return np.sort(np.concatenate([np.arange(sinks), chosen, np.arange(n, L)])).astype(np.int32)


def test_policy_without_sinks_pooling_or_mode_is_the_plain_selection():
    rng = np.random.default_rng(11)
    s1, s2 = rng.random((3, 400)), rng.random((3, 400))
    got = oracle.oracle_select_policy(s1, s2, 16, 90)
    np.testing.assert_array_equal(got, oracle.oracle_select(s1 * s2, 16, 90))


@pytest.mark.parametrize("sinks,kernel,mode", [(4, 1, 0), (0, 5, 0), (7, 7, 0), (3, 3, 1), (5, 1, 2),
                                               (0, 1, 1), (16, 9, 0)])
def test_policy_matches_library_pooling_and_sort(sinks, kernel, mode):
    """Pooling against scipy's sliding maximum (positions past the ends left out), the
    mode's key by numpy, the selection by numpy's stable lexsort."""
    from scipy.ndimage import maximum_filter1d
    rng = np.random.default_rng(100 + sinks + 10 * kernel + mode)
    L, w, B = 333, 12, 80
    s1, s2 = rng.random((2, L)), rng.random((2, L))
    s1[:, 50:60] = 0.25                                  # a block of ties
    got, key = oracle.oracle_select_policy(s1, s2, w, B, sinks, kernel, mode, want_key=True)
    n = L - w
    pooled = maximum_filter1d(s1[:, :n], size=kernel, axis=-1, mode="constant", cval=-np.inf)
    want_key = pooled * s2[:, :n] if mode == 0 else pooled if mode == 1 else s2[:, :n]
    np.testing.assert_array_equal(key[:, :n], want_key)
    for r in range(2):
        full = np.concatenate([want_key[r], np.zeros(w)])    # the window's keys are never ranked
        np.testing.assert_array_equal(got[r], _library_policy_select(full, w, B, sinks))
    assert (got[:, :sinks] == np.arange(sinks)).all()
    assert (got[:, B - w:] == np.arange(n, L)).all()


def test_pooling_spreads_a_planted_spike_over_the_kernel():
    """S1 zero but one position: max pooling with kernel k turns it into a run of k equal
    keys centred there (cut at the window), and a budget of exactly that run keeps it."""
    L, w, k = 200, 10, 7
    for j0, run in ((50, range(47, 54)), (2, range(0, 6)), (188, range(185, 190))):
        s1 = np.zeros((1, L))
        s1[0, j0] = 1.0
        s2 = np.ones((1, L))
        run = list(run)
        got = oracle.oracle_select_policy(s1, s2, w, w + len(run), 0, k, 0)
        np.testing.assert_array_equal(got[0], np.array(run + list(range(L - w, L)), dtype=np.int32))


def test_sinks_are_kept_even_with_the_lowest_scores():
    rng = np.random.default_rng(5)
    s1 = rng.random((1, 300)) + 1.0
    s1[0, :6] = 0.0                                      # the sinks score lowest of all
    s2 = np.ones((1, 300))
    got = oracle.oracle_select_policy(s1, s2, 8, 40, sinks=6)
    assert got.shape == (1, 40)
    assert (got[0, :6] == np.arange(6)).all() and (np.diff(got[0]) > 0).all()


def test_single_precision_key_is_the_rounded_product():
    rng = np.random.default_rng(9)
    s1 = rng.random((2, 256)).astype(np.float32).astype(np.float64)
    s2 = (rng.random((2, 256)) * 30).astype(np.float32).astype(np.float64)
    s1[0, 3] = 1e-30                                     # product underflows to a subnormal
    _, key = oracle.oracle_select_policy(s1, s2, 8, 64, fp32_key=True, want_key=True)
    want = (s1.astype(np.float32) * s2.astype(np.float32)).astype(np.float64)
    want[np.abs(want) < np.finfo(np.float32).tiny] = 0.0
    np.testing.assert_array_equal(key[:, :248], want[:, :248])


def test_bad_policies_raise():
    s = np.ones((1, 50))
    for kw in (dict(sinks=45), dict(sinks=-1), dict(kernel=4), dict(kernel=0), dict(mode=3)):
        with pytest.raises(ValueError):
            oracle.oracle_select_policy(s, s, 8, 40, **kw)


# ---- CurDKV leverage scores (CurDKV rebuttal page, "A clearer description of Algorithm 1")

def lev_inputs(rows, L, d, r, seed):
    k = synth.normal_bf16(rows * L, d, seed, 1).reshape(rows, L, d)
    v = synth.normal_bf16(rows * L, d, seed, 2).reshape(rows, L, d)
    g = synth.normal_bf16(d, r, seed, 3)
    return k, v, g


def test_leverage_identity_projection_gives_library_row_norms():
    """G = I (r = d): the projected rows are the rows themselves, so the key and value
    scores are numpy's squared row norms, and the combined score their normalised product."""
    d, L = 16, 50
    k, v, _ = lev_inputs(2, L, d, d, seed=11)
    g = bf16(np.eye(d))
    score, lk, lv = oracle.oracle_leverage(k, v, g, want_parts=True)
    nk = np.linalg.norm(f64(k), axis=-1) ** 2
    nv = np.linalg.norm(f64(v), axis=-1) ** 2
    np.testing.assert_allclose(lk, nk, rtol=1e-13)
    np.testing.assert_allclose(lv, nv, rtol=1e-13)
    prod = nk * nv
    np.testing.assert_allclose(score, prod / prod.sum(-1, keepdims=True), rtol=1e-12)


def test_leverage_rank_one_projection_closed_form():
    """r = 1 with G = g: the key score is (K_j . g)^2, a dot product numpy computes; a
    transposed G, a dropped square or a sum in place of the product fails this."""
    d, L = 32, 40
    k, v, _ = lev_inputs(1, L, d, 1, seed=12)
    gcol = bf16(np.linspace(-1.5, 2.0, d))
    score, lk, lv = oracle.oracle_leverage(k, v, gcol.reshape(d, 1), want_parts=True)
    gv = f64(gcol)
    ek = (f64(k[0]) @ gv) ** 2
    ev = (f64(v[0]) @ gv) ** 2
    np.testing.assert_allclose(lk[0], ek, rtol=1e-12)
    np.testing.assert_allclose(lv[0], ev, rtol=1e-12)
    np.testing.assert_allclose(score[0], ek * ev / np.sum(ek * ev), rtol=1e-12)


def test_leverage_brute_force_tiny():
    d, L, r = 5, 7, 3
    k, v, g = lev_inputs(1, L, d, r, seed=13)
    K, V, G = f64(k[0]), f64(v[0]), f64(g)
    comb = []
    for j in range(L):
        nk = math.fsum(math.fsum(K[j, t] * G[t, c] for t in range(d)) ** 2 for c in range(r))
        nv = math.fsum(math.fsum(V[j, t] * G[t, c] for t in range(d)) ** 2 for c in range(r))
        comb.append(nk * nv)
    total = math.fsum(comb)
    np.testing.assert_allclose(oracle.oracle_leverage(k, v, g)[0], [c / total for c in comb], rtol=1e-12)


def test_leverage_invariants():
    """Scores sum to 1 per row; scaling G by 2 (exact in bf16) leaves them unchanged;
    permuting the positions permutes them; a zero key row scores 0."""
    d, L, r = 64, 300, 20
    k, v, g = lev_inputs(3, L, d, r, seed=14)
    s = oracle.oracle_leverage(k, v, g)
    np.testing.assert_allclose(s.sum(-1), 1.0, rtol=1e-12)
    g2 = bf16(2.0 * f64(g))
    np.testing.assert_allclose(oracle.oracle_leverage(k, v, g2), s, rtol=1e-12)
    perm = np.random.default_rng(3).permutation(L)
    np.testing.assert_allclose(oracle.oracle_leverage(k[:, perm], v[:, perm], g), s[:, perm], rtol=1e-12)
    kz = k.copy()
    kz[1, 17] = 0
    assert oracle.oracle_leverage(kz, v, g)[1, 17] == 0.0


# ---- AdaKV adaptive budgets (CurDKV rebuttal page, "On the sensitivity of the safeguard
#      parameter (alpha)", Tables 5-6)

def unpack(idx, counts, b, h):
    off = int(counts[b, :h].sum())
    return idx[b, off:off + counts[b, h]]


def adaptive_inputs(b, hkv, L, seed):
    rng = np.random.default_rng(seed)
    s = rng.random((b, hkv, L)) ** 3 * rng.uniform(0.2, 5.0, (b, hkv, 1))
    s[:, :, 5:40] = np.round(s[:, :, 5:40], 1)        # a block of ties within and across heads
    return s


def test_adaptive_alpha_one_is_the_uniform_budget():
    """alpha = 1: every head keeps its own best B - w and the window (numpy's stable sort)."""
    b, hkv, L, w, B = 2, 3, 300, 8, 60
    s = adaptive_inputs(b, hkv, L, 21)
    idx, counts = oracle.oracle_select_adaptive(s, w, B, 1.0)
    assert (counts == B).all()
    for bi in range(b):
        for h in range(hkv):
            np.testing.assert_array_equal(unpack(idx, counts, bi, h), library_select(s[bi, h], w, B))


def test_adaptive_alpha_zero_is_one_global_top_k():
    """alpha = 0: the sequence's hkv (B - w) non-window positions are the best of all its
    heads' candidates, ordered by (score desc, head, position) with numpy's lexsort."""
    b, hkv, L, w, B = 2, 4, 200, 5, 40
    s = adaptive_inputs(b, hkv, L, 22)
    idx, counts = oracle.oracle_select_adaptive(s, w, B, 0.0)
    n = L - w
    for bi in range(b):
        hh, jj = np.meshgrid(np.arange(hkv), np.arange(n), indexing="ij")
        sc = s[bi, :, :n]
        order = np.lexsort((jj.ravel(), hh.ravel(), -sc.ravel()))[: hkv * (B - w)]
        keep = np.zeros((hkv, L), bool)
        keep[hh.ravel()[order], jj.ravel()[order]] = True
        keep[:, n:] = True
        for h in range(hkv):
            np.testing.assert_array_equal(unpack(idx, counts, bi, h), np.flatnonzero(keep[h]))


@pytest.mark.parametrize("alpha", [0.2, 0.5, 0.9])
def test_adaptive_exchange_property(alpha):
    """Any alpha: each head keeps its window and at least its best floor(alpha (B - w));
    the sequence keeps hkv B in all; and no unkept candidate outranks a kept one that is
    not in its head's floor (in (score desc, head, position) order)."""
    b, hkv, L, w, B = 2, 5, 400, 16, 80
    s = adaptive_inputs(b, hkv, L, 23)
    idx, counts = oracle.oracle_select_adaptive(s, w, B, alpha)
    n, f = L - w, int(np.floor(alpha * (B - w)))
    assert (counts.sum(1) == hkv * B).all()
    for bi in range(b):
        kept_extra, unkept = [], []
        for h in range(hkv):
            kept = unpack(idx, counts, bi, h)
            assert (np.diff(kept) > 0).all()
            assert set(range(n, L)) <= set(kept.tolist())
            floor = library_select(s[bi, h], w, f + w)[:f]
            assert set(floor.tolist()) <= set(kept.tolist())
            others = set(kept.tolist()) - set(floor.tolist()) - set(range(n, L))
            kept_extra += [(-s[bi, h, j], h, j) for j in others]
            unkept += [(-s[bi, h, j], h, j) for j in set(range(n)) - set(kept.tolist())]
        if kept_extra and unkept:
            assert max(kept_extra) < min(unkept)


def test_adaptive_equal_scores_fill_the_lowest_heads_first():
    """All scores equal, alpha = 0: the shared positions go to head 0's candidates in
    position order, then head 1's, ... (the tie rule), a closed form."""
    hkv, L, w, B = 3, 50, 4, 20
    s = np.ones((1, hkv, L))
    idx, counts = oracle.oracle_select_adaptive(s, w, B, 0.0)
    n, R = L - w, hkv * (B - w)
    expect = []
    for h in range(hkv):
        take = max(0, min(n, R - h * n))
        expect.append(np.concatenate([np.arange(take), np.arange(n, L)]))
    np.testing.assert_array_equal(counts[0], [len(e) for e in expect])
    np.testing.assert_array_equal(idx[0], np.concatenate(expect))


def test_adaptive_rejects_bad_alpha():
    with pytest.raises(ValueError):
        oracle.oracle_select_adaptive(np.ones((1, 2, 10)), 2, 5, 1.5)
