"""Pins for the CPU oracle: hand-worked examples, brute force, closed forms and
invariants that the explainer's method section fixes.  CPU only."""
import itertools

import numpy as np
import pytest

import oracle
import synth


def _floats(v):
    return np.array([float(x) for x in v], dtype=np.float64)


def _ints(v):
    return np.array([int(x, 0) for x in v], dtype=np.int64)


# ----------------------------------------------------------------- quantiser
def test_quantize_hand_worked(golden):
    g = golden("quantize_worked.txt")
    keys = np.stack([_floats(g["keys_channel_A"]), _floats(g["keys_channel_B"]),
                     _floats(g["keys_channel_C"])], axis=1).astype(np.float32)[None]
    mn, scale, codes = oracle.quantize(keys)
    assert np.array_equal(mn[0], _floats(g["mn"]).astype(np.float32))
    assert np.array_equal(scale[0], _floats(g["scale"]).astype(np.float32))
    for c, name in enumerate("ABC"):
        assert np.array_equal(codes[0, c], _ints(g["codes_" + name])), name
    s1, s2, sigma2 = oracle.channel_stats(codes, scale)
    assert np.array_equal(s1[0], _ints(g["S1"]))
    assert np.array_equal(s2[0], _ints(g["S2"]))
    assert np.array_equal(sigma2[0], _floats(g["sigma2"]).astype(np.float32))


def test_quantize_error_bound_and_extremes():
    """Round-to-nearest over 16 evenly spaced levels: each key is within half a
    step of its level; the channel min maps to 0 and the max to 15."""
    ses = synth.make_session(3, 2, 1, 1000, 16)
    mn, scale, codes = oracle.quantize(ses.keys)
    k = ses.keys.transpose(0, 2, 1).astype(np.float64)          # [H][d][n]
    deq = mn[..., None].astype(np.float64) + scale[..., None].astype(np.float64) * codes
    err = np.abs(deq - k)
    assert np.all(err <= scale[..., None] * (0.5 + 1e-5) + 1e-6)
    assert np.all(codes <= 15)
    jmin = np.argmin(k, axis=2)
    jmax = np.argmax(k, axis=2)
    assert np.all(np.take_along_axis(codes, jmin[..., None], 2) == 0)
    assert np.all(np.take_along_axis(codes, jmax[..., None], 2) == 15)
    # every level is used by a Gaussian channel of 1000 keys except possibly a few
    assert len(np.unique(codes[0, 0])) >= 10


def test_sigma2_matches_variance_of_dequantised_keys():
    """sigma^2 is the population variance of mn + scale*code: compare with
    numpy's two-pass variance (a different algorithm) in fp64."""
    ses = synth.make_session(5, 2, 1, 3000, 16)
    mn, scale, codes = oracle.quantize(ses.keys)
    _, _, sigma2 = oracle.channel_stats(codes, scale)
    deq = mn[..., None].astype(np.float64) + scale[..., None].astype(np.float64) * codes
    ref = deq.var(axis=2)
    assert np.allclose(sigma2, ref, rtol=1e-6, atol=0)
    # and it estimates the generating variance (4-bit noise adds scale^2/12)
    ratio = sigma2 / (ses.sigma ** 2)
    assert np.all((ratio > 0.8) & (ratio < 1.25))


# -------------------------------------------------------------------- planes
def test_plane_layout_hand_worked(golden):
    g = golden("plane_layout.txt")
    n = int(g["n"][0])
    codes = np.zeros((1, 1, n), np.uint8)
    codes[0, 0, 0] = int(g["code_key_0"][0])
    codes[0, 0, 37] = int(g["code_key_37"][0])
    codes[0, 0, 63] = int(g["code_key_63"][0])
    planes = oracle.pack_planes(codes)
    assert planes.shape == (1, 1, 4, 4)
    for s, name in enumerate(["slot0_bit3", "slot1_bit2", "slot2_bit1", "slot3_bit0"]):
        assert np.array_equal(planes[0, 0, s], _ints(g[name]).astype(np.uint32)), name


@pytest.mark.parametrize("n", [1, 31, 32, 33, 127, 128, 129, 1000])
def test_planes_round_trip_and_padding(n):
    rng = np.random.default_rng(n)
    codes = rng.integers(0, 16, size=(2, 3, n), dtype=np.uint8)
    planes = oracle.pack_planes(codes)
    n_w = oracle.n_words_for(n)
    assert planes.shape == (2, 3, 4, n_w) and n_w % 4 == 0
    assert np.array_equal(oracle.unpack_planes(planes, n), codes)
    # keys past n carry no bits
    full = oracle.unpack_planes(planes, n_w * 32)
    assert not full[..., n:].any()


def test_index_is_the_4bit_cache_size():
    """No extra copy: the planes of a head hold exactly n*d/2 bytes (4 bits per
    key per channel) when n is a multiple of 128."""
    ses = synth.make_session(1, 2, 1, 4096, 16)
    ix = oracle.build_index(ses.keys)
    assert ix["planes"].nbytes == 2 * 4096 * 128 // 2


# ---------------------------------------------------------------- importance
def test_importance_values():
    sigma2 = np.array([3.0, 3.0, 5.0, 0.0], np.float32)
    q = synth.f32_to_bf16_bits(np.array([2.0, -2.0, 0.0, 7.0], np.float32))
    w = oracle.importance(q, sigma2)
    assert np.array_equal(w, np.array([12.0, 12.0, 0.0, 0.0], np.float32))


def test_importance_rejects_nonfinite():
    q = synth.f32_to_bf16_bits(np.array([1e30, 1.0], np.float32))
    with pytest.raises(ValueError):
        oracle.importance(q, np.array([1e30, 1.0], np.float32))


# ---------------------------------------------------------------------- plan
def test_plan_hand_worked(golden):
    g = golden("plan_worked.txt")
    for case in ("case1", "case2", "case3", "case4", "case5"):
        w = _floats(g[case + "_w"]).astype(np.float32)
        t = oracle.plan_greedy(w, int(g[case + "_B"][0]))
        assert np.array_equal(t, _ints(g[case + "_t"])), case
    t1 = oracle.plan_greedy(_floats(g["case1_w"]).astype(np.float32), 18)
    n = int(g["case1_n"][0])
    assert oracle.plan_bytes(t1, oracle.n_words_for(n)) == int(g["case1_bytes"][0])


def _brute_force_best(w, B):
    d = len(w)
    best = -1.0
    w64 = w.astype(np.float64)
    for alloc in itertools.product(range(5), repeat=d):
        if sum(alloc) <= B:
            v = float(np.dot(w64, alloc))
            best = max(best, v)
    return best


@pytest.mark.parametrize("d", [1, 2, 3, 5])
def test_plan_is_optimal_by_brute_force_small(d):
    rng = np.random.default_rng(100 + d)
    for trial in range(6):
        w = rng.lognormal(0, 1, size=d).astype(np.float32)
        if trial == 0:
            w[:] = 1.0                      # all tied
        if trial == 1 and d > 1:
            w[0] = 0.0                      # zero importance
        for B in range(0, 4 * d + 1):
            t = oracle.plan_greedy(w, B)
            assert int(t.sum()) == min(B, 4 * d)
            assert np.all(t <= 4)
            got = float(np.dot(w.astype(np.float64), t))
            assert got == pytest.approx(_brute_force_best(w, B), rel=1e-12, abs=0)


def test_plan_is_optimal_by_brute_force_d8():
    """All 5^8 = 390625 allocations of head_dim 8, vectorised."""
    d = 8
    allocs = np.array(list(itertools.product(range(5), repeat=d)), dtype=np.int64)
    sums = allocs.sum(axis=1)
    rng = np.random.default_rng(8)
    for trial in range(4):
        w = rng.lognormal(0, 1.5, size=d).astype(np.float32)
        vals = allocs @ w.astype(np.float64)
        for B in (0, 1, 3, 4, 7, 8, 13, 18, 20, 31, 32):
            t = oracle.plan_greedy(w, B)
            best = vals[sums <= B].max()
            assert float(np.dot(w.astype(np.float64), t)) == pytest.approx(best, rel=1e-12)
            assert int(t.sum()) == min(B, 32)


def test_plan_tiny_budget_reads_two_channels():
    """Intuition example 3: at 8 bits/key or less at most 2 channels are read."""
    rng = np.random.default_rng(7)
    for _ in range(20):
        w = rng.lognormal(0, 1, size=128).astype(np.float32)
        for B in range(0, 9):
            t = oracle.plan_greedy(w, B)
            assert (t > 0).sum() == (B + 3) // 4 <= 2


def test_plan_rejects_bad_budget():
    w = np.ones(4, np.float32)
    for B in (-1, 17):
        with pytest.raises(ValueError):
            oracle.plan_greedy(w, B)


# ------------------------------------------------------------- fixed plans
def test_fixed_plan_hand_worked(golden):
    g = golden("fixed_plan_worked.txt")
    q = synth.f32_to_bf16_bits(_floats(g["q"]).astype(np.float32))
    assert np.array_equal(oracle.fixed_plan(q, int(g["r"][0])), _ints(g["t"]))
    assert np.array_equal(oracle.fixed_plan(q, int(g["r1"][0])), _ints(g["r1_t"]))


def test_fixed_plan_widths():
    """Fixed 136-bit and 68-bit scans: 34 / 17 channels at 4 bits."""
    q = synth.make_session(0, 1, 1, 128, 16).q_bf16[0]
    for r, bits in ((34, 136), (17, 68)):
        t = oracle.fixed_plan(q, r)
        assert int(t.sum()) == bits and set(np.unique(t)) <= {0, 4}
        absq = np.abs(synth.bf16_bits_to_f32(q))
        assert absq[t == 4].min() >= absq[t == 0].max()


# --------------------------------------------------------- union and bytes
def test_union_and_bytes():
    ses = synth.make_session(11, 2, 4, 4096, 92)
    ix = oracle.build_index(ses.keys)
    t, T, nb = oracle.plan_session(ix, ses.q_bf16, ses.budgets, 4)
    n = 4096
    Q = 8
    for q in range(Q):
        assert int(nb[q]) == 92 * n // 8          # bytes = B * n / 8
    for h in range(2):
        grp = t[4 * h:4 * h + 4]
        assert np.array_equal(T[h], grp.max(axis=0))
        assert int(nb[Q + h]) == int(T[h].sum()) * n // 8
        assert max(nb[4 * h:4 * h + 4]) <= nb[Q + h] <= sum(nb[4 * h:4 * h + 4])


# -------------------------------------------------------------------- score
def test_coarse_bin_midpoint_hand_worked(golden):
    g = golden("midpoint_worked.txt")
    code = int(g["code"][0])
    one = synth.f32_to_bf16_bits(np.array([1.0], np.float32))
    for t, kh in zip(_ints(g["t"]), _floats(g["khat"])):
        codes = np.array([[[code]]], np.uint8)
        planes = oracle.pack_planes(codes)
        s = oracle.score_planes(planes[0], np.zeros(1, np.float32), np.ones(1, np.float32),
                                one, np.array([t], np.uint8), 1)
        assert s[0] == kh


def test_score_and_absolute_sum_hand_worked(golden):
    """The score of a key read at t = (2, 1) bits and A_j, the sum of the
    absolute terms every score tolerance is scaled by, on a key whose terms
    have opposite signs (|s_j| < A_j) and whose planes past t are set."""
    g = golden("abs_score_worked.txt")
    n = int(g["n"][0])
    planes = np.stack([np.stack([_ints(g[f"ch{c}_slot{s}"]) for s in range(4)])
                       for c in range(2)]).astype(np.uint32)          # [d][4][n_words]
    mn = _floats(g["mn"]).astype(np.float32)
    sc = _floats(g["scale"]).astype(np.float32)
    q = synth.f32_to_bf16_bits(_floats(g["q"]).astype(np.float32))
    t = _ints(g["t"]).astype(np.uint8)
    keys = _ints(g["keys"])
    s = oracle.score_planes(planes, mn, sc, q, t, n)
    a = oracle.score_abs_planes(planes, mn, sc, q, t, n)
    assert np.array_equal(s[keys], _floats(g["s"]))
    assert np.array_equal(a[keys], _floats(g["A"]))
    # every other key has code 0 in both channels: the same terms as key 1
    rest = np.setdiff1d(np.arange(n), keys)
    assert np.all(a[rest] == a[1]) and np.all(s[rest] == s[1])


def test_exact_scores_hand_worked(golden):
    g = golden("exact_score_worked.txt")
    keys = np.stack([_floats(g["key0"]), _floats(g["key1"])]).astype(np.float32)   # [n][d]
    q = synth.f32_to_bf16_bits(_floats(g["q"]).astype(np.float32))
    assert np.array_equal(oracle.exact_scores(keys, q), _floats(g["s"]))


def test_coarse_bin_is_mean_of_its_fine_levels():
    """Reading t bits rebuilds a key at the mean of the 2^(4-t) fine levels of
    its coarse bin (all bins are equally wide)."""
    mn, sc = np.float32(-1.25), np.float32(0.375)
    one = synth.f32_to_bf16_bits(np.array([1.0], np.float32))
    codes = np.arange(16, dtype=np.uint8)[None, None, :]
    planes = oracle.pack_planes(codes)
    for t in range(5):
        s = oracle.score_planes(planes[0], np.array([mn]), np.array([sc]), one,
                                np.array([t], np.uint8), 16)
        width = 1 << (4 - t)
        for code in range(16):
            lo = (code // width) * width
            levels = float(mn) + float(sc) * np.arange(lo, lo + width, dtype=np.float64)
            assert s[code] == pytest.approx(levels.mean(), rel=1e-15, abs=1e-15)


def test_full_depth_score_is_the_4bit_dot_product():
    """t_c = 4 for every channel: the score is the exact dot product with the
    dequantised 4-bit keys (computed here by a numpy fp64 matmul)."""
    ses = synth.make_session(2, 2, 2, 700, 512)
    ix = oracle.build_index(ses.keys)
    t4 = np.full(128, 4, np.uint8)
    for h in range(2):
        deq = ix["mn"][h][:, None].astype(np.float64) + \
            ix["scale"][h][:, None].astype(np.float64) * ix["codes"][h]   # [d][n]
        for g in range(2):
            q = ses.q_bf16[2 * h + g]
            s = oracle.score_planes(ix["planes"][h], ix["mn"][h], ix["scale"][h], q, t4, 700)
            ref = synth.bf16_bits_to_f32(q).astype(np.float64) @ deq
            mag = np.abs(synth.bf16_bits_to_f32(q).astype(np.float64)) @ np.abs(deq)
            assert np.all(np.abs(s - ref) <= 1e-13 * mag)


def test_reading_t_planes_equals_requantising_to_t_bits():
    """Storage-side invariant: the score from the first t_c planes equals the
    score from the codes re-quantised to t_c bits (code >> (4 - t_c)); the two
    oracle routes agree bit for bit, for greedy and arbitrary plans."""
    ses = synth.make_session(9, 1, 3, 1500, 50)
    ix = oracle.build_index(ses.keys)
    rng = np.random.default_rng(0)
    plans = [oracle.plan_greedy(oracle.importance(ses.q_bf16[g], ix["sigma2"][0]), B)
             for g, B in ((0, 18), (1, 92), (2, 136))]
    plans.append(rng.integers(0, 5, size=128).astype(np.uint8))
    for t in plans:
        for g in range(3):
            a = oracle.score_planes(ix["planes"][0], ix["mn"][0], ix["scale"][0],
                                    ses.q_bf16[g], t, 1500)
            b = oracle.score_codes(ix["codes"][0], ix["mn"][0], ix["scale"][0],
                                   ses.q_bf16[g], t)
            assert np.array_equal(a, b)


def test_zero_depth_score_is_constant():
    ses = synth.make_session(4, 1, 1, 300, 0)
    ix = oracle.build_index(ses.keys)
    s = oracle.score_planes(ix["planes"][0], ix["mn"][0], ix["scale"][0], ses.q_bf16[0],
                            np.zeros(128, np.uint8), 300)
    qf = synth.bf16_bits_to_f32(ses.q_bf16[0]).astype(np.float64)
    const = qf @ (ix["mn"][0].astype(np.float64) + 7.5 * ix["scale"][0].astype(np.float64))
    assert np.allclose(s, const, rtol=1e-13, atol=0)
    assert np.all(s == s[0])


def test_exact_scores_match_matmul():
    ses = synth.make_session(6, 1, 1, 500, 0)
    s = oracle.exact_scores(ses.keys[0], ses.q_bf16[0])
    ref = ses.keys[0].astype(np.float64) @ synth.bf16_bits_to_f32(ses.q_bf16[0]).astype(np.float64)
    assert np.allclose(s, ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------- top-k
def test_topk_hand_worked(golden):
    g = golden("topk_worked.txt")
    s = _floats(g["scores"])
    assert np.array_equal(oracle.topk(s, 3)[0], _ints(g["k3_idx"]))
    assert np.array_equal(oracle.topk(s, 4)[0], _ints(g["k4_idx"]))


def test_topk_matches_full_sort_with_ties():
    rng = np.random.default_rng(1)
    s = rng.integers(0, 50, size=5000).astype(np.float64)      # many ties
    for k in (1, 7, 64, 2048, 5000):
        idx, top = oracle.topk(s, k)
        ref = np.lexsort((np.arange(5000), -s))[:k]
        assert np.array_equal(idx, ref)
        assert np.array_equal(top, s[ref])


def test_recall_bounds():
    assert oracle.recall([1, 2, 3], [3, 2, 1]) == 1.0
    assert oracle.recall([1, 2, 3], [4, 5, 6]) == 0.0
    assert oracle.recall([1, 2, 9], [1, 2, 3, 4]) == 0.5


def test_tiny_workload_planted_keys_rank_high():
    """Sanity (reported, not a pin): the 16 planted keys close to the query
    land in the top-64 at 64 bits/key."""
    ses = synth.tiny_4k()
    ix = oracle.build_index(ses.keys)
    t, T, nb = oracle.plan_session(ix, ses.q_bf16, ses.budgets, 1)
    idx, _, _ = oracle.scan_query(ix, ses.q_bf16[0], t[0], 0, 64)
    assert len(set(ses.planted[0].tolist()) & set(idx.tolist())) >= 12


# ------------------------------------------------------------------ append
def _split_in_range(seed, H, n, m, d):
    """n keys to pack, then m new keys clipped into the packed keys' range."""
    ses = synth.make_session(seed, H, 1, n + m, 64, head_dim=d)
    first = ses.keys[:, :n]
    lo = first.min(axis=1, keepdims=True)
    hi = first.max(axis=1, keepdims=True)
    return first, np.clip(ses.keys[:, n:], lo, hi).astype(np.float32)


@pytest.mark.parametrize("n,m", [(900, 100), (31, 2), (32, 1), (127, 129), (4096, 1)])
def test_append_in_range_equals_repacking_everything(n, m):
    """Keys inside the stored range leave min and max, so scale and every
    code are unchanged: appending must give exactly the index of all n+m."""
    first, new = _split_in_range(n + m, 2, n, m, 32)
    ix = oracle.build_index(first, capacity=n + m)
    clamped = np.zeros((2, 32), np.uint32)
    assert oracle.append(ix, new, clamped) == n + m
    full = oracle.build_index(np.concatenate([first, new], axis=1))
    for name in ("planes", "s1", "s2", "sigma2", "mn", "scale"):
        assert np.array_equal(ix[name], full[name]), name
    assert clamped.sum() == 0


def test_append_one_by_one_equals_one_batch():
    first, new = _split_in_range(7, 1, 500, 70, 16)
    a = oracle.build_index(first, capacity=570)
    b = oracle.build_index(first, capacity=570)
    oracle.append(a, new)
    for i in range(70):
        oracle.append(b, new[:, i:i + 1])
    for name in ("planes", "s1", "s2", "sigma2"):
        assert np.array_equal(a[name], b[name]), name


def test_append_clamps_out_of_range_keys_to_the_end_levels():
    keys = np.zeros((1, 16, 2), np.float32)
    keys[0, :, 0] = np.arange(16)          # channel 0: 0..15, scale 1
    keys[0, :, 1] = 3.0                    # channel 1: constant, scale 0
    ix = oracle.build_index(keys, capacity=128)
    assert ix["scale"][0, 0] == 1.0 and ix["scale"][0, 1] == 0.0
    new = np.array([[[-10.0, 3.0], [0.0, 4.0], [15.0, 3.0], [40.0, -1.0], [7.4, 3.0]]],
                   np.float32)
    clamped = np.zeros((1, 2), np.uint32)
    oracle.append(ix, new, clamped)
    codes = ix["codes"][0]
    assert list(codes[0, 16:]) == [0, 0, 15, 15, 7]
    assert list(codes[1, 16:]) == [0, 0, 0, 0, 0]
    assert list(clamped[0]) == [2, 2]      # -10 and 40; the two values != 3


def test_append_keeps_sigma2_the_variance_of_the_stored_keys():
    ses = synth.make_session(9, 2, 1, 3000, 64, head_dim=16)
    ix = oracle.build_index(ses.keys[:, :2000], capacity=3000)
    oracle.append(ix, ses.keys[:, 2000:] * 1.3)        # partly out of range
    deq = ix["mn"][:, :, None].astype(np.float64) + \
        ix["scale"][:, :, None].astype(np.float64) * ix["codes"].astype(np.float64)
    np.testing.assert_allclose(ix["sigma2"], deq.var(axis=2), rtol=1e-5)
    assert np.array_equal(ix["s1"], ix["codes"].astype(np.int64).sum(axis=2))


def test_append_rejects_overflow_and_nonfinite():
    ses = synth.make_session(3, 1, 1, 200, 64, head_dim=8)
    ix = oracle.build_index(ses.keys[:, :100])              # capacity 128
    with pytest.raises(ValueError):
        oracle.append(ix, ses.keys[:, 100:130])
    bad = ses.keys[:, 100:101].copy()
    bad[0, 0, 3] = np.inf
    with pytest.raises(ValueError):
        oracle.append(ix, bad)


# ------------------------------------------------------------- attention
def _kv(seed, n, d):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, d)).astype(np.float32),
            rng.standard_normal((n, d)).astype(np.float32),
            synth.f32_to_bf16_bits(rng.standard_normal(d).astype(np.float32)))


def test_attention_over_every_key_is_dense_attention():
    K, V, q = _kv(1, 300, 16)
    dense = oracle.attention(K, V, q)
    listed = oracle.attention(K, V, q, np.arange(300)[::-1].copy())   # order is irrelevant
    np.testing.assert_allclose(listed, dense, rtol=1e-12, atol=1e-14)
    # against the softmax written with numpy's exp and matmul
    qf = synth.bf16_bits_to_f32(q).astype(np.float64)
    logit = (K.astype(np.float64) @ qf) / 4.0
    p = np.exp(logit - logit.max())
    np.testing.assert_allclose(dense, (p / p.sum()) @ V.astype(np.float64), rtol=1e-10)


def test_attention_special_cases():
    K, V, q = _kv(2, 50, 8)
    # one key: its value row exactly
    assert np.array_equal(oracle.attention(K, V, q, np.array([17])), V[17].astype(np.float64))
    # a zero query: the plain mean of the listed value rows
    zero = np.zeros(8, np.uint16)
    sel = np.array([3, 9, 20, 41])
    np.testing.assert_allclose(oracle.attention(K, V, zero, sel), V[sel].astype(np.float64).mean(0),
                               rtol=1e-12)
    # a key far above the others takes all the weight, even with logits in
    # the thousands (softmax must stay finite)
    K2 = K.copy()
    K2[5] = 1000.0 * synth.bf16_bits_to_f32(q)
    out = oracle.attention(K2, V, q, np.array([1, 5, 7]))
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out, V[5], atol=1e-9)


def test_attention_error_metric():
    o = np.array([1.0, 0.0, 0.0])
    assert oracle.attention_error(o, o) == 0.0
    assert abs(oracle.attention_error(np.array([1.0, 0.5, 0.0]), o) - 0.5) < 1e-15
    # relative to the exact output's norm: |(0, 0, 2.5)| / |(3, 4, 0)| = 2.5 / 5
    assert abs(oracle.attention_error(np.array([3.0, 4.0, 2.5]), np.array([3.0, 4.0, 0.0])) - 0.5) < 1e-15
    with pytest.raises(ValueError):
        oracle.attention(np.zeros((4, 2), np.float32), np.zeros((4, 2), np.float32),
                         np.zeros(2, np.uint16), np.array([4]))


# ------------------------------------------------------- marginal-gain plan
def _distortion_drop(w, t):
    """Sum_c w_c (1 - 4^-t_c): the distortion a plan removes when a channel
    read at t bits keeps 4^-t of its variance."""
    return float(np.sum(np.asarray(w, np.float64) * (1.0 - 4.0 ** (-np.asarray(t, np.float64)))))


@pytest.mark.parametrize("d", [3, 5])
def test_marginal_plan_is_optimal_by_brute_force(d):
    rng = np.random.default_rng(d)
    for trial in range(6):
        w = rng.lognormal(0.0, 1.5, d).astype(np.float32)
        for B in range(0, 4 * d + 1):
            t = oracle.plan_marginal(w, B)
            assert int(t.sum()) == B and t.max() <= 4
            best = max(_distortion_drop(w, c) for c in itertools.product(range(5), repeat=d)
                       if sum(c) == B)
            assert abs(_distortion_drop(w, t) - best) <= 1e-9 * max(1.0, best)


def test_marginal_plan_spreads_uniform_importance_round_robin():
    d = 10
    w = np.full(d, 2.5, np.float32)
    for B in range(0, 4 * d + 1):
        t = oracle.plan_marginal(w, B)
        expect = np.array([B // d + (c < B % d) for c in range(d)])
        assert np.array_equal(t, expect), B


def test_marginal_plan_hand_worked():
    # gains of channel 0: 16, 4, 1, 1/4; channel 1: 1, 1/4, ...; ties -> channel 0
    w = np.array([16.0, 1.0], np.float32)
    assert [list(oracle.plan_marginal(w, B)) for B in range(1, 6)] == \
        [[1, 0], [2, 0], [3, 0], [3, 1], [4, 1]]
    # water-filling instead fills channel 0 to 4 bits before channel 1 gets any
    assert list(oracle.plan_greedy(w, 4)) == [4, 0]


# ------------------------------------------------------------ sharded keys
@pytest.mark.parametrize("S,n,k", [(2, 1000, 50), (3, 999, 64), (4, 4096, 300), (5, 60, 12)])
def test_merging_shard_topks_is_the_topk_of_all_keys(S, n, k):
    """Split the keys into S ranges, take each range's top-k, merge: the
    result is the top-k of all keys (indices ascending), ties included."""
    rng = np.random.default_rng(S * n + k)
    s = np.round(rng.standard_normal(n), 1)          # many exact ties
    cuts = np.sort(rng.choice(np.arange(1, n), S - 1, replace=False))
    bounds = [0, *cuts.tolist(), n]
    k_s = max(min(k, b - a) for a, b in zip(bounds, bounds[1:]))
    idx = np.zeros((S, k_s), np.int32)
    sc = np.full((S, k_s), -np.inf)
    for r, (a, b) in enumerate(zip(bounds, bounds[1:])):
        kk = min(k, b - a)
        li, ls = oracle.topk(s[a:b], kk)
        idx[r, :kk], sc[r, :kk] = li, ls
        idx[r, kk:] = 0                                   # padding rows never win
    gi, gs = oracle.merge_topk(idx, sc, np.array(bounds[:-1]), k)
    ref_i, _ = oracle.topk(s, k)
    assert np.array_equal(gi, np.sort(ref_i))
    assert np.all(np.diff(gi) > 0)
    np.testing.assert_array_equal(gs, s[gi])


# -------------------------------------------------------- 8-plane variant
# The explainer's deployment notes (部署前必读, item 3) say an 8-bit upstream K
# cache needs the index adapted to 8 planes per channel.  Reading: the same
# quantiser with 255 levels, slots MSB first, plans capped at 8 bits, and the
# same coarse-bin midpoint rebuild.  These pins fix that reading.
def test_quantize_8bit_hand_worked():
    """max - min = 255 makes scale exactly 1, so each code is
    floor(k - min + 0.5): worked by hand."""
    keys = np.array([-100.0, 155.0, 27.25, 27.75, 0.5, 130.5, 154.4], np.float32)
    mn, scale, codes = oracle.quantize(keys[None, :, None], bits=8)
    assert mn[0, 0] == -100.0 and scale[0, 0] == 1.0
    assert list(codes[0, 0]) == [0, 255, 127, 128, 101, 231, 254]
    s1, s2, _ = oracle.channel_stats(codes, scale)
    assert s1[0, 0] == 0 + 255 + 127 + 128 + 101 + 231 + 254
    assert s2[0, 0] == 255 ** 2 + 127 ** 2 + 128 ** 2 + 101 ** 2 + 231 ** 2 + 254 ** 2


def test_quantize_8bit_error_bound_and_extremes():
    ses = synth.make_session(13, 2, 1, 3000, 16)
    mn, scale, codes = oracle.quantize(ses.keys, bits=8)
    k = ses.keys.transpose(0, 2, 1).astype(np.float64)
    deq = mn[..., None].astype(np.float64) + scale[..., None].astype(np.float64) * codes
    assert np.all(np.abs(deq - k) <= scale[..., None] * (0.5 + 1e-4) + 1e-6)
    jmin, jmax = np.argmin(k, axis=2), np.argmax(k, axis=2)
    assert np.all(np.take_along_axis(codes, jmin[..., None], 2) == 0)
    assert np.all(np.take_along_axis(codes, jmax[..., None], 2) == 255)
    assert len(np.unique(codes[0, 0])) >= 150          # far more than 16 levels
    _, _, sigma2 = oracle.channel_stats(codes, scale)
    np.testing.assert_allclose(sigma2, deq.var(axis=2), rtol=1e-6)
    ratio = sigma2 / (ses.sigma ** 2)                   # 8-bit noise is scale^2/12
    assert np.all((ratio > 0.9) & (ratio < 1.1))


def test_plane_layout_8bit_hand_worked():
    """Code 177 = 0b10110001 at key 0 sets slots 0, 2, 3, 7 of word 0, bit 0;
    code 66 = 0b01000010 at key 37 sets slots 1 and 6 of word 1, bit 5."""
    codes = np.zeros((1, 1, 64), np.uint8)
    codes[0, 0, 0], codes[0, 0, 37] = 177, 66
    planes = oracle.pack_planes(codes, bits=8)
    assert planes.shape == (1, 1, 8, 4)
    expect = np.zeros((8, 4), np.uint32)
    for s in (0, 2, 3, 7):
        expect[s, 0] = 1
    for s in (1, 6):
        expect[s, 1] = 1 << 5
    assert np.array_equal(planes[0, 0], expect)


@pytest.mark.parametrize("n", [1, 33, 128, 1000])
def test_planes_8bit_round_trip_and_size(n):
    rng = np.random.default_rng(n)
    codes = rng.integers(0, 256, size=(2, 3, n), dtype=np.uint8)
    planes = oracle.pack_planes(codes, bits=8)
    assert planes.shape == (2, 3, 8, oracle.n_words_for(n))
    assert np.array_equal(oracle.unpack_planes(planes, n), codes)
    assert not oracle.unpack_planes(planes, planes.shape[-1] * 32)[..., n:].any()
    # one byte per key per channel when n is a multiple of 128
    if n % 128 == 0:
        assert planes.nbytes == 2 * 3 * n


def test_coarse_bin_8bit_is_mean_of_its_fine_levels():
    mn, sc = np.float32(0.75), np.float32(0.0625)
    one = synth.f32_to_bf16_bits(np.array([1.0], np.float32))
    codes = np.arange(256, dtype=np.uint8)[None, None, :]
    planes = oracle.pack_planes(codes, bits=8)
    for t in range(9):
        s = oracle.score_planes(planes[0], np.array([mn]), np.array([sc]), one,
                                np.array([t], np.uint8), 256)
        width = 1 << (8 - t)
        for code in range(0, 256, 7):
            lo = (code // width) * width
            levels = float(mn) + float(sc) * np.arange(lo, lo + width, dtype=np.float64)
            assert s[code] == pytest.approx(levels.mean(), rel=1e-15, abs=1e-15)


def test_8bit_scores_full_zero_and_prefix_depths():
    ses = synth.make_session(21, 1, 2, 600, 300)
    ix = oracle.build_index(ses.keys, bits=8)
    assert ix["planes"].shape[-2] == 8
    deq = ix["mn"][0][:, None].astype(np.float64) + \
        ix["scale"][0][:, None].astype(np.float64) * ix["codes"][0]
    rng = np.random.default_rng(3)
    for g in range(2):
        q = ses.q_bf16[g]
        qf = synth.bf16_bits_to_f32(q).astype(np.float64)
        full = oracle.score_planes(ix["planes"][0], ix["mn"][0], ix["scale"][0], q,
                                   np.full(128, 8, np.uint8), 600)
        mag = np.abs(qf) @ np.abs(deq)
        assert np.all(np.abs(full - qf @ deq) <= 1e-13 * mag)
        zero = oracle.score_planes(ix["planes"][0], ix["mn"][0], ix["scale"][0], q,
                                   np.zeros(128, np.uint8), 600)
        const = qf @ (ix["mn"][0].astype(np.float64) + 127.5 * ix["scale"][0].astype(np.float64))
        assert np.allclose(zero, const, rtol=1e-13, atol=0)
        t = rng.integers(0, 9, size=128).astype(np.uint8)
        a = oracle.score_planes(ix["planes"][0], ix["mn"][0], ix["scale"][0], q, t, 600)
        b = oracle.score_codes(ix["codes"][0], ix["mn"][0], ix["scale"][0], q, t, bits=8)
        assert np.array_equal(a, b)


@pytest.mark.parametrize("d", [1, 2, 3])
def test_plan_8bit_is_optimal_by_brute_force(d):
    rng = np.random.default_rng(200 + d)
    allocs = np.array(list(itertools.product(range(9), repeat=d)), dtype=np.int64)
    for trial in range(5):
        w = rng.lognormal(0, 1, size=d).astype(np.float32)
        vals = allocs @ w.astype(np.float64)
        for B in range(0, 8 * d + 1):
            t = oracle.plan_greedy(w, B, bits=8)
            assert int(t.sum()) == B and t.max() <= 8
            best = vals[allocs.sum(axis=1) <= B].max()
            assert float(np.dot(w.astype(np.float64), t)) == pytest.approx(best, rel=1e-12)
    with pytest.raises(ValueError):
        oracle.plan_greedy(np.ones(d, np.float32), 8 * d + 1, bits=8)


def test_marginal_plan_8bit_is_optimal_by_brute_force():
    d = 3
    rng = np.random.default_rng(33)
    allocs = list(itertools.product(range(9), repeat=d))
    for trial in range(4):
        w = rng.lognormal(0.0, 2.0, d).astype(np.float32)
        for B in range(0, 8 * d + 1):
            t = oracle.plan_marginal(w, B, bits=8)
            assert int(t.sum()) == B and t.max() <= 8
            best = max(_distortion_drop(w, c) for c in allocs if sum(c) == B)
            assert abs(_distortion_drop(w, t) - best) <= 1e-9 * max(1.0, best)


def test_fixed_plan_8bit_reads_whole_channels():
    q = synth.make_session(0, 1, 1, 128, 16).q_bf16[0]
    for r in (0, 17, 34, 128):
        t = oracle.fixed_plan(q, r, bits=8)
        assert int(t.sum()) == 8 * r and set(np.unique(t)) <= {0, 8}
        assert np.array_equal(t > 0, oracle.fixed_plan(q, r) > 0)


def test_append_8bit_in_range_equals_repacking_and_clamps():
    first, new = _split_in_range(77, 2, 300, 45, 16)
    ix = oracle.build_index(first, capacity=345, bits=8)
    clamped = np.zeros((2, 16), np.uint32)
    oracle.append(ix, new, clamped)
    full = oracle.build_index(np.concatenate([first, new], axis=1), bits=8)
    for name in ("planes", "s1", "s2", "sigma2"):
        assert np.array_equal(ix[name], full[name]), name
    assert clamped.sum() == 0
    keys = np.arange(256, dtype=np.float32)[None, :, None]      # scale 1
    ix = oracle.build_index(keys, capacity=384, bits=8)
    clamped = np.zeros((1, 1), np.uint32)
    oracle.append(ix, np.array([[[-3.0], [300.0], [17.4]]], np.float32), clamped)
    assert list(ix["codes"][0, 0, 256:]) == [0, 255, 17] and clamped[0, 0] == 2


# ------------------------------------------- grouped per-token-block scales
# Reading: the keys of each channel are cut into blocks of block_keys tokens
# and each block is quantised on its own, as grouped quantised K caches of
# serving stacks are (the explainer's index is the serving stack's quantised
# K, 亮点 / 适用边界); sigma^2 stays the variance of all dequantised keys.
def _drifting_keys(seed, H, n, d, shift_every, shift):
    """Keys whose channel means move by `shift` every `shift_every` tokens."""
    ses = synth.make_session(seed, H, 2, n, 64, head_dim=d)
    keys = ses.keys.copy()
    keys += (np.arange(n) // shift_every)[None, :, None].astype(np.float32) * np.float32(shift)
    return ses, keys


def test_blocks_as_large_as_the_keys_are_the_global_quantiser():
    ses = synth.make_session(31, 2, 2, 3000, 64)
    g = oracle.build_index(ses.keys)
    b = oracle.build_index(ses.keys, block_keys=4096)
    assert b["mn"].shape == (2, 1, 128)
    for name in ("planes", "codes"):
        assert np.array_equal(g[name], b[name])
    for name in ("mn", "scale", "s1", "s2"):
        assert np.array_equal(g[name], b[name][:, 0]), name
    np.testing.assert_allclose(b["sigma2"], g["sigma2"], rtol=1e-6)


@pytest.mark.parametrize("bits", [4, 8])
def test_block_quantiser_error_bound_and_extremes_per_block(bits):
    """Every key is within half a step of its level, the step being its own
    block's range / (2^b - 1) (numpy min/max per block); each block's min key
    maps to level 0 and its max to the top level."""
    n, block, top = 5000, 2048, (1 << bits) - 1
    _, keys = _drifting_keys(32, 2, n, 16, 1000, 3.0)
    ix = oracle.build_index(keys, block_keys=block, bits=bits)
    for b in range(3):
        j0, j1 = b * block, min(n, (b + 1) * block)
        kb = keys[:, j0:j1].transpose(0, 2, 1).astype(np.float64)      # [H][d][nb]
        lo, hi = kb.min(axis=2), kb.max(axis=2)
        step = (hi - lo) / top
        np.testing.assert_allclose(ix["mn"][:, b], lo, rtol=0, atol=0)
        np.testing.assert_allclose(ix["scale"][:, b], step, rtol=1e-6)
        cb = ix["codes"][:, :, j0:j1]
        deq = lo[..., None] + ix["scale"][:, b][..., None].astype(np.float64) * cb
        assert np.all(np.abs(deq - kb) <= step[..., None] * (0.5 + 1e-4) + 1e-6)
        assert np.all(np.take_along_axis(cb, np.argmin(kb, 2)[..., None], 2) == 0)
        assert np.all(np.take_along_axis(cb, np.argmax(kb, 2)[..., None], 2) == top)


def _dequantised_blocked(ix, h):
    n, block = ix["n"], ix["block_keys"]
    blk = np.arange(n) // block
    mn = ix["mn"][h][blk].T.astype(np.float64)          # [d][n]
    sc = ix["scale"][h][blk].T.astype(np.float64)
    return mn + sc * ix["codes"][h]


def test_blocked_sigma2_is_the_variance_of_all_dequantised_keys():
    """Drifting means make the between-block term large: numpy's two-pass
    variance over all keys (a different algorithm) must agree."""
    _, keys = _drifting_keys(33, 2, 7000, 32, 2048, 2.5)
    ix = oracle.build_index(keys, block_keys=2048)
    for h in range(2):
        ref = _dequantised_blocked(ix, h).var(axis=1)
        np.testing.assert_allclose(ix["sigma2"][h], ref, rtol=1e-6)
    # a block's own variance alone would miss the drift
    within = ix["sigma2"][0] / _dequantised_blocked(ix, 0)[:, :2048].var(axis=1)
    assert np.median(within) > 1.5


def test_blocked_scores_full_zero_and_prefix_depths():
    ses, keys = _drifting_keys(34, 1, 5000, 128, 1500, 1.0)
    ix = oracle.build_index(keys, block_keys=2048)
    deq = _dequantised_blocked(ix, 0)
    q = ses.q_bf16[0]
    qf = synth.bf16_bits_to_f32(q).astype(np.float64)
    full = oracle.score_head(ix, 0, q, np.full(128, 4, np.uint8))
    assert np.all(np.abs(full - qf @ deq) <= 1e-13 * (np.abs(qf) @ np.abs(deq)))
    zero = oracle.score_head(ix, 0, q, np.zeros(128, np.uint8))
    blk = np.arange(5000) // 2048
    const = np.array([qf @ (ix["mn"][0, b].astype(np.float64) +
                            7.5 * ix["scale"][0, b].astype(np.float64)) for b in range(3)])
    np.testing.assert_allclose(zero, const[blk], rtol=1e-13)
    assert len(np.unique(zero)) == 3                      # one constant per block
    t = np.random.default_rng(5).integers(0, 5, size=128).astype(np.uint8)
    by_codes = np.concatenate([
        oracle.score_codes(np.ascontiguousarray(ix["codes"][0][:, j0:j0 + 2048]),
                           ix["mn"][0, b], ix["scale"][0, b], q, t)
        for b, j0 in enumerate(range(0, 5000, 2048))])
    assert np.array_equal(oracle.score_head(ix, 0, q, t), by_codes)


def test_blocked_append_of_whole_blocks_equals_packing_everything():
    _, keys = _drifting_keys(35, 2, 2048 * 3 + 500, 16, 2048, 4.0)
    ix = oracle.build_index(keys[:, :4096], capacity=keys.shape[1], block_keys=2048)
    oracle.append_blocks(ix, keys[:, 4096:])
    full = oracle.build_index(keys, capacity=keys.shape[1], block_keys=2048)
    for name in ("planes", "mn", "scale", "s1", "s2", "sigma2", "codes"):
        assert np.array_equal(ix[name], full[name]), name


def test_blocks_follow_a_drifting_key_range():
    """What the grouping is for: when the keys drift, per-block scales keep the
    quantisation error near one block's range instead of the whole range."""
    _, keys = _drifting_keys(36, 1, 8192, 32, 2048, 6.0)
    g = oracle.build_index(keys)
    b = oracle.build_index(keys, block_keys=2048)
    k = keys[0].T.astype(np.float64)
    err_g = np.abs(g["mn"][0][:, None] + g["scale"][0][:, None].astype(np.float64) * g["codes"][0] - k)
    err_b = np.abs(_dequantised_blocked(b, 0) - k)
    assert err_b.mean() < 0.5 * err_g.mean()


def test_plans_of_a_blocked_index_use_its_channel_variance():
    """The read side sees one sigma^2 per channel whatever the grouping."""
    ses, keys = _drifting_keys(37, 2, 5000, 32, 2048, 2.0)
    ix = oracle.build_index(keys, block_keys=2048)
    t, T, nb = oracle.plan_session(ix, ses.q_bf16, np.full(4, 40), 2)
    for q in range(4):
        w = oracle.importance(ses.q_bf16[q], ix["sigma2"][q // 2])
        assert np.array_equal(t[q], oracle.plan_greedy(w, 40))
    assert T.shape == (2, 32) and int(nb[0]) == 40 * oracle.n_words_for(5000) * 4


def test_absolute_scores_bound_the_scores_and_equal_them_when_no_term_is_negative():
    """A_j of a whole head (score_head with absolute=True, the scale of every
    score tolerance of the parity tests) is the sum of the absolute terms:
    it bounds |s_j| (triangle inequality), is strictly larger for keys whose
    terms differ in sign, and equals s_j bit for bit when no term is
    negative (q >= 0 and every rebuilt key >= 0: the same terms, summed in
    the same order).  Checked on a one-scale and a block-scaled index."""
    ses, keys = _drifting_keys(38, 1, 5000, 128, 2048, 1.5)
    rng = np.random.default_rng(38)
    t = rng.integers(0, 5, size=128).astype(np.uint8)
    for block in (0, 2048):
        ix = oracle.build_index(keys, block_keys=block)
        q = ses.q_bf16[0]
        s = oracle.score_head(ix, 0, q, t)
        a = oracle.score_head(ix, 0, q, t, absolute=True)
        assert a.shape == s.shape == (5000,)
        assert np.all(a >= np.abs(s))
        assert np.count_nonzero(a > np.abs(s)) > 4900        # mixed-sign q: almost every key
        # non-negative terms: |q| and keys shifted so that every channel's minimum is >= 0
        q_pos = synth.f32_to_bf16_bits(np.abs(synth.bf16_bits_to_f32(q)))
        pos = keys - keys.min(axis=1, keepdims=True)
        ixp = oracle.build_index(pos, block_keys=block)
        assert np.all(ixp["mn"] >= 0)
        assert np.array_equal(oracle.score_head(ixp, 0, q_pos, t, absolute=True),
                              oracle.score_head(ixp, 0, q_pos, t))
