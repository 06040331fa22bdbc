"""The parity checker of the GPU tests (tests/helpers.check_topk) on the CPU:
it must accept the oracle's own top-k, listed in ascending key index, and a
result that differs only inside the tie band; and it must reject each
plausible mistake of a GPU result (a key from outside the band, a score off
by more than the tolerance, a duplicate, an index out of range, a missing
entry, the wrong order)."""
import numpy as np
import pytest

import oracle
import synth
from tests.helpers import SCORE_RTOL, check_topk, oracle_query

K = 64


def _case():
    """One query of the tiny workload against its index: the oracle's scores
    s, absolute sums a and top-k listed by ascending index."""
    ses = synth.tiny_4k()
    ix = oracle.build_index(ses.keys)
    t, _, _ = oracle.plan_session(ix, ses.q_bf16, ses.budgets, 1)
    idx, _, s, a = oracle_query(ix, ses.q_bf16[0], t[0], 0, K)
    order = np.argsort(idx)
    return s, a, idx[order].astype(np.int64), s[idx[order]]


def test_accepts_the_oracle_result():
    s, a, idx, sc = _case()
    assert check_topk(idx, sc.astype(np.float32), s, a, K) == 0


def test_accepts_scores_inside_the_tolerance():
    s, a, idx, sc = _case()
    assert check_topk(idx, sc + 0.5 * SCORE_RTOL * a[idx], s, a, K) == 0


def test_rejects_a_score_outside_the_tolerance():
    s, a, idx, sc = _case()
    bad = sc.copy()
    bad[K // 2] += 2.0 * SCORE_RTOL * a[idx[K // 2]]
    with pytest.raises(AssertionError, match="score mismatch"):
        check_topk(idx, bad, s, a, K)


def test_rejects_a_key_from_outside_the_tie_band():
    s, a, idx, sc = _case()
    ref_idx, ref_top = oracle.topk(s, K)
    # the best key below the top-k that is clearly below the k-th score
    below = np.argsort(-s, kind="stable")[K:]
    far = [j for j in below if ref_top[-1] - s[j] > 10 * SCORE_RTOL * max(a[j], a[ref_idx[-1]])]
    j = int(far[0])
    got = np.sort(np.concatenate([np.setdiff1d(idx, [ref_idx[-1]]), [j]]))
    with pytest.raises(AssertionError, match="outside the tie band"):
        check_topk(got, s[got], s, a, K)


def test_accepts_a_swap_inside_the_tie_band():
    s, a, idx, sc = _case()
    ref_idx, _ = oracle.topk(s, K)
    kth = int(ref_idx[-1])
    outside = np.setdiff1d(np.arange(s.shape[0]), idx)
    j = int(outside[0])
    s2 = s.copy()
    s2[j] = s[kth]                           # an exact tie with the k-th key
    a2 = a.copy()
    a2[j] = a[kth]
    # the oracle keeps the lower index of the tie; a result holding the other
    # key differs from it only inside the band
    ref2, _ = oracle.topk(s2, K)
    dropped = kth if j < kth else j
    assert dropped not in set(ref2.tolist())
    kept = j if dropped == kth else kth
    got = np.sort(np.concatenate([np.setdiff1d(ref2, [kept]), [dropped]]))
    assert check_topk(got, s2[got], s2, a2, K) == 1


def test_rejects_duplicates_range_size_and_order():
    s, a, idx, sc = _case()
    dup = idx.copy()
    dup[1] = dup[0]
    with pytest.raises(AssertionError, match="duplicate"):
        check_topk(dup, s[dup], s, a, K)
    out = idx.copy()
    out[-1] = s.shape[0]
    with pytest.raises(AssertionError, match="out of range"):
        check_topk(out, np.append(sc[:-1], 0.0), s, a, K)
    with pytest.raises(AssertionError):
        check_topk(idx[:-1], sc[:-1], s, a, K)
    rev = idx[::-1].copy()
    with pytest.raises(AssertionError, match="ascending"):
        check_topk(rev, s[rev], s, a, K)
