"""Shared helpers of the GPU parity tests: run the oracle on the same seeded
inputs and compare with the CUDA path under the stated tolerances."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle

# Floating-point tolerance: |s_gpu - s_oracle| <= SCORE_RTOL * A_j, with
# A_j = sum_c |q_c * khat_cj| (the magnitude the fp32 sum is rounded against).
SCORE_RTOL = 1e-4


def to_np_u32(t):
    return t.cpu().numpy().view(np.uint32)


def oracle_query(ix, q_row, t_row, h, k):
    """-> (idx, top, all scores, abs sums) of one query against KV head h."""
    s = oracle.score_head(ix, h, q_row, t_row)
    a = oracle.score_head(ix, h, q_row, t_row, absolute=True)
    idx, top = oracle.topk(s, k)
    return idx, top, s, a


def check_topk(gpu_idx, gpu_score, s, a, k, rtol=SCORE_RTOL):
    """Parity of one query's top-k.

    * indices valid, unique, exactly k of them;
    * every returned score within rtol * A_j of the oracle's score of that key;
    * the set equals the oracle's top-k except for keys whose oracle score is
      within rtol * A of the oracle's k-th score (both sides, equal size);
    * order: ascending key index.
    Returns the number of keys that differ (inside the tie band)."""
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    gpu_score = np.asarray(gpu_score, dtype=np.float64)
    n = s.shape[0]
    assert gpu_idx.shape == (k,)
    assert np.all((gpu_idx >= 0) & (gpu_idx < n)), "index out of range"
    assert len(np.unique(gpu_idx)) == k, "duplicate index"
    err = np.abs(gpu_score - s[gpu_idx])
    bad = err > rtol * a[gpu_idx] + 1e-30
    assert not bad.any(), (f"score mismatch at {gpu_idx[bad][:5]}: gpu {gpu_score[bad][:5]} "
                           f"oracle {s[gpu_idx][bad][:5]} tol {rtol * a[gpu_idx][bad][:5]}")
    ref_idx, ref_top = oracle.topk(s, k)
    kth = ref_top[-1]
    got, ref = set(gpu_idx.tolist()), set(ref_idx.tolist())
    diff = got ^ ref
    for j in diff:
        band = rtol * max(a[j], a[ref_idx[-1]])
        assert abs(s[j] - kth) <= band, (f"key {j} (oracle score {s[j]}) differs from the "
                                         f"oracle top-{k} outside the tie band (k-th {kth})")
    assert np.all(np.diff(gpu_idx) > 0), "indices not in ascending order"
    return len(diff) // 2


def check_queries(ix, q_bf16, t, group, k, gpu_idx, gpu_score, queries, heads=None):
    """check_topk for each query row in `queries` against oracle index `ix`,
    the oracle runs on all host cores at once (its C calls release the GIL).
    heads: KV head of each query in `ix` (default qq // group)."""
    def one(i):
        qq = queries[i]
        h = qq // group if heads is None else heads[i]
        _, _, s, a = oracle_query(ix, q_bf16[qq], t[qq], h, k)
        return check_topk(gpu_idx[qq], gpu_score[qq], s, a, k)
    with ThreadPoolExecutor(max_workers=min(len(queries), os.cpu_count() or 1)) as ex:
        return list(ex.map(one, range(len(queries))))
