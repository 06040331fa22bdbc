"""Scans of more than 2^20 keys per KV head (the index-order bitmap of the
final select covers at most 2^20 keys; past it the selected keys are put in
index order by a sort): the fast path against the forced exact path and the
oracle, on a fresh index of 2^20 + 32 keys and on a 2^20-key index that one
decode-step append takes past the limit."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import oracle
import synth
from tests.helpers import check_topk, oracle_query
from tests.test_parity_gpu import gpu_index, run_plan

pytestmark = pytest.mark.gpu

N_BIG = (1 << 20) + 32


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp.load_library()
    torch.cuda.set_device(0)
    fp.fathom_last_device_status()


def _scan_both(ix, ses, budgets, k):
    """-> plan, then (idx, score) of the default and of the forced exact path."""
    q, t, tu, _ = run_plan(ix, ses, budgets)
    out = []
    for flags in (0, fp.FATHOM_SCAN_FORCE_EXACT):
        buf = fp.ScanBuffers(ix, k)
        fp.fathom_scan_topk(ix.desc, q, t, tu, k, buf.idx, buf.score, buf.workspace, flags)
        torch.cuda.synchronize()
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        out.append((buf.idx.cpu().numpy(), buf.score.cpu().numpy()))
    return t.cpu().numpy(), out


def _check(ref, ses, t, out, k, n):
    for qq in range(ses.q_bf16.shape[0]):
        _, _, s, a = oracle_query(ref, ses.q_bf16[qq], t[qq], qq // ses.group, k)
        for idx, score in out:
            assert idx[qq].max() < n
            check_topk(idx[qq], score[qq], s, a, k)


def test_scan_past_a_million_keys():
    ses = synth.make_session(71, 1, 2, N_BIG, [68, 136])
    # the last 8 keys point along query 0, so its top-k holds keys past 2^20
    q0 = ses.q_bf16[0].astype(np.uint32) << 16
    ses.keys[0, -8:] = 3.0 * q0.view(np.float32)[None, :]
    ix = gpu_index(ses)
    ref = oracle.build_index(ses.keys)
    t, out = _scan_both(ix, ses, ses.budgets, 2048)
    _check(ref, ses, t, out, 2048, N_BIG)
    for idx, _ in out:
        assert np.count_nonzero(idx[0] >= (1 << 20)) >= 8


def test_append_takes_a_million_key_index_past_the_limit():
    n = 1 << 20
    ses = synth.make_session(72, 1, 2, n + 1, [92, 18])
    ix = fp.KeyIndex(1, 2, n, 128, "device", capacity=n + 1)
    ix.pack(torch.from_numpy(np.ascontiguousarray(ses.keys[:, :n])).cuda())
    ref = oracle.build_index(ses.keys[:, :n], capacity=n + 1)
    new = np.ascontiguousarray(ses.keys[:, n:])
    ix.append(torch.from_numpy(new).cuda())
    oracle.append(ref, new)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    assert ix.n_keys == n + 1
    t, out = _scan_both(ix, ses, ses.budgets, 2048)
    _check(ref, ses, t, out, 2048, n + 1)
