"""fathom_scan_topk_static: the scan + top-k for callers that cannot
allocate device memory (a plugin inside an engine whose pool owns the free
HBM, or a decode loop that must not call cudaMalloc).  It runs on the
library's fixed per-GPU scratch array instead of a caller workspace; its
results must match fathom_scan_topk's on the same inputs, call after call,
since every call reuses the same scratch.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import synth

pytestmark = pytest.mark.gpu

SCORE_RTOL = 1e-4   # the tolerance of the parity tests


def _prepare(seed, budgets, n=20000, H=8, G=4, residency="device"):
    ses = synth.make_session(seed, H, G, n, budgets)
    ix = fp.KeyIndex(H, G, n, 128, residency)
    ix.pack(torch.from_numpy(ses.keys).cuda())
    q = torch.from_numpy(ses.q_bf16.view(np.int16)).cuda()
    b = torch.from_numpy(ses.budgets).cuda()
    t = torch.empty((H * G, 128), dtype=torch.uint8, device="cuda")
    tu = torch.empty((H, 128), dtype=torch.uint8, device="cuda")
    nb = torch.empty(H * G + H, dtype=torch.int64, device="cuda")
    fp.fathom_plan(ix.desc, q, b, t, tu, nb)
    return ix, q, t, tu


def _outputs(Q, k):
    return (torch.full((Q, k), -1, dtype=torch.int32, device="cuda"),
            torch.full((Q, k), float("nan"), dtype=torch.float32, device="cuda"))


def _assert_same(idx_a, sc_a, idx_b, sc_b):
    idx_a, idx_b = idx_a.cpu().numpy(), idx_b.cpu().numpy()
    sc_a, sc_b = sc_a.cpu().numpy().astype(np.float64), sc_b.cpu().numpy().astype(np.float64)
    for qq in range(idx_a.shape[0]):
        assert set(idx_a[qq].tolist()) == set(idx_b[qq].tolist()), f"query {qq}: sets differ"
    scale = np.maximum(np.abs(sc_b), 1.0)
    assert np.all(np.abs(sc_a - sc_b) <= SCORE_RTOL * scale)
    assert np.array_equal(idx_a, idx_b)


def test_static_scratch_matches_workspace_call_twice_in_a_row():
    torch.cuda.set_device(0)
    fp.load_library()
    k = 256
    calls = [(_prepare(301, np.tile([68, 92, 136, 18], 8)), 0),
             (_prepare(302, np.tile([136, 18, 92, 68], 8)), fp.FATHOM_SCAN_FORCE_EXACT),
             # a small host-resident index: its two-head plane ring fits the scratch too
             (_prepare(303, np.tile([18, 136, 68, 92], 8), residency="host_mapped"), 0)]
    for (ix, q, t, tu), flags in calls:
        Q = ix.n_kv_heads * ix.group
        ref_i, ref_s = _outputs(Q, k)
        ws = torch.empty(fp.fathom_scan_workspace_bytes(ix.desc, k), dtype=torch.uint8,
                         device="cuda")
        fp.fathom_scan_topk(ix.desc, q, t, tu, k, ref_i, ref_s, ws, flags)
        got_i, got_s = _outputs(Q, k)
        fp.fathom_scan_topk_static(ix.desc, q, t, tu, k, got_i, got_s, flags)
        torch.cuda.synchronize()
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        _assert_same(got_i, got_s, ref_i, ref_s)


def test_static_scratch_rejects_problems_beyond_its_size():
    fp.load_library()
    n = 1 << 20
    fake = 0x10000    # never dereferenced: the size check comes first
    big = fp.fathom_index(16, 8, 128, n, fp.fathom_n_words(n), 0, fake, fake, fake, fake,
                          fake, fake)
    assert fp.fathom_scan_workspace_bytes(big, 2048) > 8 << 20
    rc = fp.load_library().fathom_scan_topk_static(ctypes.byref(big), fake, fake, fake, 2048,
                                                   fake, fake, 0, 0)
    assert rc == fp.FATHOM_ERR_WORKSPACE
