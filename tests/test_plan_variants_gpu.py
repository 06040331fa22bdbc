"""Marginal-gain plan on the GPU vs the oracle: plans, unions and byte
counts bit-exact; the scan runs unchanged on its plans."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import oracle
import synth
from tests.test_parity_gpu import check_scan, gpu_index, run_scan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp.load_library()
    torch.cuda.set_device(0)
    fp.fathom_last_device_status()


def run_marginal(ix, ses, budgets):
    H, G, d = ses.n_kv_heads, ses.group, ses.head_dim
    Q = H * G
    q = torch.from_numpy(ses.q_bf16.view(np.int16)).cuda()
    b = torch.from_numpy(np.asarray(budgets, np.int32)).cuda()
    t = torch.empty((Q, d), dtype=torch.uint8, device="cuda")
    tu = torch.empty((H, d), dtype=torch.uint8, device="cuda")
    nb = torch.empty(Q + H, dtype=torch.int64, device="cuda")
    fp.fathom_plan_marginal(ix.desc, q, b, t, tu, nb)
    torch.cuda.synchronize()
    return q, t, tu, nb


@pytest.mark.parametrize("d,G", [(32, 1), (64, 4), (96, 3), (128, 4), (128, 8), (256, 2)])
def test_marginal_plan_bit_exact(d, G):
    H = 3
    rng = np.random.default_rng(d + G)
    budgets = rng.integers(0, 4 * d + 1, H * G).astype(np.int32)
    budgets[0], budgets[-1] = 0, 4 * d
    ses = synth.make_session(300 + d + G, H, G, 2000, budgets, head_dim=d)
    ix = gpu_index(ses)
    ref = oracle.build_index(ses.keys)
    _, t, tu, nb = run_marginal(ix, ses, budgets)
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    rt, rT, rnb = oracle.plan_session(ref, ses.q_bf16, budgets, G, marginal=True)
    assert np.array_equal(t.cpu().numpy(), rt)
    assert np.array_equal(tu.cpu().numpy(), rT)
    assert np.array_equal(nb.cpu().numpy().astype(np.uint64), rnb)
    assert np.array_equal(t.cpu().numpy().astype(np.int64).sum(axis=1), budgets)


def test_marginal_plan_budget_out_of_range_sets_status():
    ses = synth.make_session(5, 1, 2, 500, 64)
    ix = gpu_index(ses)
    _, t, _, _ = run_marginal(ix, ses, [64, 4 * 128 + 1])
    assert fp.fathom_last_device_status() == fp.FATHOM_ERR_INVALID_ARG
    assert int(t[1].sum()) == 0 and int(t[0].sum()) == 64


def test_scan_with_marginal_plans():
    budgets = np.tile(np.array([18, 68, 92, 137], np.int32), 2)
    ses = synth.make_session(11, 2, 4, 15000, budgets)
    ix = gpu_index(ses)
    ref = oracle.build_index(ses.keys)
    q, t, tu, _ = run_marginal(ix, ses, budgets)
    oi, os_ = run_scan(ix, ses, q, t, tu, 400)
    check_scan(ses, ref, t, oi, os_, 400)
