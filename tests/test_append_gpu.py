"""Append path on the GPU vs the oracle through the C ABI: decode-step keys
quantised with the stored scales, planes, sums, sigma^2 and clamp counters
bit-exact after every append; the scan then finds the new keys."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import oracle
import synth
from tests.helpers import check_topk, oracle_query
from tests.test_parity_gpu import check_pack, run_plan, run_scan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp.load_library()
    torch.cuda.set_device(0)
    fp.fathom_last_device_status()


def _grow(seed, H, G, n, d, chunks, residency, scale_new=1.0):
    """Pack n keys with room for the chunks, append them one call per chunk
    on the GPU and in the oracle; compare after every call."""
    total = n + sum(chunks)
    ses = synth.make_session(seed, H, G, total, 64, head_dim=d)
    keys = ses.keys.copy()
    keys[:, n:] *= scale_new                         # > 1: some keys leave the range
    ix = fp.KeyIndex(H, G, n, d, residency, capacity=total)
    ix.pack(torch.from_numpy(np.ascontiguousarray(keys[:, :n])).cuda())
    ref = oracle.build_index(keys[:, :n], capacity=total)
    cl_gpu = torch.zeros((H, d), dtype=torch.int32, device="cuda")
    cl_ref = np.zeros((H, d), np.uint32)
    at = n
    for m in chunks:
        new = np.ascontiguousarray(keys[:, at:at + m])
        ix.append(torch.from_numpy(new).cuda(), cl_gpu)
        oracle.append(ref, new, cl_ref)
        at += m
        torch.cuda.synchronize()
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        assert ix.n_keys == at
        check_pack(ix, ref)
        assert np.array_equal(cl_gpu.cpu().numpy().view(np.uint32), cl_ref)
    return ses, keys, ix, ref, cl_ref


@pytest.mark.parametrize("residency", ["device", "host_mapped"])
def test_append_decode_steps_bit_exact(residency):
    """One key per step across word boundaries, then a ragged chunk."""
    _grow(3, 2, 4, 1000, 128, [1] * 30 + [37, 100, 1], residency)


def test_append_out_of_range_keys_are_clamped_and_counted():
    *_, clamped = _grow(4, 2, 1, 3000, 64, [1, 5, 500], "device", scale_new=1.8)
    assert clamped.sum() > 0


def test_append_in_range_gives_the_packed_index():
    ses = synth.make_session(5, 2, 4, 6000, 64)
    lo = ses.keys[:, :5000].min(axis=1, keepdims=True)
    hi = ses.keys[:, :5000].max(axis=1, keepdims=True)
    keys = ses.keys.copy()
    keys[:, 5000:] = np.clip(keys[:, 5000:], lo, hi)
    ix = fp.KeyIndex(2, 4, 5000, 128, "device", capacity=6000)
    ix.pack(torch.from_numpy(np.ascontiguousarray(keys[:, :5000])).cuda())
    ix.append(torch.from_numpy(np.ascontiguousarray(keys[:, 5000:])).cuda())
    torch.cuda.synchronize()
    check_pack(ix, oracle.build_index(keys, capacity=6000))


def test_scan_after_appends_finds_the_new_keys():
    """Keys appended next to the first query head's direction rank on top."""
    H, G, n, d = 2, 4, 20000, 128
    ses = synth.make_session(6, H, G, n + 64, 92)
    keys = ses.keys.copy()
    q0 = synth.bf16_bits_to_f32(ses.q_bf16[0]).astype(np.float32)
    rng = np.random.default_rng(0)
    keys[0, n:n + 16] = q0[None, :] * 3.0 + rng.normal(0, 0.1, (16, d)).astype(np.float32)
    ses_all = synth.Session(seed=6, n_kv_heads=H, group=G, n_keys=n + 64, head_dim=d,
                            sigma=ses.sigma, outliers=ses.outliers, keys=keys,
                            q_bf16=ses.q_bf16, budgets=ses.budgets)
    ix = fp.KeyIndex(H, G, n, d, "device", capacity=n + 64)
    ix.pack(torch.from_numpy(np.ascontiguousarray(keys[:, :n])).cuda())
    for i in range(64):
        ix.append(torch.from_numpy(np.ascontiguousarray(keys[:, n + i:n + i + 1])).cuda())
    ref = oracle.build_index(keys[:, :n], capacity=n + 64)
    oracle.append(ref, np.ascontiguousarray(keys[:, n:]))
    check_pack(ix, ref)
    q, t, tu, _ = run_plan(ix, ses_all, ses_all.budgets)
    k = 256
    oi, os_ = run_scan(ix, ses_all, q, t, tu, k)
    tt = t.cpu().numpy()
    for qq in range(H * G):
        _, _, s, a = oracle_query(ref, ses.q_bf16[qq], tt[qq], qq // G, k)
        check_topk(oi[qq], os_[qq], s, a, k)
    assert len(set(range(n, n + 16)) & set(oi[0].tolist())) >= 12


def test_append_nonfinite_key_sets_status():
    ses = synth.make_session(7, 1, 1, 300, 16)
    ix = fp.KeyIndex(1, 1, 200, 128, "device", capacity=300)
    ix.pack(torch.from_numpy(np.ascontiguousarray(ses.keys[:, :200])).cuda())
    bad = np.ascontiguousarray(ses.keys[:, 200:201]).copy()
    bad[0, 0, 5] = np.nan
    ix.append(torch.from_numpy(bad).cuda())
    assert fp.fathom_last_device_status() == fp.FATHOM_ERR_NONFINITE
