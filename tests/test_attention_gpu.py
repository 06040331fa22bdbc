"""Attention over the selected keys on the GPU vs the fp64 oracle through
the C ABI: every head_dim load path, split boundaries, dense (k = n),
host-resident K/V, bad indices, and the scan -> attention chain."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import oracle
import synth
from tests.test_parity_gpu import gpu_index, run_plan, run_scan

pytestmark = pytest.mark.gpu

# fp32 softmax-weighted sums of <= 4096 rows against fp64: relative L2 error
# of the output vector, and per coordinate c an error of at most
# ATTN_COORD_RTOL * sum_i p_i |V_ic| (the magnitude the fp32 sum of that
# coordinate is rounded against; the weights' own fp32 error enters as a
# relative error of each p_i)
ATTN_RTOL = 2e-5
ATTN_COORD_RTOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp.load_library()
    torch.cuda.set_device(0)
    fp.fathom_last_device_status()


def _values(seed, H, n, d):
    return np.random.default_rng(seed).standard_normal((H, n, d)).astype(np.float32)


def run_attention(keys, values, H, G, d, n, q, idx, k, scale, residency="device"):
    Q = H * G
    if residency == "device":
        kt, vt = torch.from_numpy(keys).cuda(), torch.from_numpy(values).cuda()
    else:
        kt, vt = torch.from_numpy(keys).pin_memory(), torch.from_numpy(values).pin_memory()
    qt = torch.from_numpy(np.ascontiguousarray(q).view(np.int16)).cuda()
    it = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
    out = torch.full((Q, d), np.nan, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(16, fp.fathom_sparse_attention_workspace_bytes(Q, d, k)),
                     dtype=torch.uint8, device="cuda")
    fp.fathom_sparse_attention(kt, vt, H, G, d, n, qt, it, k, scale, out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def coordinate_scale(keys_h, values_h, q_row, idx, scale):
    """sum_i p_i |V_ic| per coordinate c, with p the softmax weights of the
    selected rows (fp64; the tolerance's scale, not an expected value)."""
    qf = (np.asarray(q_row, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rows = np.asarray(idx, np.int64)
    logits = scale * (keys_h[rows].astype(np.float64) @ qf)
    p = np.exp(logits - logits.max())
    p /= p.sum()
    return p @ np.abs(values_h[rows].astype(np.float64))


def check_against_oracle(keys, values, q, idx, out, G, scale):
    for qq in range(out.shape[0]):
        h = qq // G
        ref = oracle.attention(keys[h], values[h], q[qq], idx[qq], scale)
        assert oracle.attention_error(out[qq], ref) < ATTN_RTOL, qq
        bound = ATTN_COORD_RTOL * coordinate_scale(keys[h], values[h], q[qq], idx[qq], scale)
        err = np.abs(out[qq].astype(np.float64) - ref)
        assert np.all(err <= bound + 1e-12), (qq, np.argmax(err - bound))


@pytest.mark.parametrize("d,k,G", [(128, 300, 4), (32, 1, 1), (64, 128, 2), (96, 129, 3),
                                   (192, 255, 4), (256, 1000, 8), (128, 4096, 4)])
def test_attention_matches_oracle(d, k, G):
    H, n = 2, 5000
    ses = synth.make_session(200 + d + k, H, G, n, 64, head_dim=d)
    values = _values(d + k, H, n, d)
    rng = np.random.default_rng(k)
    idx = np.stack([np.sort(rng.choice(n, k, replace=False)) for _ in range(H * G)])
    scale = 1.0 / np.sqrt(d)
    out = run_attention(ses.keys, values, H, G, d, n, ses.q_bf16, idx, k, scale)
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    check_against_oracle(ses.keys, values, ses.q_bf16, idx, out, G, scale)


def test_attention_over_all_keys_is_dense_attention():
    H, G, n, d = 1, 2, 777, 128
    ses = synth.make_session(7, H, G, n, 64)
    values = _values(7, H, n, d)
    idx = np.tile(np.arange(n, dtype=np.int32), (H * G, 1))
    out = run_attention(ses.keys, values, H, G, d, n, ses.q_bf16, idx, n, 0.088)
    for qq in range(H * G):
        dense = oracle.attention(ses.keys[0], values[0], ses.q_bf16[qq], None, 0.088)
        assert oracle.attention_error(out[qq], dense) < ATTN_RTOL
    check_against_oracle(ses.keys, values, ses.q_bf16, idx, out, G, 0.088)


def test_attention_host_resident_kv():
    H, G, n, d, k = 2, 4, 3000, 128, 512
    ses = synth.make_session(8, H, G, n, 64)
    values = _values(8, H, n, d)
    rng = np.random.default_rng(1)
    idx = np.stack([rng.choice(n, k, replace=False) for _ in range(H * G)]).astype(np.int32)
    out = run_attention(ses.keys, values, H, G, d, n, ses.q_bf16, idx, k, 0.1, "host_mapped")
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    check_against_oracle(ses.keys, values, ses.q_bf16, idx, out, G, 0.1)


def test_attention_bad_index_sets_status_and_is_skipped():
    H, G, n, d, k = 1, 1, 100, 32, 4
    ses = synth.make_session(9, H, G, n, 64, head_dim=d)
    values = _values(9, H, n, d)
    idx = np.array([[3, 100, 7, -1]], np.int32)
    out = run_attention(ses.keys, values, H, G, d, n, ses.q_bf16, idx, k, 0.2)
    assert fp.fathom_last_device_status() == fp.FATHOM_ERR_INVALID_ARG
    ref = oracle.attention(ses.keys[0], values[0], ses.q_bf16[0], np.array([3, 7]), 0.2)
    assert oracle.attention_error(out[0], ref) < ATTN_RTOL
    check_against_oracle(ses.keys, values, ses.q_bf16, np.array([[3, 7]]), out, G, 0.2)


def test_scan_then_attention_chain():
    """The scan's top-k feeds the attention directly (device pointers)."""
    H, G, n, d, k = 2, 4, 20000, 128, 1024
    ses = synth.make_session(10, H, G, n, 136)
    ix = gpu_index(ses)
    q, t, tu, _ = run_plan(ix, ses, ses.budgets)
    oi, _ = run_scan(ix, ses, q, t, tu, k)
    values = _values(10, H, n, d)
    out = run_attention(ses.keys, values, H, G, d, n, ses.q_bf16, oi, k, 1 / np.sqrt(d))
    check_against_oracle(ses.keys, values, ses.q_bf16, oi, out, G, 1 / np.sqrt(d))
