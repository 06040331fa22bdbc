"""One KV head's keys split into shards: scanning word-range shards of one
packed index and merging their top-k lists through the C ABI reproduces
the whole-index scan bit for bit; the merge matches the oracle's."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import oracle
import synth
from tests.test_parity_gpu import gpu_index, run_plan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp.load_library()
    torch.cuda.set_device(0)
    fp.fathom_last_device_status()


def shard_index(ix, key0, key1):
    """Descriptor of keys [key0, key1) of a packed index (key0 a multiple of
    128): its own copy of that word range of the planes, the whole index's
    statistics."""
    w0 = key0 // 32
    n = key1 - key0
    nw = fp.fathom_n_words(n)
    planes = ix.planes[:, :, :, w0:w0 + nw].contiguous()
    d = ix.desc
    desc = fp.fathom_index(d.n_kv_heads, d.group, d.head_dim, n, nw, 0, planes.data_ptr(),
                           d.mn, d.scale, d.sigma2, d.sum_code, d.sum_code2)
    return desc, planes


def scan(desc, q, t, tu, k, Q):
    oi = torch.full((Q, k), -1, dtype=torch.int32, device="cuda")
    os_ = torch.full((Q, k), np.nan, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(16, fp.fathom_scan_workspace_bytes(desc, k)), dtype=torch.uint8,
                     device="cuda")
    fp.fathom_scan_topk(desc, q, t, tu, k, oi, os_, ws)
    return oi, os_


@pytest.mark.parametrize("bounds,k", [([0, 12800, 25600, 40000], 512), ([0, 20096, 40000], 64),
                                      ([0, 4096, 8192, 12288, 40000], 1000)])
def test_sharded_scan_and_merge_equal_the_whole_scan(bounds, k):
    H, G, n = 2, 4, 40000
    budgets = np.tile(np.array([68, 92, 136, 18], np.int32), H)
    ses = synth.make_session(500 + k, H, G, n, budgets)
    ix = gpu_index(ses)
    q, t, tu, _ = run_plan(ix, ses, ses.budgets)
    Q = H * G
    whole_i, whole_s = scan(ix.desc, q, t, tu, k, Q)
    lists_i, lists_s, keep = [], [], []
    for a, b in zip(bounds, bounds[1:]):
        desc, planes = shard_index(ix, a, b)
        oi, os_ = scan(desc, q, t, tu, k, Q)
        lists_i.append(oi)
        lists_s.append(os_)
        keep.append(planes)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    mi = torch.empty((Q, k), dtype=torch.int32, device="cuda")
    ms = torch.empty((Q, k), dtype=torch.float32, device="cuda")
    fp.fathom_merge_topk(torch.stack(lists_i), torch.stack(lists_s), bounds[:-1], k, mi, ms)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    assert np.array_equal(mi.cpu().numpy(), whole_i.cpu().numpy())
    assert np.array_equal(ms.cpu().numpy().view(np.uint32), whole_s.cpu().numpy().view(np.uint32))


def test_merge_matches_the_oracle_with_ties():
    S, Q, k_s, k = 4, 6, 300, 500
    rng = np.random.default_rng(3)
    offsets = np.array([0, 1000, 1700, 5000])
    idx = np.stack([np.stack([np.sort(rng.choice(600, k_s, replace=False)) for _ in range(Q)])
                    for _ in range(S)]).astype(np.int32)
    score = np.round(rng.standard_normal((S, Q, k_s)), 1).astype(np.float32)   # many ties
    mi = torch.empty((Q, k), dtype=torch.int32, device="cuda")
    ms = torch.empty((Q, k), dtype=torch.float32, device="cuda")
    fp.fathom_merge_topk(torch.from_numpy(idx).cuda(), torch.from_numpy(score).cuda(), offsets,
                         k, mi, ms)
    torch.cuda.synchronize()
    for qq in range(Q):
        ri, rs = oracle.merge_topk(idx[:, qq], score[:, qq].astype(np.float64), offsets, k)
        assert np.array_equal(mi[qq].cpu().numpy(), ri)
        assert np.array_equal(ms[qq].cpu().numpy(), rs.astype(np.float32))
