"""Parity at the full benchmark sizes, in the launch configuration the
benchmark times, on sampled queries the oracle scores one by one.

* Qwen3-8B-shaped layer, HBM-resident: 8 KV heads x 4 query heads,
  head_dim 128, 131072 keys, B in {68, 92, 136}, k = 2048.
* The same layer as an 8-plane index (8-bit K cache) and with grouped
  per-token-block scales (2048-token blocks), as the benchmark's
  qwen3_8b_layer_128k_8plane and qwen3_8b_layer_128k_blocked workloads.
* Million-token host-resident scan, 2 of the 8 KV heads (the oracle's cost
  grows with the heads checked; the kernel's per-head work is the same),
  1,048,576 keys, B in {18, 92}, k = 2048."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import oracle
import synth
from tests.helpers import check_topk, oracle_query
from tests.test_parity_gpu import check_pack, gpu_index, run_plan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer():
    ses = synth.qwen3_8b_layer(131072, 92)
    return ses, gpu_index(ses), oracle.build_index(ses.keys)


def _scan(ix, ses, budgets, k, flags=0):
    q, t, tu, nb = run_plan(ix, ses, budgets)
    buf = fp.ScanBuffers(ix, k)
    fp.fathom_scan_topk(ix.desc, q, t, tu, k, buf.idx, buf.score, buf.workspace, flags)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    return t.cpu().numpy(), nb.cpu().numpy(), buf.idx.cpu().numpy(), buf.score.cpu().numpy()


def test_layer_pack_bit_exact(layer):
    ses, ix, ref = layer
    check_pack(ix, ref)


@pytest.mark.parametrize("B", [68, 92, 136])
def test_layer_scan_sampled_queries(layer, B):
    ses, ix, ref = layer
    budgets = np.full(32, B, np.int32)
    t, nb, oi, os_ = _scan(ix, ses, budgets, 2048)
    rt, rT, rnb = oracle.plan_session(ref, ses.q_bf16, budgets, 4)
    assert np.array_equal(t, rt)
    assert np.array_equal(nb.astype(np.uint64), rnb)
    assert np.all(nb[:32] == B * 131072 // 8)
    for qq in (0, 13, 31):
        _, _, s, a = oracle_query(ref, ses.q_bf16[qq], t[qq], qq // 4, 2048)
        check_topk(oi[qq], os_[qq], s, a, 2048)


def _variant_index(ses, **kw):
    ix = fp.KeyIndex(ses.n_kv_heads, ses.group, ses.n_keys, ses.head_dim, **kw)
    ix.pack(torch.from_numpy(ses.keys).cuda())
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    return ix


@pytest.mark.parametrize("variant", ["8plane", "blocked"])
def test_layer_variants_pack_plans_and_sampled_queries(layer, variant):
    ses, _, _ = layer
    kw = dict(bits=8) if variant == "8plane" else dict(block_keys=2048)
    ix = _variant_index(ses, **kw)
    ref = oracle.build_index(ses.keys, **kw)
    nbf = oracle.n_blocks_for(131072, 2048) if variant == "blocked" else None
    planes = ix.planes.cpu().numpy().view(np.uint32)
    assert np.array_equal(planes, ref["planes"])
    for name, got in (("mn", ix.mn), ("scale", ix.scale), ("s1", ix.sum_code),
                      ("s2", ix.sum_code2)):
        g = got.cpu().numpy()
        r = ref[name]
        if nbf:
            g, r = g[:, :nbf], r[:, :nbf]
        assert np.array_equal(np.ascontiguousarray(g).view(np.uint8),
                              np.ascontiguousarray(r).view(np.uint8)), name
    assert np.array_equal(ix.sigma2.cpu().numpy().view(np.uint32), ref["sigma2"].view(np.uint32))
    for B in (68, 136):
        budgets = np.full(32, B, np.int32)
        t, nb, oi, os_ = _scan(ix, ses, budgets, 2048)
        rt, rT, rnb = oracle.plan_session(ref, ses.q_bf16, budgets, 4)
        assert np.array_equal(t, rt)
        assert np.array_equal(nb.astype(np.uint64), rnb)
        for qq in (0, 31):
            _, _, s, a = oracle_query(ref, ses.q_bf16[qq], t[qq], qq // 4, 2048)
            check_topk(oi[qq], os_[qq], s, a, 2048)


@pytest.mark.slow
def test_host_million_token_heads():
    ses = synth.make_session(0, 2, 4, 1 << 20, [18, 92, 92, 18, 92, 18, 18, 92])
    ix = gpu_index(ses, "host_mapped")
    ref = oracle.build_index(ses.keys)
    t, nb, oi, os_ = _scan(ix, ses, ses.budgets, 2048)
    for qq in (0, 5):
        _, _, s, a = oracle_query(ref, ses.q_bf16[qq], t[qq], qq // 4, 2048)
        check_topk(oi[qq], os_[qq], s, a, 2048)
