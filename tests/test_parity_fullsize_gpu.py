"""Parity at the full benchmark sizes, in the launch configuration the
benchmark times, on every query head (the oracle scores them on all host
cores at once).

* Qwen3-8B-shaped layer, HBM-resident: 8 KV heads x 4 query heads,
  head_dim 128, 131072 keys, B in {68, 92, 136}, k = 2048.
* The same layer as an 8-plane index (8-bit K cache) and with grouped
  per-token-block scales (2048-token blocks), as the benchmark's
  qwen3_8b_layer_128k_8plane and qwen3_8b_layer_128k_blocked workloads.
* Million-token host-resident layer, all 8 KV heads x 4 query heads,
  1,048,576 keys, the four budgets 18 / 68 / 92 / 136 on each head's four
  query heads, and the fixed 136-bit (top 34 channels) and 68-bit (top 17)
  plans, k = 2048 (the benchmark's host_1m and fixed_vs_wf_1m workloads).
* The 16-session agent batch (n drawn in [64K, 512K], per-session budgets,
  k = 1024) through the batched call, every query head of three sessions.
Keys of the million-key and agent workloads are drawn on the device by the
input generator (synth.device_keys), as the benchmark draws them."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import oracle
import synth
from tests.helpers import check_queries
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
def test_layer_scan_every_query(layer, B):
    ses, ix, ref = layer
    budgets = np.full(32, B, np.int32)
    t, nb, oi, os_ = _scan(ix, ses, budgets, 2048)
    rt, rT, rnb = oracle.plan_session(ref, ses.q_bf16, budgets, 4)
    assert np.array_equal(t, rt)
    assert np.array_equal(nb.astype(np.uint64), rnb)
    assert np.all(nb[:32] == B * 131072 // 8)
    check_queries(ref, ses.q_bf16, t, 4, 2048, oi, os_, list(range(32)))


def _variant_index(ses, **kw):
    ix = fp.KeyIndex(ses.n_kv_heads, ses.group, ses.n_keys, ses.head_dim, **kw)
    ix.pack(torch.from_numpy(ses.keys).cuda())
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    return ix


@pytest.mark.parametrize("variant", ["8plane", "blocked"])
def test_layer_variants_pack_plans_and_every_query(layer, variant):
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
        check_queries(ref, ses.q_bf16, t, 4, 2048, oi, os_, list(range(32)))


def _device_session(seed, H, n, d=128):
    sigma, _ = synth.channel_sigma(seed, H, d)
    return synth.device_keys(torch, sigma, n, seed)


@pytest.mark.slow
def test_host_million_token_layer_every_head():
    H, G, n, d, k = 8, 4, 1 << 20, 128, 2048
    keys = _device_session(0, H, n)
    ix = fp.KeyIndex(H, G, n, d, "host_mapped")
    ix.pack(keys)
    q_np = synth.draw_queries(31, H * G, d)[0]
    q = torch.from_numpy(q_np.view(np.int16)).cuda()
    budgets = np.tile(np.array([18, 68, 92, 136], np.int32), H)
    runs = {}
    for name, fixed in (("wf", None), ("fixed34", 34), ("fixed17", 17)):
        buf = fp.ScanBuffers(ix, k)
        fp.plan_and_scan(ix, q, torch.from_numpy(budgets).cuda(), buf, fixed_r=fixed)
        torch.cuda.synchronize()
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        runs[name] = (fixed, buf.t.cpu().numpy(), buf.nbytes.cpu().numpy(), buf.idx.cpu().numpy(),
                      buf.score.cpu().numpy())
    for h in range(H):
        ref = oracle.build_index(keys[h:h + 1].cpu().numpy())
        rows = slice(h * G, (h + 1) * G)
        for name, (fixed, t, nb, oi, os_) in runs.items():
            rt, _, rnb = oracle.plan_session(ref, q_np[rows], budgets[rows], G, fixed_r=fixed)
            assert np.array_equal(t[rows], rt), (name, h)
            assert np.array_equal(nb[rows].astype(np.uint64), rnb[:G]), (name, h)
            assert nb[H * G + h] == rnb[G], (name, h)
            check_queries(ref, q_np[rows], t[rows], G, k, oi[rows], os_[rows], list(range(G)),
                          heads=[0] * G)


@pytest.mark.slow
def test_agent_sessions_batched_full_size():
    """The 16 sessions of the agent workload in one batched call (host-
    resident planes, one budget per session, k = 1024); every query head of
    three sessions against the oracle."""
    H, G, d, k = 8, 4, 128, 1024
    params = synth.agent_session_params(16, 1000, H, head_dim=d)
    checked = (0, 7, 15)
    indices, qs, bufs, kept = [], [], [], {}
    for si, p in enumerate(params):
        keys = synth.device_keys(torch, p["sigma"], p["n"], p["seed"])
        ix = fp.KeyIndex(H, G, p["n"], d, "host_mapped")
        ix.pack(keys)
        q_np = synth.draw_queries(p["seed"] + 500, H * G, d)[0]
        q = torch.from_numpy(q_np.view(np.int16)).cuda()
        buf = fp.ScanBuffers(ix, k)
        b = torch.full((H * G,), p["budget"], dtype=torch.int32, device="cuda")
        fp.fathom_plan(ix.desc, q, b, buf.t, buf.t_union, buf.nbytes)
        if si in checked:
            kept[si] = (keys, q_np)
        del keys
        indices.append(ix)
        qs.append(q)
        bufs.append(buf)
    descs = [ix.desc for ix in indices]
    ws = torch.empty(fp.fathom_scan_batched_workspace_bytes(descs, k), dtype=torch.uint8,
                     device="cuda")
    fp.fathom_scan_topk_batched(descs, qs, [b.t for b in bufs], [b.t_union for b in bufs], k,
                                [b.idx for b in bufs], [b.score for b in bufs], ws)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    for si in checked:
        keys, q_np = kept.pop(si)
        ref = oracle.build_index(keys.cpu().numpy())
        del keys
        t = bufs[si].t.cpu().numpy()
        budgets = np.full(H * G, params[si]["budget"], np.int32)
        rt, _, rnb = oracle.plan_session(ref, q_np, budgets, G)
        assert np.array_equal(t, rt), si
        assert np.array_equal(bufs[si].nbytes.cpu().numpy().astype(np.uint64), rnb), si
        check_queries(ref, q_np, t, G, k, bufs[si].idx.cpu().numpy(),
                      bufs[si].score.cpu().numpy(), list(range(H * G)))
