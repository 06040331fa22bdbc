"""GPU vs oracle parity through the C ABI, on seeded inputs small enough for
the oracle, spanning several tiles and ragged tails.

Bars: pack outputs, plans and byte counts bit-exact; scores within
1e-4 * sum_c |q_c khat_cj|; top-k sets equal up to keys inside that band
around the k-th score; outputs listed in ascending key index."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import oracle
import synth
from tests.helpers import check_topk, oracle_query, to_np_u32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp.load_library()
    torch.cuda.set_device(0)
    fp.fathom_last_device_status()


def gpu_index(ses, residency="device"):
    ix = fp.KeyIndex(ses.n_kv_heads, ses.group, ses.n_keys, ses.head_dim, residency)
    ix.pack(torch.from_numpy(ses.keys).cuda())
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    return ix


def check_pack(ix, ref):
    planes = ix.planes.cpu().numpy().view(np.uint32)
    assert np.array_equal(planes, ref["planes"]), "planes differ"
    assert np.array_equal(ix.mn.cpu().numpy(), ref["mn"])           # float equality
    assert np.array_equal(ix.scale.cpu().numpy().view(np.uint32), ref["scale"].view(np.uint32))
    assert np.array_equal(ix.sum_code.cpu().numpy(), ref["s1"])
    assert np.array_equal(ix.sum_code2.cpu().numpy(), ref["s2"])
    assert np.array_equal(ix.sigma2.cpu().numpy().view(np.uint32), ref["sigma2"].view(np.uint32))


# ---------------------------------------------------------------- pack
@pytest.mark.parametrize("H,n,d,planted", [(1, 4096, 128, 16), (2, 1000, 128, 0),
                                            (1, 33, 64, 0), (2, 4097, 256, 0),
                                            (1, 129, 32, 0), (3, 20000, 96, 0)])
def test_pack_bit_exact(H, n, d, planted):
    ses = synth.make_session(40 + n, H, 1, n, 8, head_dim=d, n_planted=planted)
    check_pack(gpu_index(ses), oracle.build_index(ses.keys))


def test_pack_host_mapped_bit_exact():
    ses = synth.make_session(7, 2, 2, 5000, 8)
    ix = gpu_index(ses, "host_mapped")
    assert not ix.planes.is_cuda
    check_pack(ix, oracle.build_index(ses.keys))


def test_pack_constant_channel():
    ses = synth.make_session(8, 1, 1, 300, 8)
    ses.keys[0, :, 5] = 2.5
    ref = oracle.build_index(ses.keys)
    assert ref["scale"][0, 5] == 0
    check_pack(gpu_index(ses), ref)


def test_pack_nonfinite_key_sets_status():
    ses = synth.make_session(9, 1, 1, 200, 8)
    ses.keys[0, 17, 3] = np.inf
    ix = fp.KeyIndex(1, 1, 200, 128)
    ix.pack(torch.from_numpy(ses.keys).cuda())
    assert fp.fathom_last_device_status() == fp.FATHOM_ERR_NONFINITE
    assert fp.fathom_last_device_status() == fp.FATHOM_OK     # cleared


# ---------------------------------------------------------------- plan
def run_plan(ix, ses, budgets, fixed_r=None):
    H, G, d = ses.n_kv_heads, ses.group, ses.head_dim
    Q = H * G
    q = torch.from_numpy(ses.q_bf16.view(np.int16)).cuda()
    b = torch.from_numpy(np.asarray(budgets, np.int32)).cuda()
    t = torch.empty((Q, d), dtype=torch.uint8, device="cuda")
    tu = torch.empty((H, d), dtype=torch.uint8, device="cuda")
    nb = torch.empty(Q + H, dtype=torch.int64, device="cuda")
    if fixed_r is None:
        fp.fathom_plan(ix.desc, q, b, t, tu, nb)
    else:
        fp.fathom_fixed_plan(ix.desc, q, fixed_r, t, tu, nb)
    torch.cuda.synchronize()
    return q, t, tu, nb


@pytest.mark.parametrize("d", [32, 128, 256])
def test_plan_bit_exact(d):
    ses = synth.make_session(11 + d, 4, 4, 3000, 8, head_dim=d)
    ix = gpu_index(ses)
    ref_ix = oracle.build_index(ses.keys)
    rng = np.random.default_rng(d)
    budgets = rng.integers(0, 4 * d + 1, size=16).astype(np.int32)
    budgets[:6] = [0, 1, 8, 18, 4 * d, 4 * d - 1]
    _, t, tu, nb = run_plan(ix, ses, budgets)
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    rt, rT, rnb = oracle.plan_session(ref_ix, ses.q_bf16, budgets, 4)
    assert np.array_equal(t.cpu().numpy(), rt)
    assert np.array_equal(tu.cpu().numpy(), rT)
    assert np.array_equal(nb.cpu().numpy().astype(np.uint64), rnb)


@pytest.mark.parametrize("r", [0, 1, 17, 34, 128])
def test_fixed_plan_bit_exact(r):
    ses = synth.make_session(21, 2, 4, 2000, 8)
    ix = gpu_index(ses)
    ref_ix = oracle.build_index(ses.keys)
    _, t, tu, nb = run_plan(ix, ses, np.zeros(8, np.int32), fixed_r=r)
    rt, rT, rnb = oracle.plan_session(ref_ix, ses.q_bf16, np.zeros(8), 4, fixed_r=r)
    assert np.array_equal(t.cpu().numpy(), rt)
    assert np.array_equal(tu.cpu().numpy(), rT)
    assert np.array_equal(nb.cpu().numpy().astype(np.uint64), rnb)


def test_plan_budget_out_of_range_sets_status():
    ses = synth.make_session(12, 1, 2, 500, 8)
    ix = gpu_index(ses)
    _, t, _, _ = run_plan(ix, ses, [-1, 40])
    assert fp.fathom_last_device_status() == fp.FATHOM_ERR_INVALID_ARG
    assert int(t[0].sum()) == 0 and int(t[1].sum()) == 40
    run_plan(ix, ses, [513, 40])
    assert fp.fathom_last_device_status() == fp.FATHOM_ERR_INVALID_ARG


# ---------------------------------------------------------------- scan
def run_scan(ix, ses, q, t, tu, k, flags=0):
    Q = ses.n_kv_heads * ses.group
    out_i = torch.full((Q, k), -1, dtype=torch.int32, device="cuda")
    out_s = torch.full((Q, k), np.nan, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(16, fp.fathom_scan_workspace_bytes(ix.desc, k)), dtype=torch.uint8,
                     device="cuda")
    fp.fathom_scan_topk(ix.desc, q, t, tu, k, out_i, out_s, ws, flags)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    return out_i.cpu().numpy(), out_s.cpu().numpy()


def check_scan(ses, ref_ix, t, out_i, out_s, k, queries=None):
    G = ses.group
    t = t.cpu().numpy()
    diffs = 0
    for qq in (range(ses.n_queries) if queries is None else queries):
        _, _, s, a = oracle_query(ref_ix, ses.q_bf16[qq], t[qq], qq // G, k)
        diffs += check_topk(out_i[qq], out_s[qq], s, a, k)
    return diffs


@pytest.mark.parametrize("flags", [0, fp.FATHOM_SCAN_FORCE_EXACT])
def test_scan_tiny_4k(flags):
    ses = synth.tiny_4k()
    ix = gpu_index(ses)
    ref = oracle.build_index(ses.keys)
    q, t, tu, _ = run_plan(ix, ses, ses.budgets)
    oi, os_ = run_scan(ix, ses, q, t, tu, 64, flags)
    check_scan(ses, ref, t, oi, os_, 64)
    assert len(set(ses.planted[0].tolist()) & set(oi[0].tolist())) >= 12


@pytest.mark.parametrize("flags", [0, fp.FATHOM_SCAN_FORCE_EXACT])
def test_scan_layer_ragged_sampled_path(flags):
    """8 KV heads x 4 query heads, 20000 keys (ragged last tile), budgets
    mixed inside each GQA group, k = 256: the sampled-threshold path."""
    budgets = np.tile(np.array([68, 92, 136, 18], np.int32), 8)
    ses = synth.make_session(31, 8, 4, 20000, budgets)
    ix = gpu_index(ses)
    ref = oracle.build_index(ses.keys)
    q, t, tu, _ = run_plan(ix, ses, ses.budgets)
    oi, os_ = run_scan(ix, ses, q, t, tu, 256, flags)
    check_scan(ses, ref, t, oi, os_, 256)


@pytest.mark.parametrize("G,d,n,k,B", [(1, 128, 33, 1, 16), (1, 128, 33, 33, 64),
                                       (2, 64, 1000, 7, 40), (3, 128, 9000, 100, 92),
                                       (8, 32, 5000, 64, 50), (8, 256, 9001, 512, 300),
                                       (4, 128, 40000, 2048, 136), (2, 128, 6000, 3000, 68)])
def test_scan_shapes(G, d, n, k, B):
    H = 2
    ses = synth.make_session(50 + n + G, H, G, n, B, head_dim=d)
    ix = gpu_index(ses)
    ref = oracle.build_index(ses.keys)
    q, t, tu, _ = run_plan(ix, ses, ses.budgets)
    oi, os_ = run_scan(ix, ses, q, t, tu, k)
    check_scan(ses, ref, t, oi, os_, k)


@pytest.mark.parametrize("flags", [0, fp.FATHOM_SCAN_FORCE_EXACT])
def test_scan_exact_ties_resolve_to_lower_index(flags):
    """B = 4: one channel read at 4 bits -> at most 16 distinct scores, equal
    on both sides bit for bit; the top-k must be the oracle's exactly.
    B = 0: every score equal -> the first k keys."""
    ses = synth.make_session(61, 2, 2, 30000, [4, 4, 0, 0])
    ix = gpu_index(ses)
    ref = oracle.build_index(ses.keys)
    q, t, tu, _ = run_plan(ix, ses, ses.budgets)
    oi, os_ = run_scan(ix, ses, q, t, tu, 300, flags)
    assert check_scan(ses, ref, t, oi, os_, 300) == 0
    for qq in (2, 3):
        assert np.array_equal(oi[qq], np.arange(300))


def test_scan_fixed_plans():
    ses = synth.make_session(71, 2, 4, 12000, 0)
    ix = gpu_index(ses)
    ref = oracle.build_index(ses.keys)
    for r in (34, 17):
        q, t, tu, _ = run_plan(ix, ses, ses.budgets, fixed_r=r)
        oi, os_ = run_scan(ix, ses, q, t, tu, 512)
        check_scan(ses, ref, t, oi, os_, 512)


def test_scan_host_mapped():
    budgets = np.tile(np.array([68, 92, 136, 18], np.int32), 2)
    ses = synth.make_session(81, 2, 4, 25000, budgets)
    ix = gpu_index(ses, "host_mapped")
    ref = oracle.build_index(ses.keys)
    q, t, tu, _ = run_plan(ix, ses, ses.budgets)
    for flags in (0, fp.FATHOM_SCAN_FORCE_EXACT):
        oi, os_ = run_scan(ix, ses, q, t, tu, 512, flags)
        check_scan(ses, ref, t, oi, os_, 512)


def test_scan_batched_sessions():
    """Independent sessions of different lengths and budgets in one call."""
    sessions = [synth.make_session(90 + i, 2, 4, n, B)
                for i, (n, B) in enumerate([(9000, 68), (20000, 136), (4096, 92)])]
    k = 128
    gix, refs, qs, ts, tus, ois, oss = [], [], [], [], [], [], []
    for ses in sessions:
        ix = gpu_index(ses, "host_mapped" if ses.n_keys == 20000 else "device")
        q, t, tu, _ = run_plan(ix, ses, ses.budgets)
        gix.append(ix)
        refs.append(oracle.build_index(ses.keys))
        qs.append(q), ts.append(t), tus.append(tu)
        ois.append(torch.full((8, k), -1, dtype=torch.int32, device="cuda"))
        oss.append(torch.zeros((8, k), dtype=torch.float32, device="cuda"))
    descs = [ix.desc for ix in gix]
    ws = torch.empty(fp.fathom_scan_batched_workspace_bytes(descs, k), dtype=torch.uint8,
                     device="cuda")
    fp.fathom_scan_topk_batched(descs, qs, ts, tus, k, ois, oss, ws)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    for ses, ref, t, oi, os_ in zip(sessions, refs, ts, ois, oss):
        check_scan(ses, ref, t, oi.cpu().numpy(), os_.cpu().numpy(), k)


def test_host_mapped_scan_replays_as_a_cuda_graph():
    """A host-resident scan fetches its heads on a side stream forked from the
    caller's stream and joined back: captured (global capture mode, on a
    stream of its own) as one CUDA graph and replayed twice, it gives the
    eager call's result bit for bit, and the oracle's."""
    ses = synth.make_session(61, 3, 4, 40000, [18, 68, 92, 136] * 3)
    ix = gpu_index(ses, "host_mapped")
    q, t, tu, _ = run_plan(ix, ses, ses.budgets)
    k = 512
    eager_i, eager_s = run_scan(ix, ses, q, t, tu, k)
    check_scan(ses, oracle.build_index(ses.keys), t, eager_i, eager_s, k)
    Q = 12
    out_i = torch.full((Q, k), -1, dtype=torch.int32, device="cuda")
    out_s = torch.zeros((Q, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(fp.fathom_scan_workspace_bytes(ix.desc, k), dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    # first call on this stream outside the capture (creates its side stream)
    with torch.cuda.stream(side):
        fp.fathom_scan_topk(ix.desc, q, t, tu, k, out_i, out_s, ws)
    side.synchronize()
    g = torch.cuda.CUDAGraph()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            fp.fathom_scan_topk(ix.desc, q, t, tu, k, out_i, out_s, ws)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        out_i.fill_(-1)
        out_s.fill_(0.0)
        g.replay()
        torch.cuda.synchronize()
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        assert np.array_equal(out_i.cpu().numpy(), eager_i)
        assert np.array_equal(out_s.cpu().numpy().view(np.uint32), eager_s.view(np.uint32))
    del g


def test_scan_rejects_small_workspace():
    ses = synth.make_session(5, 1, 1, 1000, 16)
    ix = gpu_index(ses)
    q, t, tu, _ = run_plan(ix, ses, ses.budgets)
    oi = torch.empty((1, 8), dtype=torch.int32, device="cuda")
    os_ = torch.empty((1, 8), dtype=torch.float32, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fp.FathomError) as e:
        fp.fathom_scan_topk(ix.desc, q, t, tu, 8, oi, os_, ws)
    assert e.value.status == fp.FATHOM_ERR_WORKSPACE


def test_scan_profile_flag_times_the_scan_kernel():
    """FATHOM_SCAN_PROFILE records events around the main scan kernel, both
    when launched eagerly and inside a CUDA graph capture."""
    ses = synth.make_session(77, 2, 4, 30000, 92)
    ix = gpu_index(ses)
    q, t, tu, _ = run_plan(ix, ses, ses.budgets)
    buf = fp.ScanBuffers(ix, 128)
    fp.fathom_profile_read()
    fp.fathom_scan_topk(ix.desc, q, t, tu, 128, buf.idx, buf.score, buf.workspace,
                        fp.FATHOM_SCAN_PROFILE)
    torch.cuda.synchronize()
    ms, n = fp.fathom_profile_read()
    assert n == 1 and ms > 0
    ref_idx = buf.idx.clone()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
            fp.fathom_scan_topk(ix.desc, q, t, tu, 128, buf.idx, buf.score, buf.workspace,
                                fp.FATHOM_SCAN_PROFILE)
    torch.cuda.current_stream().wait_stream(side)
    buf.idx.zero_()
    g.replay()
    torch.cuda.synchronize()
    ms, n = fp.fathom_profile_read()
    assert n == 1 and ms > 0
    assert torch.equal(buf.idx, ref_idx)
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    del g
