"""8-plane K variant (an 8-bit upstream K cache, the adaptation the Fathom
explainer's deployment notes, 部署前必读 item 3, call for) on the GPU vs the
oracle through the C ABI.

Bars as for the 4-plane path: pack, append, plans and byte counts bit-exact;
scores within 1e-4 * sum_c |q_c khat_cj|; top-k sets equal up to keys inside
that band around the k-th score; outputs in ascending key index."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import oracle
import synth
from tests.helpers import check_topk, oracle_query
from tests.test_parity_gpu import check_pack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp.load_library()
    torch.cuda.set_device(0)
    fp.fathom_last_device_status()


def index8(ses, residency="device", keys=None, capacity=None):
    keys = ses.keys if keys is None else keys
    ix = fp.KeyIndex(ses.n_kv_heads, ses.group, keys.shape[1], ses.head_dim, residency,
                     capacity=capacity, bits=8)
    ix.pack(torch.from_numpy(np.ascontiguousarray(keys)).cuda())
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    return ix


def plan8(ix, ses, budgets=None, fixed_r=None, marginal=False):
    H, G, d = ses.n_kv_heads, ses.group, ses.head_dim
    Q = H * G
    q = torch.from_numpy(ses.q_bf16.view(np.int16)).cuda()
    b = torch.from_numpy(np.asarray(budgets if budgets is not None else np.zeros(Q),
                                    np.int32)).cuda()
    t = torch.empty((Q, d), dtype=torch.uint8, device="cuda")
    tu = torch.empty((H, d), dtype=torch.uint8, device="cuda")
    nb = torch.empty(Q + H, dtype=torch.int64, device="cuda")
    if fixed_r is not None:
        fp.fathom_fixed_plan(ix.desc, q, fixed_r, t, tu, nb)
    elif marginal:
        fp.fathom_plan_marginal(ix.desc, q, b, t, tu, nb)
    else:
        fp.fathom_plan(ix.desc, q, b, t, tu, nb)
    torch.cuda.synchronize()
    return q, t, tu, nb


def scan8(ix, ses, q, t, tu, k, flags=0):
    Q = ses.n_kv_heads * ses.group
    out_i = torch.full((Q, k), -1, dtype=torch.int32, device="cuda")
    out_s = torch.full((Q, k), np.nan, dtype=torch.float32, device="cuda")
    ws = torch.empty(fp.fathom_scan_workspace_bytes(ix.desc, k), dtype=torch.uint8,
                     device="cuda")
    fp.fathom_scan_topk(ix.desc, q, t, tu, k, out_i, out_s, ws, flags)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    return out_i.cpu().numpy(), out_s.cpu().numpy()


def check_all(ses, ref, t, out_i, out_s, k, queries=None):
    t = t.cpu().numpy()
    for qq in (range(ses.n_queries) if queries is None else queries):
        _, _, s, a = oracle_query(ref, ses.q_bf16[qq], t[qq], qq // ses.group, k)
        check_topk(out_i[qq], out_s[qq], s, a, k)


# ---------------------------------------------------------------- storage
@pytest.mark.parametrize("H,n,d", [(1, 4096, 128), (2, 1000, 128), (1, 33, 64),
                                   (3, 20000, 96), (2, 4097, 32)])
def test_pack8_bit_exact(H, n, d):
    ses = synth.make_session(80 + n, H, 1, n, 8, head_dim=d)
    ix = index8(ses)
    assert tuple(ix.planes.shape) == (H, d, 8, fp.fathom_n_words(n))
    check_pack(ix, oracle.build_index(ses.keys, bits=8))


def test_pack8_host_mapped_and_constant_channel():
    ses = synth.make_session(81, 2, 2, 5000, 8)
    ses.keys[1, :, 7] = -0.5
    ref = oracle.build_index(ses.keys, bits=8)
    assert ref["scale"][1, 7] == 0
    ix = index8(ses, "host_mapped")
    assert not ix.planes.is_cuda
    check_pack(ix, ref)


@pytest.mark.parametrize("residency", ["device", "host_mapped"])
def test_append8_decode_steps_bit_exact(residency):
    H, G, n, d = 2, 4, 1000, 128
    chunks = [1] * 20 + [45, 200, 1]
    total = n + sum(chunks)
    ses = synth.make_session(82, H, G, total, 64, head_dim=d)
    keys = ses.keys.copy()
    keys[:, n + 30:] *= 1.5                          # some keys leave the range
    ix = index8(ses, residency, keys=keys[:, :n], capacity=total)
    ref = oracle.build_index(keys[:, :n], capacity=total, bits=8)
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
        check_pack(ix, ref)
        assert np.array_equal(cl_gpu.cpu().numpy().view(np.uint32), cl_ref)
    assert cl_ref.sum() > 0


# ------------------------------------------------------------------ plans
@pytest.mark.parametrize("d", [32, 128])
def test_plan8_bit_exact(d):
    ses = synth.make_session(83 + d, 4, 4, 3000, 8, head_dim=d)
    ix = index8(ses)
    ref = oracle.build_index(ses.keys, bits=8)
    rng = np.random.default_rng(d)
    budgets = rng.integers(0, 8 * d + 1, size=16).astype(np.int32)
    budgets[:7] = [0, 1, 8, 9, 136, 8 * d, 8 * d - 1]
    for marginal in (False, True):
        _, t, tu, nb = plan8(ix, ses, budgets, marginal=marginal)
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        rt, rT, rnb = oracle.plan_session(ref, ses.q_bf16, budgets, 4, marginal=marginal)
        assert np.array_equal(t.cpu().numpy(), rt), marginal
        assert np.array_equal(tu.cpu().numpy(), rT), marginal
        assert np.array_equal(nb.cpu().numpy().astype(np.uint64), rnb), marginal
        assert t.cpu().numpy().max() <= 8


@pytest.mark.parametrize("r", [0, 17, 128])
def test_fixed_plan8_bit_exact(r):
    ses = synth.make_session(84, 2, 4, 2000, 8)
    ix = index8(ses)
    ref = oracle.build_index(ses.keys, bits=8)
    _, t, tu, nb = plan8(ix, ses, fixed_r=r)
    rt, rT, rnb = oracle.plan_session(ref, ses.q_bf16, np.zeros(8), 4, fixed_r=r)
    assert np.array_equal(t.cpu().numpy(), rt)
    assert np.array_equal(tu.cpu().numpy(), rT)
    assert np.array_equal(nb.cpu().numpy().astype(np.uint64), rnb)


def test_plan8_budget_out_of_range_sets_status():
    ses = synth.make_session(85, 1, 2, 500, 8)
    ix = index8(ses)
    _, t, _, _ = plan8(ix, ses, [8 * 128 + 1, 600])
    assert fp.fathom_last_device_status() == fp.FATHOM_ERR_INVALID_ARG
    assert int(t[0].sum()) == 0 and int(t[1].sum()) == 600


# ------------------------------------------------------------------- scan
@pytest.mark.parametrize("flags", [0, fp.FATHOM_SCAN_FORCE_EXACT])
def test_scan8_layer_ragged(flags):
    """Several tiles, a ragged tail, budgets from 0 to full depth."""
    H, G, n, d, k = 2, 4, 20011, 128, 64
    ses = synth.make_session(86, H, G, n, 136, n_planted=8)
    ses.budgets[:] = [0, 1, 9, 68, 136, 300, 777, 8 * d]
    ix = index8(ses)
    ref = oracle.build_index(ses.keys, bits=8)
    q, t, tu, _ = plan8(ix, ses, ses.budgets)
    out_i, out_s = scan8(ix, ses, q, t, tu, k, flags)
    check_all(ses, ref, t, out_i, out_s, k)


@pytest.mark.parametrize("G,d,n,k,B", [(1, 128, 33, 33, 64), (8, 64, 5000, 100, 200),
                                       (2, 32, 131, 7, 1), (4, 128, 4096, 1, 1024)])
def test_scan8_shapes(G, d, n, k, B):
    ses = synth.make_session(87 + n, 1, G, n, B, head_dim=d)
    ix = index8(ses)
    ref = oracle.build_index(ses.keys, bits=8)
    q, t, tu, _ = plan8(ix, ses, ses.budgets)
    out_i, out_s = scan8(ix, ses, q, t, tu, k)
    check_all(ses, ref, t, out_i, out_s, k)


def test_scan8_fixed_plan_and_host_mapped():
    H, G, n, k = 2, 4, 9000, 50
    ses = synth.make_session(88, H, G, n, 136)
    ref = oracle.build_index(ses.keys, bits=8)
    for residency in ("device", "host_mapped"):
        ix = index8(ses, residency)
        q, t, tu, _ = plan8(ix, ses, fixed_r=17)
        out_i, out_s = scan8(ix, ses, q, t, tu, k)
        check_all(ses, ref, t, out_i, out_s, k)


def test_scan8_full_depth_is_the_8bit_dot_product_topk():
    """B = 8d reads every plane: the scores are the exact dot products with
    the dequantised 8-bit keys (numpy fp64 matmul), so the GPU top-k is the
    top-k of those up to the tie band."""
    H, G, n, d, k = 1, 2, 6000, 128, 40
    ses = synth.make_session(89, H, G, n, 8 * d)
    ix = index8(ses)
    ref = oracle.build_index(ses.keys, bits=8)
    q, t, tu, _ = plan8(ix, ses, ses.budgets)
    assert int(t.min()) == 8
    out_i, out_s = scan8(ix, ses, q, t, tu, k)
    deq = ref["mn"][0][:, None].astype(np.float64) + \
        ref["scale"][0][:, None].astype(np.float64) * ref["codes"][0]
    for g in range(G):
        qf = synth.bf16_bits_to_f32(ses.q_bf16[g]).astype(np.float64)
        s = qf @ deq
        a = np.abs(qf) @ np.abs(deq)
        check_topk(out_i[g], out_s[g], s, a, k)


def test_scan8_batched_sessions():
    k = 32
    sess = [synth.make_session(90 + i, 2, 4, n, 200) for i, n in enumerate((3000, 7777))]
    ixs = [index8(s) for s in sess]
    plans = [plan8(ix, s, s.budgets) for ix, s in zip(ixs, sess)]
    descs = [ix.desc for ix in ixs]
    ws = torch.empty(fp.fathom_scan_batched_workspace_bytes(descs, k), dtype=torch.uint8,
                     device="cuda")
    outs = [(torch.empty((8, k), dtype=torch.int32, device="cuda"),
             torch.empty((8, k), dtype=torch.float32, device="cuda")) for _ in sess]
    fp.fathom_scan_topk_batched(descs, [p[0] for p in plans], [p[1] for p in plans],
                                [p[2] for p in plans], k, [o[0] for o in outs],
                                [o[1] for o in outs], ws)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    for s, p, o in zip(sess, plans, outs):
        check_all(s, oracle.build_index(s.keys, bits=8), p[1], o[0].cpu().numpy(),
                  o[1].cpu().numpy(), k)
