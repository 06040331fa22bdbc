"""Grouped per-token-block scales on the GPU vs the oracle through the C ABI:
each block of block_keys tokens of a channel quantised on its own (the
grouped quantised K of a serving stack, which the Fathom explainer's index
reuses, 亮点 / 适用边界).

Bars: pack (planes, per-block min / scale / sums, sigma^2), whole-block
appends and plans bit-exact; scores within 1e-4 * sum_c |q_c khat_cj|;
top-k sets equal up to keys inside that band around the k-th score;
outputs in ascending key index."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import oracle
import synth
from tests.helpers import check_topk, oracle_query

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp.load_library()
    torch.cuda.set_device(0)
    fp.fathom_last_device_status()


def drifting(seed, H, G, n, d=128, shift_every=3000, shift=1.5, budget=92):
    """A session whose key means move by `shift` every `shift_every` tokens
    (the case per-block scales are for)."""
    ses = synth.make_session(seed, H, G, n, budget, head_dim=d)
    ses.keys += (np.arange(n) // shift_every)[None, :, None].astype(np.float32) * np.float32(shift)
    return ses


def blocked_index(ses, block, residency="device", keys=None, capacity=None, bits=4):
    keys = ses.keys if keys is None else keys
    ix = fp.KeyIndex(ses.n_kv_heads, ses.group, keys.shape[1], ses.head_dim, residency,
                     capacity=capacity, bits=bits, block_keys=block)
    ix.pack(torch.from_numpy(np.ascontiguousarray(keys)).cuda())
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    return ix


def check_blocked_pack(ix, ref):
    nbf = oracle.n_blocks_for(ref["n"], ref["block_keys"])
    assert np.array_equal(ix.planes.cpu().numpy().view(np.uint32), ref["planes"]), "planes"
    assert np.array_equal(ix.mn.cpu().numpy()[:, :nbf], ref["mn"][:, :nbf])
    assert np.array_equal(ix.scale.cpu().numpy()[:, :nbf].view(np.uint32),
                          ref["scale"][:, :nbf].view(np.uint32))
    assert np.array_equal(ix.sum_code.cpu().numpy()[:, :nbf], ref["s1"][:, :nbf])
    assert np.array_equal(ix.sum_code2.cpu().numpy()[:, :nbf], ref["s2"][:, :nbf])
    assert np.array_equal(ix.sigma2.cpu().numpy().view(np.uint32), ref["sigma2"].view(np.uint32))


def plan(ix, ses, budgets=None, fixed_r=None):
    H, G, d = ses.n_kv_heads, ses.group, ses.head_dim
    Q = H * G
    q = torch.from_numpy(ses.q_bf16.view(np.int16)).cuda()
    b = torch.from_numpy(np.asarray(ses.budgets if budgets is None else budgets,
                                    np.int32)).cuda()
    t = torch.empty((Q, d), dtype=torch.uint8, device="cuda")
    tu = torch.empty((H, d), dtype=torch.uint8, device="cuda")
    nb = torch.empty(Q + H, dtype=torch.int64, device="cuda")
    if fixed_r is None:
        fp.fathom_plan(ix.desc, q, b, t, tu, nb)
    else:
        fp.fathom_fixed_plan(ix.desc, q, fixed_r, t, tu, nb)
    torch.cuda.synchronize()
    return q, t, tu, nb


def scan(ix, ses, q, t, tu, k, flags=0):
    Q = ses.n_kv_heads * ses.group
    out_i = torch.full((Q, k), -1, dtype=torch.int32, device="cuda")
    out_s = torch.full((Q, k), np.nan, dtype=torch.float32, device="cuda")
    ws = torch.empty(fp.fathom_scan_workspace_bytes(ix.desc, k), dtype=torch.uint8,
                     device="cuda")
    fp.fathom_scan_topk(ix.desc, q, t, tu, k, out_i, out_s, ws, flags)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    return out_i.cpu().numpy(), out_s.cpu().numpy()


def check_all(ses, ref, t, out_i, out_s, k):
    t = t.cpu().numpy()
    for qq in range(ses.n_queries):
        _, _, s, a = oracle_query(ref, ses.q_bf16[qq], t[qq], qq // ses.group, k)
        check_topk(out_i[qq], out_s[qq], s, a, k)


# ---------------------------------------------------------------- storage
@pytest.mark.parametrize("H,n,d,block,cap", [(1, 4096, 128, 2048, None), (2, 5000, 128, 2048, None),
                                             (1, 20000, 64, 4096, 30000), (3, 2047, 32, 2048, None),
                                             (2, 9000, 256, 8192, None)])
def test_blocked_pack_bit_exact(H, n, d, block, cap):
    ses = drifting(60 + n, H, 1, n, d)
    ix = blocked_index(ses, block, capacity=cap)
    check_blocked_pack(ix, oracle.build_index(ses.keys, capacity=cap, block_keys=block))


def test_blocked_pack_8plane_and_host_mapped():
    ses = drifting(61, 2, 2, 7000)
    ref = oracle.build_index(ses.keys, bits=8, block_keys=2048)
    check_blocked_pack(blocked_index(ses, 2048, bits=8), ref)
    check_blocked_pack(blocked_index(ses, 2048, "host_mapped", bits=8), ref)


@pytest.mark.parametrize("residency", ["device", "host_mapped"])
def test_blocked_append_of_whole_blocks_bit_exact(residency):
    ses = drifting(62, 2, 4, 4096 + 2048 + 1500, shift_every=2048, shift=3.0)
    total = ses.keys.shape[1]
    ix = blocked_index(ses, 2048, residency, keys=ses.keys[:, :4096], capacity=total)
    ref = oracle.build_index(ses.keys[:, :4096], capacity=total, block_keys=2048)
    at = 4096
    for m in (2048, 1500):
        new = np.ascontiguousarray(ses.keys[:, at:at + m])
        ix.append(torch.from_numpy(new).cuda())
        oracle.append_blocks(ref, new)
        at += m
        torch.cuda.synchronize()
        assert fp.fathom_last_device_status() == fp.FATHOM_OK
        assert ix.n_keys == at
        check_blocked_pack(ix, ref)
    # the last block is short: appending into it is refused before any launch
    with pytest.raises(fp.FathomError):
        ix.append(torch.zeros((2, 1, 128), dtype=torch.float32, device="cuda"))
    check_blocked_pack(ix, oracle.build_index(ses.keys, capacity=total, block_keys=2048))


# ------------------------------------------------------------------ plans
def test_blocked_plans_bit_exact():
    ses = drifting(63, 4, 4, 9000, budget=68)
    ix = blocked_index(ses, 2048)
    ref = oracle.build_index(ses.keys, block_keys=2048)
    budgets = np.random.default_rng(1).integers(0, 513, size=16).astype(np.int32)
    _, t, tu, nb = plan(ix, ses, budgets)
    rt, rT, rnb = oracle.plan_session(ref, ses.q_bf16, budgets, 4)
    assert np.array_equal(t.cpu().numpy(), rt)
    assert np.array_equal(tu.cpu().numpy(), rT)
    assert np.array_equal(nb.cpu().numpy().astype(np.uint64), rnb)


# ------------------------------------------------------------------- scan
@pytest.mark.parametrize("flags", [0, fp.FATHOM_SCAN_FORCE_EXACT])
def test_blocked_scan_layer_ragged(flags):
    H, G, n, k = 2, 4, 20011, 64
    ses = drifting(64, H, G, n)
    ses.budgets[:] = [0, 1, 18, 68, 92, 136, 300, 512]
    ix = blocked_index(ses, 2048)
    ref = oracle.build_index(ses.keys, block_keys=2048)
    q, t, tu, _ = plan(ix, ses)
    out_i, out_s = scan(ix, ses, q, t, tu, k, flags)
    check_all(ses, ref, t, out_i, out_s, k)


@pytest.mark.parametrize("G,d,n,k,B,block", [(1, 128, 33, 33, 64, 2048), (8, 64, 5000, 100, 200, 2048),
                                             (2, 32, 131, 7, 1, 4096), (4, 128, 40000, 2048, 136, 8192),
                                             (3, 256, 9001, 512, 300, 2048)])
def test_blocked_scan_shapes(G, d, n, k, B, block):
    ses = drifting(65 + n, 2, G, n, d, budget=B)
    ix = blocked_index(ses, block)
    ref = oracle.build_index(ses.keys, block_keys=block)
    q, t, tu, _ = plan(ix, ses)
    out_i, out_s = scan(ix, ses, q, t, tu, k)
    check_all(ses, ref, t, out_i, out_s, k)


def test_blocked_scan_full_depth_is_the_blocked_dot_product():
    """B = 4d: the score is the exact dot product with each key dequantised
    by its own block's scales (numpy fp64)."""
    H, G, n, k = 1, 2, 9000, 50
    ses = drifting(66, H, G, n, budget=512, shift_every=2048, shift=4.0)
    ix = blocked_index(ses, 2048)
    ref = oracle.build_index(ses.keys, block_keys=2048)
    q, t, tu, _ = plan(ix, ses)
    out_i, out_s = scan(ix, ses, q, t, tu, k)
    blk = np.arange(n) // 2048
    deq = ref["mn"][0][blk].T.astype(np.float64) + \
        ref["scale"][0][blk].T.astype(np.float64) * ref["codes"][0]
    for g in range(G):
        qf = synth.bf16_bits_to_f32(ses.q_bf16[g]).astype(np.float64)
        check_topk(out_i[g], out_s[g], qf @ deq, np.abs(qf) @ np.abs(deq), k)


def test_blocked_scan_8plane_fixed_plan_and_host_mapped():
    H, G, n, k = 2, 4, 9000, 40
    ses = drifting(67, H, G, n, budget=136)
    ref = oracle.build_index(ses.keys, bits=8, block_keys=2048)
    for residency in ("device", "host_mapped"):
        ix = blocked_index(ses, 2048, residency, bits=8)
        q, t, tu, _ = plan(ix, ses)
        out_i, out_s = scan(ix, ses, q, t, tu, k)
        check_all(ses, ref, t, out_i, out_s, k)
        q, t, tu, _ = plan(ix, ses, fixed_r=17)
        out_i, out_s = scan(ix, ses, q, t, tu, k)
        check_all(ses, ref, t, out_i, out_s, k)


def test_blocked_scan_batched_sessions():
    k = 32
    sess = [drifting(68 + i, 2, 4, n) for i, n in enumerate((5000, 12000))]
    ixs = [blocked_index(s, 2048 * (i + 1)) for i, s in enumerate(sess)]
    plans = [plan(ix, s) for ix, s in zip(ixs, sess)]
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
    for i, (s, p, o) in enumerate(zip(sess, plans, outs)):
        check_all(s, oracle.build_index(s.keys, block_keys=2048 * (i + 1)), p[1],
                  o[0].cpu().numpy(), o[1].cpu().numpy(), k)
