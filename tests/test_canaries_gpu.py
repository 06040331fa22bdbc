"""Canary words after every output buffer of the C ABI: each call writes
exactly the bytes its header declares.  Outputs are views of larger device
buffers filled with a canary byte; after the call (and a sync) every byte
past the declared size must still hold the canary.  Covers the storage
side (4-bit, 8-plane, grouped scales), appends, plans, scans, sparse
attention and the shard merge."""
import numpy as np
import pytest
import torch

import decode_fathom_plan_b200 as fp
import synth

pytestmark = pytest.mark.gpu

CANARY = 0xA5
TAIL = 4096   # bytes of canary after every output


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp.load_library()
    torch.cuda.set_device(0)
    fp.fathom_last_device_status()


class Guarded:
    """A device tensor of `shape` and `dtype` followed by TAIL canary bytes."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((n + TAIL,), CANARY, dtype=torch.uint8, device="cuda")
        self.nbytes = n
        self.t = self.raw[:n].view(dtype).view(shape)

    def intact(self):
        torch.cuda.synchronize()
        return bool((self.raw[self.nbytes:] == CANARY).all())


def guarded_index(H, G, n, d, bits=4, block_keys=0, capacity=None):
    nw = fp.fathom_n_words(max(n, capacity or n))
    nb = -(-32 * nw // block_keys) if block_keys else 1
    stat = (H, nb, d) if block_keys else (H, d)
    bufs = dict(planes=Guarded((H, d, bits, nw), torch.int32),
                mn=Guarded(stat, torch.float32), scale=Guarded(stat, torch.float32),
                sigma2=Guarded((H, d), torch.float32), s1=Guarded(stat, torch.int64),
                s2=Guarded(stat, torch.int64))
    desc = fp.fathom_index(H, G, d, n, nw, 0, bufs["planes"].t.data_ptr(),
                           bufs["mn"].t.data_ptr(), bufs["scale"].t.data_ptr(),
                           bufs["sigma2"].t.data_ptr(), bufs["s1"].t.data_ptr(),
                           bufs["s2"].t.data_ptr(), bits, block_keys)
    return desc, bufs


def pack(desc, keys):
    ws = Guarded((max(16, fp.fathom_pack_workspace_bytes(desc)),), torch.uint8)
    fp.fathom_pack_keys(torch.from_numpy(np.ascontiguousarray(keys)).cuda(), desc, ws.t)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    assert ws.intact()


@pytest.mark.parametrize("bits,block_keys", [(4, 0), (8, 0), (4, 2048), (8, 4096)])
def test_storage_side_writes_only_its_arrays(bits, block_keys):
    H, G, n, d = 2, 4, 5000, 64
    ses = synth.make_session(300 + bits + block_keys, H, G, n + 2048, 64, head_dim=d)
    desc, bufs = guarded_index(H, G, n if not block_keys else 4096, d, bits, block_keys,
                               capacity=n + 2048)
    pack(desc, ses.keys[:, :desc.n_keys])
    assert all(b.intact() for b in bufs.values())
    # an append (whole blocks with grouped scales) keeps inside them too
    m = 2048 if block_keys else 37
    new = torch.from_numpy(np.ascontiguousarray(ses.keys[:, desc.n_keys:desc.n_keys + m])).cuda()
    clamped = Guarded((H, d), torch.int32)
    clamped.t.zero_()
    fp.fathom_append_keys(new, desc, m, clamped.t)
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
    assert all(b.intact() for b in bufs.values()) and clamped.intact()


@pytest.mark.parametrize("bits,block_keys", [(4, 0), (8, 0), (4, 2048)])
def test_read_side_writes_only_its_outputs(bits, block_keys):
    H, G, n, d, k = 2, 4, 20000, 128, 100
    Q = H * G
    ses = synth.make_session(310 + bits, H, G, n, 92, head_dim=d)
    desc, bufs = guarded_index(H, G, n, d, bits, block_keys)
    pack(desc, ses.keys)
    q = torch.from_numpy(ses.q_bf16.view(np.int16)).cuda()
    b = torch.from_numpy(ses.budgets).cuda()
    for kind in ("wf", "mg", "fixed"):
        t, tu, nb = Guarded((Q, d), torch.uint8), Guarded((H, d), torch.uint8), \
            Guarded((Q + H,), torch.int64)
        if kind == "wf":
            fp.fathom_plan(desc, q, b, t.t, tu.t, nb.t)
        elif kind == "mg":
            fp.fathom_plan_marginal(desc, q, b, t.t, tu.t, nb.t)
        else:
            fp.fathom_fixed_plan(desc, q, 17, t.t, tu.t, nb.t)
        assert t.intact() and tu.intact() and nb.intact(), kind
        for flags in (0, fp.FATHOM_SCAN_FORCE_EXACT):
            oi, os_ = Guarded((Q, k), torch.int32), Guarded((Q, k), torch.float32)
            ws = Guarded((fp.fathom_scan_workspace_bytes(desc, k),), torch.uint8)
            fp.fathom_scan_topk(desc, q, t.t, tu.t, k, oi.t, os_.t, ws.t, flags)
            torch.cuda.synchronize()
            assert fp.fathom_last_device_status() == fp.FATHOM_OK
            assert oi.intact() and os_.intact() and ws.intact(), (kind, flags)
            assert int(oi.t.min()) >= 0 and int(oi.t.max()) < n
    assert all(x.intact() for x in bufs.values())


def test_attention_and_merge_write_only_their_outputs():
    H, G, n, d, k = 2, 4, 3000, 128, 64
    Q = H * G
    rng = np.random.default_rng(5)
    keys = torch.from_numpy(rng.standard_normal((H, n, d)).astype(np.float32)).cuda()
    values = torch.from_numpy(rng.standard_normal((H, n, d)).astype(np.float32)).cuda()
    q = torch.from_numpy(synth.f32_to_bf16_bits(
        rng.standard_normal((Q, d)).astype(np.float32)).view(np.int16)).cuda()
    idx = np.sort(rng.choice(n, (Q, k), replace=False), axis=1).astype(np.int32)
    idx = torch.from_numpy(idx).cuda()
    out = Guarded((Q, d), torch.float32)
    ws = Guarded((max(16, fp.fathom_sparse_attention_workspace_bytes(Q, d, k)),), torch.uint8)
    fp.fathom_sparse_attention(keys, values, H, G, d, n, q, idx, k, 1.0 / np.sqrt(d), out.t, ws.t)
    assert out.intact() and ws.intact()
    S, k_s = 3, 40
    sidx = torch.from_numpy(np.sort(np.stack([rng.choice(1000, (Q, k_s), replace=False)
                                              for _ in range(S)]), axis=2).astype(np.int32)).cuda()
    ssc = torch.from_numpy(rng.standard_normal((S, Q, k_s)).astype(np.float32)).cuda()
    oi, os_ = Guarded((Q, 50), torch.int32), Guarded((Q, 50), torch.float32)
    fp.fathom_merge_topk(sidx, ssc, [0, 1000, 2000], 50, oi.t, os_.t)
    assert oi.intact() and os_.intact()
    torch.cuda.synchronize()
    assert fp.fathom_last_device_status() == fp.FATHOM_OK
