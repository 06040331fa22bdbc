"""The C-ABI library loads and exports every symbol include/fathom.h declares;
host-side validation rejects bad arguments before touching the GPU.  CPU only:
no call here reaches a kernel."""
import ctypes
import os
import re

import pytest

import decode_fathom_plan_b200 as fp
from decode_fathom_plan_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "fathom.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fathom_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    fbuild.build()
    return fp.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert len(names) >= 13
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(fp.EXPORTED)


def test_n_words_rounds_to_16_byte_rows(lib):
    for n, w in ((1, 4), (32, 4), (128, 4), (129, 8), (4096, 128), (131072, 4096),
                 (1 << 20, 32768)):
        assert fp.fathom_n_words(n) == w
    assert fp.fathom_n_words(0) == 0


def test_status_strings(lib):
    for code in range(7):
        assert fp.status_str(code)
    assert "workspace" in fp.status_str(fp.FATHOM_ERR_WORKSPACE)


def _desc(H=2, G=4, d=128, n=4096, residency=0, fake=0x1000):
    return fp.fathom_index(H, G, d, n, fp.fathom_n_words(n), residency,
                           fake, fake, fake, fake, fake, fake)


def test_workspace_sizes_are_host_computable(lib):
    ix = _desc()
    assert fp.fathom_pack_workspace_bytes(ix) == 8 * 2 * 128
    ws = fp.fathom_scan_workspace_bytes(ix, 64)
    assert ws > 0 and ws % 256 == 0
    # larger k needs a larger candidate buffer
    big = _desc(n=1 << 20)
    assert fp.fathom_scan_workspace_bytes(big, 2048) > fp.fathom_scan_workspace_bytes(big, 64)
    assert fp.fathom_scan_batched_workspace_bytes([ix, big], 64) == \
        fp.fathom_scan_workspace_bytes(ix, 64) + fp.fathom_scan_workspace_bytes(big, 64)


def test_host_resident_workspace_holds_a_two_head_ring(lib):
    # a HOST_MAPPED index is scanned one KV head at a time: the workspace holds
    # the scratch of a one-head scan and a ring of two one-head plane slots
    # [d][4][n_words] uint32, so it does not grow with the number of heads
    for H, d, n in ((2, 128, 4096), (8, 128, 1 << 20), (1, 64, 1000)):
        one_head = fp.fathom_scan_workspace_bytes(_desc(H=1, d=d, n=n, residency=0), 64)
        host = fp.fathom_scan_workspace_bytes(_desc(H=H, d=d, n=n, residency=1), 64)
        slot = d * 4 * fp.fathom_n_words(n) * 4
        assert host == (one_head + 255) // 256 * 256 + 2 * ((slot + 255) // 256 * 256)
    # the million-key layer: well under the size of the index it scans
    index = 8 * 128 * 4 * fp.fathom_n_words(1 << 20) * 4
    assert fp.fathom_scan_workspace_bytes(_desc(H=8, d=128, n=1 << 20, residency=1), 2048) \
        < 0.3 * index


@pytest.mark.parametrize("field,value", [("head_dim", 48), ("head_dim", 512), ("group", 9),
                                         ("group", 0), ("n_words", 6), ("n_keys", 0),
                                         ("residency", 7), ("bits", 5), ("bits", 2),
                                         ("n_words", (1 << 22) + 4), ("block_keys", 1000),
                                         ("block_keys", -2048)])
def test_bad_index_shapes_are_rejected(lib, field, value):
    ix = _desc()
    setattr(ix, field, value)
    assert fp.fathom_scan_workspace_bytes(ix, 64) == 0
    assert fp.fathom_pack_workspace_bytes(ix) == 0
    rc = lib.fathom_plan(ctypes.byref(ix), 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0)
    assert rc == fp.FATHOM_ERR_INVALID_ARG


def test_null_pointers_are_rejected(lib):
    ix = _desc()
    assert lib.fathom_plan(ctypes.byref(ix), 0, 0x1000, 0x1000, 0x1000, 0x1000, 0) == \
        fp.FATHOM_ERR_INVALID_ARG
    assert lib.fathom_fixed_plan(ctypes.byref(ix), 0x1000, 200, 0x1000, 0x1000, 0x1000, 0) == \
        fp.FATHOM_ERR_INVALID_ARG
    assert lib.fathom_scan_topk(ctypes.byref(ix), 0, 0x1000, 0x1000, 64, 0x1000, 0x1000,
                                0x1000, 1 << 30, 0, 0) == fp.FATHOM_ERR_INVALID_ARG
    assert lib.fathom_pack_keys(0, ctypes.byref(ix), 0x1000, 1 << 20, 0) == \
        fp.FATHOM_ERR_INVALID_ARG


def test_bad_k_and_flags_are_rejected(lib):
    ix = _desc(n=100)
    for k in (0, 101, 5000):
        assert lib.fathom_scan_topk(ctypes.byref(ix), 0x1000, 0x1000, 0x1000, k, 0x1000, 0x1000,
                                    0x1000, 1 << 30, 0, 0) == fp.FATHOM_ERR_INVALID_ARG
    assert lib.fathom_scan_topk(ctypes.byref(ix), 0x1000, 0x1000, 0x1000, 8, 0x1000, 0x1000,
                                0x1000, 1 << 30, 1 << 7, 0) == fp.FATHOM_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(fp, "_lib", None)
    with pytest.raises(ImportError):
        fp.load_library(str(tmp_path / "missing.so"))


def test_append_rejects_bad_arguments_before_launching(lib):
    ix = _desc(n=100)                       # capacity: 128 keys
    fake = 0x1000
    F = fp.FATHOM_ERR_INVALID_ARG
    append = lib.fathom_append_keys
    assert append(ctypes.byref(ix), None, 1, None, None) == F           # no keys
    assert append(ctypes.byref(ix), fake, 0, None, None) == F           # m < 1
    assert append(ctypes.byref(ix), fake, 29, None, None) == F          # past the capacity
    bad = _desc(d=48)
    assert append(ctypes.byref(bad), fake, 1, None, None) == F
    assert ix.n_keys == 100                  # untouched on error


def test_sparse_attention_sizes_and_argument_checks(lib):
    ws = fp.fathom_sparse_attention_workspace_bytes
    assert ws(32, 128, 2048) == 32 * 16 * 130 * 4       # 16 runs of 128 keys per query
    assert ws(1, 32, 1) == 1 * 1 * 34 * 4
    assert ws(1, 48, 10) == 0 and ws(0, 128, 10) == 0 and ws(1, 128, 0) == 0
    fake = 0x1000
    att = lib.fathom_sparse_attention
    F = fp.FATHOM_ERR_INVALID_ARG
    args = lambda **kw: dict(dict(keys=fake, values=fake, H=1, G=1, d=128, n=10, q=fake,
                                  idx=fake, k=4, scale=0.1, out=fake, ws=fake, wsb=1 << 20), **kw)
    def call(a):
        return att(a["keys"], a["values"], a["H"], a["G"], a["d"], a["n"], a["q"], a["idx"],
                   a["k"], ctypes.c_float(a["scale"]), a["out"], a["ws"], a["wsb"], None)
    assert call(args(k=11)) == F            # k > n
    assert call(args(k=0)) == F
    assert call(args(d=40)) == F
    assert call(args(G=9)) == F
    assert call(args(idx=None)) == F
    assert call(args(scale=float("nan"))) == F


def test_merge_rejects_bad_arguments_before_launching(lib):
    fake = 0x1000
    F = fp.FATHOM_ERR_INVALID_ARG
    merge = lib.fathom_merge_topk
    offs = lambda *v: (ctypes.c_int64 * len(v))(*v)
    assert merge(fake, fake, offs(0, 10), 2, 4, 64, 64, fake, fake, None) == F      # overlapping ranges
    assert merge(fake, fake, offs(100, 0), 2, 4, 64, 64, fake, fake, None) == F     # not ascending
    assert merge(fake, fake, offs(0, 100), 2, 4, 64, 129, fake, fake, None) == F    # k > S*k_s
    assert merge(fake, fake, offs(0, 10000), 2, 4, 9000, 64, fake, fake, None) == F  # too many candidates
    assert merge(None, fake, offs(0, 100), 2, 4, 64, 64, fake, fake, None) == F


def test_eight_plane_index_sizes_and_limits(lib):
    """An 8-plane index scans as 2d nibble channels of 4 planes: its workspace
    is that of a 4-plane index of head_dim 2d plus the nibble-channel
    arguments (mn', scale' float [H][2d], q' bf16 [Q][2d], t' [Q][2d],
    t_union' [H][2d], each rounded up to 16 bytes)."""
    for H, G, d, n, res in ((2, 4, 128, 4096, 0), (8, 4, 128, 1 << 20, 0), (1, 1, 32, 100, 1)):
        ix8 = _desc(H=H, G=G, d=d, n=n, residency=res)
        ix8.bits = 8
        ix4 = _desc(H=H, G=G, d=2 * d, n=n, residency=res)
        a16 = lambda b: (b + 15) // 16 * 16
        Q, d2 = H * G, 2 * d
        lift = 2 * a16(H * d2 * 4) + a16(Q * d2 * 2) + a16(Q * d2) + a16(H * d2)
        assert fp.fathom_scan_workspace_bytes(ix8, 64) == \
            fp.fathom_scan_workspace_bytes(ix4, 64) + lift
        assert fp.fathom_pack_workspace_bytes(ix8) == 8 * H * d
    wide = _desc(d=256)
    wide.bits = 8                              # 2d = 512 nibble channels: too wide
    assert fp.fathom_scan_workspace_bytes(wide, 64) == 0
    long8 = _desc(n=(1 << 23) + 128)
    long8.bits = 8                             # n * sum_code2 would overflow int64
    assert fp.fathom_scan_workspace_bytes(long8, 64) == 0
    long8.bits = 4
    assert fp.fathom_scan_workspace_bytes(long8, 64) > 0
    a, b = _desc(), _desc()
    b.bits = 8                                 # one batch, one code width
    assert fp.fathom_scan_batched_workspace_bytes([a, b], 64) == 0
    a.bits = 8
    assert fp.fathom_scan_batched_workspace_bytes([a, b], 64) == \
        2 * fp.fathom_scan_workspace_bytes(b, 64)


def test_grouped_scale_workspace_holds_the_block_biases(lib):
    """Grouped per-token-block scales add one float per (KV head, block,
    query head) to the scan workspace; a batch mixes no scale modes."""
    for H, G, n, block in ((2, 4, 4096, 2048), (8, 4, 1 << 20, 2048), (1, 8, 5000, 4096)):
        plain = _desc(H=H, G=G, n=n)
        grouped = _desc(H=H, G=G, n=n)
        grouped.block_keys = block
        nb = -(-32 * fp.fathom_n_words(n) // block)
        extra = (H * nb * G * 4 + 255) // 256 * 256
        assert fp.fathom_scan_workspace_bytes(grouped, 64) == \
            fp.fathom_scan_workspace_bytes(plain, 64) + extra
    a, b = _desc(), _desc()
    b.block_keys = 2048
    assert fp.fathom_scan_batched_workspace_bytes([a, b], 64) == 0
    a.block_keys = 4096
    assert fp.fathom_scan_batched_workspace_bytes([a, b], 64) > 0
