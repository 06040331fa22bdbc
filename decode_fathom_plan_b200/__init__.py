"""Python binding of libfathom.so, the sm_100a Fathom read-depth key scan.

Argument marshalling only: every step of the path (pack, plan, scan, select)
runs in the library's CUDA kernels.  PyTorch supplies device memory, pinned
host memory and streams.  There is no CPU fallback: if the library is
missing or no GPU is present, the calls raise.

The entry points carry the C names of include/fathom.h and take torch
tensors (or raw addresses) where the C call takes pointers.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libfathom.so")

FATHOM_OK = 0
FATHOM_ERR_INVALID_ARG = 1
FATHOM_ERR_CUDA = 2
FATHOM_ERR_NONFINITE = 3
FATHOM_ERR_TIMEOUT = 4
FATHOM_ERR_WORKSPACE = 5
FATHOM_ERR_UNIMPLEMENTED = 6

FATHOM_RES_DEVICE = 0
FATHOM_RES_HOST_MAPPED = 1

FATHOM_SCAN_DEFAULT = 0
FATHOM_SCAN_FORCE_EXACT = 1
FATHOM_SCAN_PROFILE = 2

EXPORTED = (
    "fathom_n_words", "fathom_status_str", "fathom_pack_workspace_bytes", "fathom_pack_keys",
    "fathom_plan", "fathom_fixed_plan", "fathom_scan_workspace_bytes", "fathom_scan_topk",
    "fathom_scan_batched_workspace_bytes", "fathom_scan_topk_batched",
    "fathom_last_device_status", "fathom_launch_count", "fathom_profile_read",
    "fathom_scan_topk_static", "fathom_link_probe", "fathom_append_keys",
    "fathom_sparse_attention_workspace_bytes", "fathom_sparse_attention", "fathom_plan_marginal",
    "fathom_merge_topk",
)


class FathomError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} (status {status})")


class fathom_index(ctypes.Structure):
    """Mirror of the C fathom_index descriptor."""
    _fields_ = [
        ("n_kv_heads", ctypes.c_int32), ("group", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("n_keys", ctypes.c_int32),
        ("n_words", ctypes.c_int32), ("residency", ctypes.c_int32),
        ("planes", ctypes.c_void_p), ("mn", ctypes.c_void_p), ("scale", ctypes.c_void_p),
        ("sigma2", ctypes.c_void_p), ("sum_code", ctypes.c_void_p),
        ("sum_code2", ctypes.c_void_p), ("bits", ctypes.c_int32),
        ("block_keys", ctypes.c_int32),
    ]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libfathom.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python decode_fathom_plan_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    P, I32, SZ, U32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_uint32
    IX = ctypes.POINTER(fathom_index)
    sig = {
        "fathom_n_words": ([I32], I32),
        "fathom_status_str": ([ctypes.c_int], ctypes.c_char_p),
        "fathom_pack_workspace_bytes": ([IX], SZ),
        "fathom_pack_keys": ([P, IX, P, SZ, P], ctypes.c_int),
        "fathom_append_keys": ([IX, P, I32, P, P], ctypes.c_int),
        "fathom_sparse_attention_workspace_bytes": ([I32, I32, I32], SZ),
        "fathom_sparse_attention": ([P, P, I32, I32, I32, I32, P, P, I32, ctypes.c_float, P, P,
                                     SZ, P], ctypes.c_int),
        "fathom_plan": ([IX, P, P, P, P, P, P], ctypes.c_int),
        "fathom_fixed_plan": ([IX, P, I32, P, P, P, P], ctypes.c_int),
        "fathom_plan_marginal": ([IX, P, P, P, P, P, P], ctypes.c_int),
        "fathom_merge_topk": ([P, P, P, I32, I32, I32, I32, P, P, P], ctypes.c_int),
        "fathom_scan_workspace_bytes": ([IX, I32], SZ),
        "fathom_scan_topk": ([IX, P, P, P, I32, P, P, P, SZ, U32, P], ctypes.c_int),
        "fathom_scan_topk_static": ([IX, P, P, P, I32, P, P, U32, P], ctypes.c_int),
        "fathom_scan_batched_workspace_bytes": ([IX, I32, I32], SZ),
        "fathom_scan_topk_batched": ([IX, I32, P, P, P, I32, P, P, P, SZ, U32, P], ctypes.c_int),
        "fathom_last_device_status": ([P], ctypes.c_int),
        "fathom_launch_count": ([], ctypes.c_uint64),
        "fathom_link_probe": ([P, SZ, P, P], ctypes.c_int),
        "fathom_profile_read": ([ctypes.POINTER(ctypes.c_double),
                                 ctypes.POINTER(ctypes.c_uint64)], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _ptr(x) -> int:
    """Address of a torch tensor (or pass through an int / None)."""
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, what: str):
    if rc != FATHOM_OK:
        raise FathomError(rc, what)


def status_str(status: int) -> str:
    return load_library().fathom_status_str(int(status)).decode()


# --------------------------------------------------------------- C entry points
def fathom_n_words(n_keys: int) -> int:
    return int(load_library().fathom_n_words(int(n_keys)))


def fathom_status_str(status: int) -> str:
    return status_str(status)


def fathom_pack_workspace_bytes(index: fathom_index) -> int:
    return int(load_library().fathom_pack_workspace_bytes(ctypes.byref(index)))


def fathom_pack_keys(keys, index: fathom_index, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load_library().fathom_pack_keys(_ptr(keys), ctypes.byref(index), _ptr(workspace),
                                           ws_bytes, _stream(stream)), "fathom_pack_keys")


def fathom_append_keys(keys, index: fathom_index, m: int, clamped=None, stream=None):
    """Append m keys (device float32 [H][m][d]) to the index; index.n_keys
    grows by m.  clamped: optional device uint32 [H][d] drift counters."""
    _check(load_library().fathom_append_keys(ctypes.byref(index), _ptr(keys), int(m),
                                             None if clamped is None else _ptr(clamped),
                                             _stream(stream)), "fathom_append_keys")


def fathom_plan(index: fathom_index, q_bf16, budget, t, t_union, nbytes, stream=None):
    _check(load_library().fathom_plan(ctypes.byref(index), _ptr(q_bf16), _ptr(budget), _ptr(t),
                                      _ptr(t_union), _ptr(nbytes), _stream(stream)),
           "fathom_plan")


def fathom_plan_marginal(index: fathom_index, q_bf16, budget, t, t_union, nbytes, stream=None):
    _check(load_library().fathom_plan_marginal(ctypes.byref(index), _ptr(q_bf16), _ptr(budget),
                                               _ptr(t), _ptr(t_union), _ptr(nbytes),
                                               _stream(stream)), "fathom_plan_marginal")


def fathom_fixed_plan(index: fathom_index, q_bf16, r: int, t, t_union, nbytes, stream=None):
    _check(load_library().fathom_fixed_plan(ctypes.byref(index), _ptr(q_bf16), int(r), _ptr(t),
                                            _ptr(t_union), _ptr(nbytes), _stream(stream)),
           "fathom_fixed_plan")


def fathom_scan_workspace_bytes(index: fathom_index, k: int) -> int:
    return int(load_library().fathom_scan_workspace_bytes(ctypes.byref(index), int(k)))


def fathom_scan_topk(index: fathom_index, q_bf16, t, t_union, k: int, out_idx, out_score,
                     workspace, flags: int = 0, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load_library().fathom_scan_topk(ctypes.byref(index), _ptr(q_bf16), _ptr(t),
                                           _ptr(t_union), int(k), _ptr(out_idx), _ptr(out_score),
                                           _ptr(workspace), ws_bytes, int(flags),
                                           _stream(stream)), "fathom_scan_topk")


def fathom_scan_topk_static(index: fathom_index, q_bf16, t, t_union, k: int, out_idx,
                            out_score, flags: int = 0, stream=None):
    """fathom_scan_topk without a workspace argument, for callers that cannot
    allocate device memory: runs on the library's fixed 8 MiB per-GPU scratch
    array (see include/fathom.h for the limits and the sharing rule)."""
    _check(load_library().fathom_scan_topk_static(ctypes.byref(index), _ptr(q_bf16), _ptr(t),
                                                  _ptr(t_union), int(k), _ptr(out_idx),
                                                  _ptr(out_score), int(flags), _stream(stream)),
           "fathom_scan_topk_static")


def _index_array(sessions: Sequence[fathom_index]):
    arr = (fathom_index * len(sessions))()
    for i, s in enumerate(sessions):
        arr[i] = s
    return arr


def fathom_scan_batched_workspace_bytes(sessions: Sequence[fathom_index], k: int) -> int:
    arr = _index_array(sessions)
    return int(load_library().fathom_scan_batched_workspace_bytes(arr, len(sessions), int(k)))


def fathom_scan_topk_batched(sessions: Sequence[fathom_index], q_bf16, t, t_union, k: int,
                             out_idx, out_score, workspace, flags: int = 0, stream=None):
    n = len(sessions)
    arr = _index_array(sessions)
    vp = ctypes.c_void_p * n
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load_library().fathom_scan_topk_batched(
        arr, n, vp(*[_ptr(x) for x in q_bf16]), vp(*[_ptr(x) for x in t]),
        vp(*[_ptr(x) for x in t_union]), int(k), vp(*[_ptr(x) for x in out_idx]),
        vp(*[_ptr(x) for x in out_score]), _ptr(workspace), ws_bytes, int(flags),
        _stream(stream)), "fathom_scan_topk_batched")


def fathom_sparse_attention_workspace_bytes(n_queries: int, head_dim: int, k: int) -> int:
    return int(load_library().fathom_sparse_attention_workspace_bytes(int(n_queries),
                                                                       int(head_dim), int(k)))


def fathom_sparse_attention(keys, values, n_kv_heads: int, group: int, head_dim: int,
                            n_keys: int, q_bf16, idx, k: int, softmax_scale: float, out,
                            workspace, stream=None):
    """Softmax attention of each query over its k selected keys (fp32)."""
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load_library().fathom_sparse_attention(
        _ptr(keys), _ptr(values), int(n_kv_heads), int(group), int(head_dim), int(n_keys),
        _ptr(q_bf16), _ptr(idx), int(k), float(softmax_scale), _ptr(out), _ptr(workspace),
        ws_bytes, _stream(stream)), "fathom_sparse_attention")


def fathom_merge_topk(shard_idx, shard_score, shard_offset, k: int, out_idx, out_score,
                      stream=None):
    """Exact top-k over S shard lists ([S][Q][k_shard] device tensors) of key
    ranges starting at shard_offset (S ints, ascending)."""
    S, Q, k_s = shard_idx.shape
    offs = (ctypes.c_int64 * S)(*[int(o) for o in shard_offset])
    _check(load_library().fathom_merge_topk(_ptr(shard_idx), _ptr(shard_score), offs, S, Q, k_s,
                                            int(k), _ptr(out_idx), _ptr(out_score),
                                            _stream(stream)), "fathom_merge_topk")


def fathom_last_device_status(stream=None) -> int:
    return int(load_library().fathom_last_device_status(_stream(stream)))


def fathom_link_probe(buffer, nbytes: int, sink, stream=None):
    """Zero-copy read of `nbytes` of a pinned host (or device) buffer."""
    _check(load_library().fathom_link_probe(_ptr(buffer), int(nbytes), _ptr(sink),
                                            _stream(stream)), "fathom_link_probe")


def fathom_launch_count() -> int:
    return int(load_library().fathom_launch_count())


def fathom_profile_read():
    """-> (summed milliseconds of profiled main-scan launches, launches)."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_uint64(0)
    _check(load_library().fathom_profile_read(ctypes.byref(ms), ctypes.byref(n)),
           "fathom_profile_read")
    return ms.value, n.value


# ---------------------------------------------------------- memory plumbing
class KeyIndex:
    """Owns the torch buffers of one packed K index and its C descriptor.

    residency "device" keeps the planes in HBM; "host_mapped" keeps them in
    pinned host memory read zero-copy by the scan.  Statistics stay on the
    device either way.  bits: 4 (the 4-bit K cache) or 8 (the 8-plane
    variant for an 8-bit K cache).  block_keys: 0 for one scale per channel,
    or grouped per-token-block scales over blocks of that many tokens (a
    multiple of 2048); mn, scale, sum_code and sum_code2 are then
    [H][n_blocks][d] with n_blocks counted over the capacity."""

    def __init__(self, n_kv_heads: int, group: int, n_keys: int, head_dim: int = 128,
                 residency: str = "device", device: Optional[int] = None,
                 capacity: Optional[int] = None, bits: int = 4, block_keys: int = 0):
        import torch
        if bits not in (4, 8):
            raise ValueError(f"bits must be 4 or 8, not {bits}")
        if block_keys < 0 or block_keys % 2048:
            raise ValueError(f"block_keys must be 0 or a multiple of 2048, not {block_keys}")
        dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
        self.n_words = fathom_n_words(max(n_keys, capacity or n_keys))
        H, d = n_kv_heads, head_dim
        shape = (H, d, bits, self.n_words)
        if residency == "device":
            self.planes = torch.empty(shape, dtype=torch.int32, device=dev)
            res = FATHOM_RES_DEVICE
        elif residency == "host_mapped":
            self.planes = torch.empty(shape, dtype=torch.int32, pin_memory=True)
            res = FATHOM_RES_HOST_MAPPED
        else:
            raise ValueError(f"unknown residency {residency!r}")
        stat = (H, d)
        if block_keys:
            stat = (H, -(-32 * self.n_words // block_keys), d)
        self.mn = torch.empty(stat, dtype=torch.float32, device=dev)
        self.scale = torch.empty_like(self.mn)
        self.sigma2 = torch.empty((H, d), dtype=torch.float32, device=dev)
        self.sum_code = torch.empty(stat, dtype=torch.int64, device=dev)
        self.sum_code2 = torch.empty_like(self.sum_code)
        self.residency = residency
        self.desc = fathom_index(H, group, d, n_keys, self.n_words, res,
                                 self.planes.data_ptr(), self.mn.data_ptr(),
                                 self.scale.data_ptr(), self.sigma2.data_ptr(),
                                 self.sum_code.data_ptr(), self.sum_code2.data_ptr(), bits,
                                 block_keys)
        self.device = dev

    @property
    def n_kv_heads(self):
        return self.desc.n_kv_heads

    @property
    def group(self):
        return self.desc.group

    @property
    def head_dim(self):
        return self.desc.head_dim

    @property
    def n_keys(self):
        return self.desc.n_keys

    @property
    def bits(self):
        return self.desc.bits

    @property
    def block_keys(self):
        return self.desc.block_keys

    @property
    def capacity(self):
        return 32 * self.n_words

    def append(self, keys, clamped=None, stream=None):
        """Append device float32 keys [H][m][d] (decode-step keys) to this
        index; clamped: optional device uint32 [H][d] drift counters."""
        fathom_append_keys(keys, self.desc, keys.shape[1], clamped, stream)
        return self

    def pack(self, keys, stream=None):
        """Quantise and pack device float32 keys [H][n][d] into this index."""
        import torch
        ws = torch.empty(max(16, fathom_pack_workspace_bytes(self.desc)), dtype=torch.uint8,
                         device=self.device)
        fathom_pack_keys(keys, self.desc, ws, stream)
        return self


class ScanBuffers:
    """Device outputs and workspace for planning and scanning one session."""

    def __init__(self, index: KeyIndex, k: int):
        import torch
        dev = index.device
        Q, H, d = index.n_kv_heads * index.group, index.n_kv_heads, index.head_dim
        self.k = k
        self.t = torch.empty((Q, d), dtype=torch.uint8, device=dev)
        self.t_union = torch.empty((H, d), dtype=torch.uint8, device=dev)
        self.nbytes = torch.empty((Q + H,), dtype=torch.int64, device=dev)
        self.idx = torch.empty((Q, k), dtype=torch.int32, device=dev)
        self.score = torch.empty((Q, k), dtype=torch.float32, device=dev)
        self.workspace = torch.empty(max(16, fathom_scan_workspace_bytes(index.desc, k)),
                                     dtype=torch.uint8, device=dev)


def plan_and_scan(index: KeyIndex, q_bf16, budget, buf: ScanBuffers, flags: int = 0,
                  stream=None, fixed_r: Optional[int] = None):
    """One decode-step scan of a layer: plan (or fixed plan) then scan+top-k."""
    if fixed_r is None:
        fathom_plan(index.desc, q_bf16, budget, buf.t, buf.t_union, buf.nbytes, stream)
    else:
        fathom_fixed_plan(index.desc, q_bf16, fixed_r, buf.t, buf.t_union, buf.nbytes, stream)
    fathom_scan_topk(index.desc, q_bf16, buf.t, buf.t_union, buf.k, buf.idx, buf.score,
                     buf.workspace, flags, stream)
    return buf
