"""CPU oracle for the Fathom per-query read-depth top-k key scan.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The CUDA
library never imports or links it, and it imports nothing from the CUDA
library.  The arithmetic lives in ``fathom_oracle.c`` (plain C, fp64 scores);
this module compiles it with gcc and marshals numpy arrays.

Parity unpinned: ``recall`` (a quality number; the pages print none).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fathom_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_fathom_oracle.so")
_lib = None

OK, ERR_ARG, ERR_NONFINITE = 0, 1, 3


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fused multiply-add, IEEE float)."""
    if (force or not os.path.exists(_LIB_PATH)
            or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off",
                               "-fno-fast-math", "-fPIC", "-shared", "-o", tmp,
                               _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int64
        sig = {
            "fo_quantize": ([P, I, I, I, I, P, P, P], ctypes.c_int),
            "fo_pack_planes": ([P, I, I, I, I, I, P], ctypes.c_int),
            "fo_unpack_planes": ([P, I, I, I, I, I, P], ctypes.c_int),
            "fo_append": ([P, I, I, I, I, I, I, P, P, P, P, P, P, P], ctypes.c_int),
            "fo_channel_stats": ([P, I, I, I, P, P, P, P], ctypes.c_int),
            "fo_blocked_sigma2": ([P, P, P, P, I, I, I, P], ctypes.c_int),
            "fo_importance": ([P, P, I, P], ctypes.c_int),
            "fo_plan_greedy": ([P, I, I, I, P], ctypes.c_int),
            "fo_plan_marginal": ([P, I, I, I, P], ctypes.c_int),
            "fo_fixed_plan": ([P, I, I, I, P], ctypes.c_int),
            "fo_union": ([P, I, I, P], None),
            "fo_plan_bytes": ([P, I, I], ctypes.c_uint64),
            "fo_score_planes": ([P, P, P, P, P, I, I, I, I, P], ctypes.c_int),
            "fo_score_codes": ([P, P, P, P, P, I, I, I, P], ctypes.c_int),
            "fo_score_abs_planes": ([P, P, P, P, P, I, I, I, I, P], ctypes.c_int),
            "fo_exact_scores": ([P, P, I, I, P], None),
            "fo_topk": ([P, I, I, P, P], ctypes.c_int),
            "fo_attention": ([P, P, I, I, P, P, I, ctypes.c_double, P], ctypes.c_int),
            "fo_merge_topk": ([P, P, P, I, I, I, P, P], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != OK:
        raise ValueError(f"oracle {what} failed with code {rc}")


def n_words_for(n: int) -> int:
    """Words per plane: keys rounded up to 128 (16-byte plane rows)."""
    return ((n + 127) // 128) * 4


# ---------------------------------------------------------------- storage side
def quantize(keys: np.ndarray, bits: int = 4):
    """keys float32 [H][n][d] -> (mn [H][d], scale [H][d], codes uint8 [H][d][n]),
    codes of `bits` bits (4: the 4-bit K cache; 8: the 8-plane variant)."""
    keys = np.ascontiguousarray(keys, dtype=np.float32)
    H, n, d = keys.shape
    mn = np.empty((H, d), np.float32)
    scale = np.empty((H, d), np.float32)
    codes = np.empty((H, d, n), np.uint8)
    _check(_load().fo_quantize(_p(keys), H, n, d, int(bits), _p(mn), _p(scale), _p(codes)),
           "quantize")
    return mn, scale, codes


def pack_planes(codes: np.ndarray, n_words: Optional[int] = None, bits: int = 4) -> np.ndarray:
    """codes uint8 [H][d][n] -> planes uint32 [H][d][bits][n_words]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    H, d, n = codes.shape
    n_words = n_words_for(n) if n_words is None else n_words
    planes = np.empty((H, d, int(bits), n_words), np.uint32)
    _check(_load().fo_pack_planes(_p(codes), H, n, d, int(bits), n_words, _p(planes)),
           "pack_planes")
    return planes


def unpack_planes(planes: np.ndarray, n: int) -> np.ndarray:
    """planes uint32 [H][d][bits][n_words] -> codes uint8 [H][d][n]."""
    planes = np.ascontiguousarray(planes, dtype=np.uint32)
    H, d, bits, n_words = planes.shape
    codes = np.empty((H, d, n), np.uint8)
    _check(_load().fo_unpack_planes(_p(planes), H, n, d, bits, n_words, _p(codes)),
           "unpack_planes")
    return codes


def append(index: Dict[str, np.ndarray], keys: np.ndarray, clamped=None):
    """Append keys float32 [H][m][d] to an index dict (build_index's layout)
    in place: planes, s1, s2, sigma2, codes and n are updated; clamped
    (uint32 [H][d], optional) is incremented.  Returns the new key count."""
    keys = np.ascontiguousarray(keys, dtype=np.float32)
    H, m, d = keys.shape
    n = index["n"]
    bits, n_words = index["planes"].shape[-2:]
    for name in ("planes", "s1", "s2", "sigma2"):
        assert index[name].flags["C_CONTIGUOUS"]
    if clamped is not None:
        assert clamped.dtype == np.uint32 and clamped.flags["C_CONTIGUOUS"]
    _check(_load().fo_append(_p(keys), H, n, m, d, bits, n_words, _p(index["mn"]), _p(index["scale"]),
                             _p(index["planes"]), _p(index["s1"]), _p(index["s2"]),
                             _p(index["sigma2"]), None if clamped is None else _p(clamped)),
           "append")
    index["n"] = n + m
    index["codes"] = unpack_planes(index["planes"], n + m)
    return n + m


def channel_stats(codes: np.ndarray, scale: np.ndarray):
    """-> (S1 int64 [H][d], S2 int64 [H][d], sigma2 float32 [H][d])."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    H, d, n = codes.shape
    s1 = np.empty((H, d), np.int64)
    s2 = np.empty((H, d), np.int64)
    sigma2 = np.empty((H, d), np.float32)
    _check(_load().fo_channel_stats(_p(codes), H, n, d, _p(scale), _p(s1), _p(s2),
                                    _p(sigma2)), "channel_stats")
    return s1, s2, sigma2


def blocked_sigma2(mn_h, scale_h, s1_h, s2_h, n: int, block: int) -> np.ndarray:
    """sigma^2 [d] of one KV head of a block-scaled index: the variance of
    all n dequantised keys from the blocks' sums (mn_h ... s2_h [nb][d])."""
    mn_h = np.ascontiguousarray(mn_h, np.float32)
    d = mn_h.shape[-1]
    out = np.empty(d, np.float32)
    _check(_load().fo_blocked_sigma2(_p(mn_h), _p(np.ascontiguousarray(scale_h, np.float32)),
                                     _p(np.ascontiguousarray(s1_h, np.int64)),
                                     _p(np.ascontiguousarray(s2_h, np.int64)), d, int(n),
                                     int(block), _p(out)), "blocked_sigma2")
    return out


def n_blocks_for(n: int, block: int) -> int:
    return (n + block - 1) // block


# ------------------------------------------------------------------- read side
def importance(q_bf16: np.ndarray, sigma2: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
    s2 = np.ascontiguousarray(sigma2, dtype=np.float32)
    d = q.shape[-1]
    w = np.empty(d, np.float32)
    _check(_load().fo_importance(_p(q), _p(s2), d, _p(w)), "importance")
    return w


def plan_greedy(w: np.ndarray, B: int, bits: int = 4) -> np.ndarray:
    """Reverse water-filling with at most `bits` bits per channel."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    t = np.empty(w.shape[0], np.uint8)
    _check(_load().fo_plan_greedy(_p(w), w.shape[0], int(B), int(bits), _p(t)), "plan_greedy")
    return t


def plan_marginal(w: np.ndarray, B: int, bits: int = 4) -> np.ndarray:
    """Marginal-gain plan: bits one at a time to the largest w_c * 4^-t_c."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    t = np.empty(w.shape[0], np.uint8)
    _check(_load().fo_plan_marginal(_p(w), w.shape[0], int(B), int(bits), _p(t)),
           "plan_marginal")
    return t


def fixed_plan(q_bf16: np.ndarray, r: int, bits: int = 4) -> np.ndarray:
    q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
    t = np.empty(q.shape[0], np.uint8)
    _check(_load().fo_fixed_plan(_p(q), q.shape[0], int(r), int(bits), _p(t)), "fixed_plan")
    return t


def union(t_group: np.ndarray) -> np.ndarray:
    t = np.ascontiguousarray(t_group, dtype=np.uint8)
    G, d = t.shape
    T = np.empty(d, np.uint8)
    _load().fo_union(_p(t), G, d, _p(T))
    return T


def plan_bytes(t: np.ndarray, n_words: int) -> int:
    t = np.ascontiguousarray(t, dtype=np.uint8)
    return int(_load().fo_plan_bytes(_p(t), t.shape[0], int(n_words)))


def score_planes(planes_h, mn_h, scale_h, q_bf16, t, n: int) -> np.ndarray:
    planes_h = np.ascontiguousarray(planes_h, dtype=np.uint32)
    d, bits, n_words = planes_h.shape
    mn_h = np.ascontiguousarray(mn_h, np.float32)
    scale_h = np.ascontiguousarray(scale_h, np.float32)
    q = np.ascontiguousarray(q_bf16, np.uint16)
    t = np.ascontiguousarray(t, np.uint8)
    s = np.empty(n, np.float64)
    _check(_load().fo_score_planes(_p(planes_h), _p(mn_h), _p(scale_h), _p(q), _p(t),
                                   d, bits, n, n_words, _p(s)), "score_planes")
    return s


def score_abs_planes(planes_h, mn_h, scale_h, q_bf16, t, n: int) -> np.ndarray:
    planes_h = np.ascontiguousarray(planes_h, dtype=np.uint32)
    d, bits, n_words = planes_h.shape
    a = np.empty(n, np.float64)
    _check(_load().fo_score_abs_planes(
        _p(planes_h), _p(np.ascontiguousarray(mn_h, np.float32)),
        _p(np.ascontiguousarray(scale_h, np.float32)),
        _p(np.ascontiguousarray(q_bf16, np.uint16)), _p(np.ascontiguousarray(t, np.uint8)),
        d, bits, n, n_words, _p(a)), "score_abs_planes")
    return a


def score_codes(codes_h, mn_h, scale_h, q_bf16, t, bits: int = 4) -> np.ndarray:
    codes_h = np.ascontiguousarray(codes_h, dtype=np.uint8)
    d, n = codes_h.shape
    s = np.empty(n, np.float64)
    _check(_load().fo_score_codes(
        _p(codes_h), _p(np.ascontiguousarray(mn_h, np.float32)),
        _p(np.ascontiguousarray(scale_h, np.float32)),
        _p(np.ascontiguousarray(q_bf16, np.uint16)), _p(np.ascontiguousarray(t, np.uint8)),
        d, int(bits), n, _p(s)), "score_codes")
    return s


def exact_scores(keys_h: np.ndarray, q_bf16: np.ndarray) -> np.ndarray:
    keys_h = np.ascontiguousarray(keys_h, dtype=np.float32)
    n, d = keys_h.shape
    s = np.empty(n, np.float64)
    _load().fo_exact_scores(_p(keys_h), _p(np.ascontiguousarray(q_bf16, np.uint16)), n, d, _p(s))
    return s


def topk(s: np.ndarray, k: int):
    """-> (idx int32 [k], score float64 [k]) by (score desc, index asc)."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    idx = np.empty(k, np.int32)
    top = np.empty(k, np.float64)
    _check(_load().fo_topk(_p(s), s.shape[0], int(k), _p(idx), _p(top)), "topk")
    return idx, top


def recall(selected, reference) -> float:
    """|S intersect S*| / |S*|.  Parity unpinned: a quality number only."""
    ref = set(int(x) for x in np.asarray(reference).ravel())
    got = set(int(x) for x in np.asarray(selected).ravel())
    return len(ref & got) / max(1, len(ref))


# --------------------------------------------------------------- whole pipeline
def build_index(keys: np.ndarray, capacity: Optional[int] = None,
                bits: int = 4, block_keys: int = 0) -> Dict[str, np.ndarray]:
    """Storage side for one session: quantise, pack, channel statistics.
    capacity: keys the planes can hold (for appends); default n.
    bits: planes per channel (4, or 8 for an 8-bit K cache).
    block_keys: 0 for one scale per channel over all keys; else grouped
    per-token-block scales, each block of block_keys tokens quantised on
    its own (mn, scale, s1, s2 then hold [H][n_blocks][d], n_blocks counted
    over the capacity; blocks past the keys stay zero)."""
    n = keys.shape[1]
    n_words = n_words_for(max(n, capacity or n))
    if not block_keys:
        mn, scale, codes = quantize(keys, bits)
        planes = pack_planes(codes, n_words, bits)
        s1, s2, sigma2 = channel_stats(codes, scale)
        return dict(mn=mn, scale=scale, codes=codes, planes=planes, s1=s1, s2=s2,
                    sigma2=sigma2, n=n, n_words=n_words, bits=int(bits), block_keys=0)
    H, _, d = keys.shape
    nb_cap = n_blocks_for(32 * n_words, block_keys)
    mn = np.zeros((H, nb_cap, d), np.float32)
    scale = np.zeros_like(mn)
    s1 = np.zeros((H, nb_cap, d), np.int64)
    s2 = np.zeros_like(s1)
    codes = np.empty((H, d, n), np.uint8)
    for b in range(n_blocks_for(n, block_keys)):
        j0, j1 = b * block_keys, min(n, (b + 1) * block_keys)
        mn[:, b], scale[:, b], codes[:, :, j0:j1] = quantize(keys[:, j0:j1], bits)
        s1[:, b], s2[:, b], _ = channel_stats(codes[:, :, j0:j1], scale[:, b])
    planes = pack_planes(codes, n_words, bits)
    sigma2 = np.stack([blocked_sigma2(mn[h], scale[h], s1[h], s2[h], n, block_keys)
                       for h in range(H)])
    return dict(mn=mn, scale=scale, codes=codes, planes=planes, s1=s1, s2=s2,
                sigma2=sigma2, n=n, n_words=n_words, bits=int(bits), block_keys=int(block_keys))


def append_blocks(index: Dict[str, np.ndarray], keys: np.ndarray) -> int:
    """Append keys float32 [H][m][d] to a block-scaled index whose key count
    is a whole number of blocks: each new block is quantised on its own, as
    packing all keys would.  Returns the new key count."""
    block = index["block_keys"]
    n = index["n"]
    assert block and n % block == 0, "appends start a new block"
    H, m, d = keys.shape
    bits, n_words = index["planes"].shape[-2:]
    assert n + m <= 32 * n_words
    new_codes = np.empty((H, d, m), np.uint8)
    for i0 in range(0, m, block):
        b = (n + i0) // block
        i1 = min(m, i0 + block)
        mb, sb, cb = quantize(keys[:, i0:i1], bits)
        index["mn"][:, b], index["scale"][:, b] = mb, sb
        index["s1"][:, b], index["s2"][:, b], _ = channel_stats(cb, sb)
        new_codes[:, :, i0:i1] = cb
    words = pack_planes(new_codes, None, bits)
    w0 = n // 32
    nw = min(words.shape[-1], n_words - w0)
    index["planes"][..., w0:w0 + nw] |= words[..., :nw]
    index["n"] = n + m
    index["codes"] = np.concatenate([index["codes"], new_codes], axis=2)
    for h in range(H):
        index["sigma2"][h] = blocked_sigma2(index["mn"][h], index["scale"][h], index["s1"][h],
                                            index["s2"][h], n + m, block)
    return n + m


def plan_session(index, q_bf16: np.ndarray, budgets: np.ndarray, group: int,
                 fixed_r: Optional[int] = None, marginal: bool = False):
    """-> (t uint8 [Q][d], T uint8 [H][d], bytes uint64 [Q+H])."""
    H, d = index["sigma2"].shape
    bits = index["planes"].shape[-2]
    Q = H * group
    t = np.empty((Q, d), np.uint8)
    for q in range(Q):
        h = q // group
        if fixed_r is not None:
            t[q] = fixed_plan(q_bf16[q], fixed_r, bits)
        elif marginal:
            t[q] = plan_marginal(importance(q_bf16[q], index["sigma2"][h]), int(budgets[q]), bits)
        else:
            t[q] = plan_greedy(importance(q_bf16[q], index["sigma2"][h]), int(budgets[q]), bits)
    T = np.stack([union(t[h * group:(h + 1) * group]) for h in range(H)])
    nb = np.array([plan_bytes(t[q], index["n_words"]) for q in range(Q)]
                  + [plan_bytes(T[h], index["n_words"]) for h in range(H)], np.uint64)
    return t, T, nb


def _head_blocks(index, h: int):
    """(key range, planes, mn, scale) of each scale block of KV head h."""
    n, block = index["n"], index.get("block_keys", 0)
    if not block:
        return [((0, n), index["planes"][h], index["mn"][h], index["scale"][h])]
    out = []
    for b in range(n_blocks_for(n, block)):
        j0, j1 = b * block, min(n, (b + 1) * block)
        w0, w1 = j0 // 32, (j1 + 31) // 32           # the block's own plane words
        out.append(((j0, j1), np.ascontiguousarray(index["planes"][h][..., w0:w1]),
                    index["mn"][h, b], index["scale"][h, b]))
    return out


def score_head(index, h: int, q_bf16_row, t_row, absolute: bool = False) -> np.ndarray:
    """Scores [n] of one query against KV head h from its plan t (each key
    with the scales of its block); absolute=True gives sum_c |q_c khat_cj|."""
    fn = score_abs_planes if absolute else score_planes
    parts = [fn(planes, mn, sc, q_bf16_row, t_row, j1 - j0)
             for (j0, j1), planes, mn, sc in _head_blocks(index, h)]
    return np.concatenate(parts)


def scan_query(index, q_bf16_row, t_row, h: int, k: int):
    """Score one query against KV head h and select its top-k.
    -> (idx [k], top scores [k], all scores [n])."""
    s = score_head(index, h, q_bf16_row, t_row)
    idx, top = topk(s, k)
    return idx, top, s


# ------------------------------------------------------------------ after the scan
def attention(keys_h: np.ndarray, values_h: np.ndarray, q_bf16_row: np.ndarray, idx=None,
              scale: Optional[float] = None) -> np.ndarray:
    """fp64 softmax attention of one query over keys idx (all keys if None).
    keys_h, values_h float32 [n][d]; scale defaults to 1/sqrt(d)."""
    keys_h = np.ascontiguousarray(keys_h, np.float32)
    values_h = np.ascontiguousarray(values_h, np.float32)
    n, d = keys_h.shape
    q = np.ascontiguousarray(q_bf16_row, np.uint16)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    out = np.empty(d, np.float64)
    if idx is None:
        rc = _load().fo_attention(_p(keys_h), _p(values_h), n, d, _p(q), None, 0, scale, _p(out))
    else:
        ii = np.ascontiguousarray(idx, np.int32)
        rc = _load().fo_attention(_p(keys_h), _p(values_h), n, d, _p(q), _p(ii), ii.shape[0],
                                  scale, _p(out))
    _check(rc, "attention")
    return out


def attention_error(o: np.ndarray, o_exact: np.ndarray) -> float:
    """Relative L2 error ||o - o_exact|| / ||o_exact|| (the pages name an
    attention error but give no formula; this is the reading used)."""
    o = np.asarray(o, np.float64)
    o_exact = np.asarray(o_exact, np.float64)
    return float(np.linalg.norm(o - o_exact) / np.linalg.norm(o_exact))


# ------------------------------------------------------------ sharded keys
def merge_topk(idx, score, offset, k: int):
    """Exact top-k over S shard lists (idx int32 [S][k_s] local, score [S][k_s],
    offset [S]): -> (global idx ascending [k], scores [k])."""
    idx = np.ascontiguousarray(idx, np.int32)
    score = np.ascontiguousarray(score, np.float64)
    offset = np.ascontiguousarray(offset, np.int64)
    S, k_s = idx.shape
    out_i = np.empty(k, np.int32)
    out_s = np.empty(k, np.float64)
    _check(_load().fo_merge_topk(_p(idx), _p(score), _p(offset), S, k_s, int(k), _p(out_i),
                                 _p(out_s)), "merge_topk")
    return out_i, out_s
