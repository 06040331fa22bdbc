"""Seeded synthetic inputs for the Fathom key scan.

This module only draws random inputs; it holds none of the scan's arithmetic
(no quantisation, planning, scoring or selection).  Both the CPU oracle tests
and the CUDA path consume exactly what it returns.

The pages describe the workloads (Qwen3-8B, 1M-token decode, multi-session
coding agents) but ship no data, so keys and queries are drawn here with the
shapes of a Qwen3-8B layer: 8 KV heads, 4 query heads per KV head, head_dim
128.  Recipe, per session, from one ``numpy.random.Generator(PCG64(seed))``
in this fixed order:

1. per-channel scale sigma[h][c] ~ lognormal(0, 0.5);
2. per KV head, 4 distinct outlier channels (``choice(d, 4, replace=False)``)
   whose sigma is multiplied by 10;
3. keys[h][j][c] = N(0, 1) * sigma[h][c], drawn in C order as float64 and
   rounded to float32;
4. queries q[Q][d] = N(0, 1) rounded to bfloat16 (round to nearest even);
5. optionally, planted keys: per KV head ``choice(n, planted, replace=False)``
   positions whose key is set to the head's first query + N(0, 0.1).

Multi-session batches draw each session from seed ``base + s``; the session's
key count n and bit budget B are drawn first from that session's generator.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

HEAD_DIM = 128
N_OUTLIERS = 4
OUTLIER_MULT = 10.0
SIGMA_LOGNORMAL = 0.5
PLANTED_NOISE = 0.1

# Rows drawn per numpy call while generating keys; drawing in C-order chunks
# yields the same stream as one large draw, so this only bounds host memory.
_CHUNK_ROWS = 1 << 16


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the
    16-bit patterns as uint16.  NaN inputs are not expected here."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Session:
    """One independent scan problem: H KV heads x G query heads over n keys."""
    seed: int
    n_kv_heads: int
    group: int
    n_keys: int
    head_dim: int
    sigma: np.ndarray            # float64 [H][d] (outliers applied)
    outliers: np.ndarray         # int64 [H][N_OUTLIERS]
    keys: np.ndarray             # float32 [H][n][d]
    q_bf16: np.ndarray           # uint16 [H*G][d]
    budgets: np.ndarray          # int32 [H*G]
    planted: Optional[np.ndarray] = None   # int64 [H][n_planted] or None
    meta: dict = field(default_factory=dict)

    @property
    def n_queries(self) -> int:
        return self.n_kv_heads * self.group

    @property
    def q_f32(self) -> np.ndarray:
        return bf16_bits_to_f32(self.q_bf16)


def _draw_keys(rng: np.random.Generator, sigma: np.ndarray, n: int) -> np.ndarray:
    H, d = sigma.shape
    keys = np.empty((H, n, d), dtype=np.float32)
    for h in range(H):
        for j0 in range(0, n, _CHUNK_ROWS):
            j1 = min(n, j0 + _CHUNK_ROWS)
            z = rng.standard_normal((j1 - j0, d))
            keys[h, j0:j1] = (z * sigma[h][None, :]).astype(np.float32)
    return keys


def channel_sigma(seed: int, n_kv_heads: int, head_dim: int = HEAD_DIM,
                  rng: Optional[np.random.Generator] = None):
    """Steps 1-2 of the recipe alone (the first draws of make_session):
    -> (sigma float64 [H][d] with outliers applied, outliers int64 [H][4])."""
    if rng is None:
        rng = np.random.Generator(np.random.PCG64(seed))
    sigma = rng.lognormal(0.0, SIGMA_LOGNORMAL, size=(n_kv_heads, head_dim))
    outliers = np.empty((n_kv_heads, N_OUTLIERS), dtype=np.int64)
    for h in range(n_kv_heads):
        outliers[h] = rng.choice(head_dim, N_OUTLIERS, replace=False)
        sigma[h, outliers[h]] *= OUTLIER_MULT
    return sigma, outliers


def device_keys(torch, sigma: np.ndarray, n: int, seed: int, device="cuda"):
    """Keys of step 3 drawn on a device: N(0, 1) from torch's generator on
    `device` seeded with `seed`, times sigma, as float32 [H][n][d].  This is
    a different random stream from step 3's numpy draw (same distribution);
    the benchmark uses it for workloads whose keys would take minutes and
    tens of GB to draw on the host."""
    H, d = sigma.shape
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    sig = torch.as_tensor(sigma, dtype=torch.float32, device=device)
    keys = torch.empty((H, n, d), dtype=torch.float32, device=device)
    for h in range(H):
        keys[h] = torch.randn((n, d), generator=gen, device=device, dtype=torch.float32) * sig[h]
    return keys


def agent_session_params(n_sessions: int = 16, base_seed: int = 1000, n_kv_heads: int = 8,
                         n_min: int = 65536, n_max: int = 524288,
                         budget_choices=(68, 92, 136), head_dim: int = HEAD_DIM):
    """The draws of make_agent_sessions that precede the keys: per session s
    (seed base_seed + s) its key count n, budget B, sigma and outliers.
    -> list of dicts {seed, n, budget, sigma, outliers}."""
    out = []
    for s in range(n_sessions):
        rng = np.random.Generator(np.random.PCG64(base_seed + s))
        n = int(rng.integers(n_min, n_max, endpoint=True))
        B = int(rng.choice(np.asarray(budget_choices)))
        sigma, outliers = channel_sigma(base_seed + s, n_kv_heads, head_dim, rng=rng)
        out.append(dict(seed=base_seed + s, n=n, budget=B, sigma=sigma, outliers=outliers))
    return out


def make_session(seed: int, n_kv_heads: int, group: int, n_keys: int,
                 budget, head_dim: int = HEAD_DIM, n_planted: int = 0,
                 rng: Optional[np.random.Generator] = None) -> Session:
    """Draw one session.  ``budget`` is an int (same B for every query head)
    or a sequence of Q ints."""
    if rng is None:
        rng = np.random.Generator(np.random.PCG64(seed))
    H, G, n, d = n_kv_heads, group, n_keys, head_dim
    sigma, outliers = channel_sigma(seed, H, d, rng=rng)
    keys = _draw_keys(rng, sigma, n)
    q32 = rng.standard_normal((H * G, d)).astype(np.float32)
    q_bf16 = f32_to_bf16_bits(q32)
    planted = None
    if n_planted:
        planted = np.empty((H, n_planted), dtype=np.int64)
        qf = bf16_bits_to_f32(q_bf16).astype(np.float64)
        for h in range(H):
            planted[h] = rng.choice(n, n_planted, replace=False)
            noise = rng.standard_normal((n_planted, d)) * PLANTED_NOISE
            keys[h, planted[h]] = (qf[h * G][None, :] + noise).astype(np.float32)
    if np.isscalar(budget):
        budgets = np.full(H * G, int(budget), dtype=np.int32)
    else:
        budgets = np.asarray(budget, dtype=np.int32).reshape(H * G)
    return Session(seed=seed, n_kv_heads=H, group=G, n_keys=n, head_dim=d,
                   sigma=sigma, outliers=outliers, keys=keys, q_bf16=q_bf16,
                   budgets=budgets, planted=planted)


def make_agent_sessions(n_sessions: int = 16, base_seed: int = 1000,
                        n_kv_heads: int = 8, group: int = 4,
                        n_min: int = 65536, n_max: int = 524288,
                        budget_choices=(68, 92, 136),
                        head_dim: int = HEAD_DIM) -> List[Session]:
    """Multi-session agent batch: session s uses seed base_seed + s; its key
    count n ~ U[n_min, n_max] (inclusive) and its budget B (shared by all of
    its query heads) are drawn first, then the session as in make_session."""
    out = []
    for s in range(n_sessions):
        rng = np.random.Generator(np.random.PCG64(base_seed + s))
        n = int(rng.integers(n_min, n_max, endpoint=True))
        B = int(rng.choice(np.asarray(budget_choices)))
        ses = make_session(base_seed + s, n_kv_heads, group, n, B,
                           head_dim=head_dim, rng=rng)
        ses.meta["budget"] = B
        out.append(ses)
    return out


# Named workloads, with the sizes of the pages' experiments.
def tiny_4k(seed: int = 0) -> Session:
    """1 KV head x 1 query head, head_dim 128, 4096 keys, 16 planted keys,
    B = 64 bits/key (k = 64)."""
    return make_session(seed, 1, 1, 4096, 64, n_planted=16)


def qwen3_8b_layer(n_keys: int = 131072, budget: int = 92, seed: int = 0) -> Session:
    """One Qwen3-8B-shaped layer: 8 KV heads x 4 query heads, head_dim 128."""
    return make_session(seed, 8, 4, n_keys, budget)


WORKLOADS = {
    "tiny_4k": dict(H=1, G=1, n=4096, budgets=(64,), k=64, residency="device"),
    "qwen3_8b_layer_128k": dict(H=8, G=4, n=131072, budgets=(68, 92, 136), k=2048,
                                residency="device"),
    "host_1m": dict(H=8, G=4, n=1 << 20, budgets=(18, 68, 92, 136), k=2048,
                    residency="host_mapped"),
    "agent_16_sessions": dict(H=8, G=4, n=None, budgets=(68, 92, 136), k=1024,
                              residency="host_mapped"),
    "fixed_vs_wf_1m": dict(H=8, G=4, n=1 << 20, budgets=(68, 92), fixed_r=(34, 17),
                           k=2048, residency="host_mapped"),
}


def draw_queries(seed: int, n_queries: int, head_dim: int = HEAD_DIM, count: int = 1) -> np.ndarray:
    """`count` further query sets (one per decode step) with the recipe's
    query distribution: N(0, 1) rounded to bfloat16.  -> uint16 [count][Q][d]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = rng.standard_normal((count, n_queries, head_dim)).astype(np.float32)
    return f32_to_bf16_bits(q).reshape(count, n_queries, head_dim)
