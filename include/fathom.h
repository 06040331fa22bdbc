/*
 * fathom.h -- C ABI of the B200 (sm_100a) Fathom per-query read-depth
 * top-k key scan.
 *
 * The method: "Fathom：面向卸载 KV 缓存稀疏解码的每查询读取深度" (the
 * papers.ananclaw.com explainer of arXiv 2609.17652), section 核心方法:
 *   storage side (存储侧) -- the K cache is quantised to 4 bits and stored
 *     channel-major as bit planes; the first t planes of a channel are its
 *     t-bit quantiser;
 *   read side (读侧) -- each query spends a per-key bit budget B over the
 *     channels by reverse water-filling on the importance w_c, up to 4 bits
 *     per channel, letting unimportant channels take 0 bits; bytes read =
 *     sum_c t_c * bytes_per_plane;
 * and section 解决什么真问题: every decode step ranks n keys and keeps the
 * top-k.
 *
 * A decode step of one layer, all calls on one stream with no host sync
 * between them (the sequence may be captured in a CUDA graph):
 *   fathom_pack_keys once per index, fathom_append_keys as keys arrive;
 *   fathom_plan (or fathom_plan_marginal / fathom_fixed_plan) per step;
 *   fathom_scan_topk (workspace sized by fathom_scan_workspace_bytes);
 *   optionally fathom_sparse_attention over the returned key indices;
 * then, after a synchronisation, fathom_last_device_status() reports any
 * error only the device could see.
 *
 * Conventions for every call:
 *   - All buffers are owned by the caller.  The library allocates no device
 *     or host memory; scratch space is a caller-supplied workspace sized by
 *     the matching *_workspace_bytes call (16-byte aligned).  The one
 *     exception is the fixed scratch array behind fathom_scan_topk_static.
 *   - Per-device state is set up on the first call that needs it and kept
 *     until the process exits: the status word's address, the raised
 *     shared-memory limits of the kernels, and the side stream of
 *     host-resident scans.  A cudaDeviceReset discards what it refers to, so
 *     make no call on a device after resetting it in the same process.
 *   - Calls are stream-ordered and asynchronous: they validate what the host
 *     can see, enqueue kernels on `stream` and return.  Argument errors are
 *     returned at once and enqueue nothing.  Errors that only the device can
 *     see (a non-finite key or importance, a budget out of range) are
 *     recorded in a per-device status word read by
 *     fathom_last_device_status().
 *   - Layouts (H = KV heads, G = query heads per KV head, Q = H*G,
 *     d = head_dim, n = keys, n_words = words per plane, b = bits per
 *     stored code: 4, or 8 for the 8-plane variant):
 *       keys      float32 [H][n][d]            (token-major, as a K cache)
 *       planes    uint32  [H][d][b][n_words]   slot s holds bit b-1-s of
 *                 the b-bit code (slot 0 = most significant); bit i of word
 *                 w belongs to key 32*w+i; words past the last key are zero
 *       mn, scale, sigma2  float32 [H][d]; sum_code, sum_code2 int64 [H][d]
 *                 -- with grouped per-token-block scales (block_keys > 0)
 *                 mn, scale, sum_code and sum_code2 are [H][n_blocks][d],
 *                 n_blocks = ceil(32*n_words / block_keys), key j belonging
 *                 to block j / block_keys; sigma2 stays [H][d]
 *       q         bfloat16 bits (uint16) [Q][d], query q served by KV head
 *                 q / G
 *       budget    int32 [Q] bits per key, 0 <= B <= b*d
 *       t         uint8 [Q][d] bits read per channel (0..b);
 *                 t_union uint8 [H][d]
 *       bytes     uint64 [Q + H]: per query, then per KV head (union)
 *       out_idx   int32 [Q][k], out_score float32 [Q][k]: the k keys of
 *                 largest score (ties to the lower key index), listed in
 *                 ascending key index (the order a gather of their K/V rows
 *                 wants), each with its score
 *   - head_dim is a multiple of 32 and at most 256 (at most 128 when
 *     b = 8); G is 1..8; n_words is a multiple of 4 (16-byte plane rows)
 *     with 32*n_words >= n and 32*n_words <= 2^27 keys (2^23 when b = 8, so
 *     that n*sum_code2 fits in 64 bits); 1 <= k <= min(n, 4096).
 *   - The 8-plane variant (b = 8) is the adaptation the explainer's
 *     deployment notes (部署前必读, item 3) call for when the upstream K
 *     cache is 8-bit: the same quantiser with 255 levels, plans capped at 8
 *     bits per channel, the same coarse-bin rebuild.
 *   - Grouped per-token-block scales (block_keys > 0, a multiple of 2048):
 *     the index is the grouped quantised K of a serving stack (the
 *     explainer, 亮点 / 适用边界: Fathom reads the 4-bit K the stack already
 *     holds); every block of block_keys tokens of a channel is quantised on
 *     its own, and a key is rebuilt with its block's mn and scale.
 */
#ifndef FATHOM_H
#define FATHOM_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FATHOM_OK = 0,
    FATHOM_ERR_INVALID_ARG = 1,   /* bad pointer, size or layout            */
    FATHOM_ERR_CUDA = 2,          /* a CUDA runtime call failed             */
    FATHOM_ERR_NONFINITE = 3,     /* non-finite key, query or importance    */
    FATHOM_ERR_TIMEOUT = 4,       /* a bounded device wait ran out          */
    FATHOM_ERR_WORKSPACE = 5,     /* workspace missing or too small         */
    FATHOM_ERR_UNIMPLEMENTED = 6  /* a mode the library does not provide    */
} fathom_status;

/* Where the planes live.  DEVICE: HBM.  HOST_MAPPED: pinned, device-mapped
 * host memory (the explainer's setting: the 4-bit K index is offloaded to
 * host memory).  A scan of a HOST_MAPPED index moves only the planes its
 * union plan selects over the host link, one unit of KV heads at a time (one
 * head for a single index, one index for a batched call), into a two-slot
 * device ring held in the workspace: unit u + 1 is fetched on a side stream
 * while unit u is scored from the other slot.  The workspace therefore holds
 * two units' planes (2 * heads_per_unit * d*4*n_words*4 bytes) plus one
 * unit's scan scratch, not the whole index.  The side stream and its events
 * are created on the first such call for a (device, stream) pair and kept
 * until the process exits (make that first call before a stream capture,
 * and make no such call across a cudaDeviceReset); they fork from and join
 * the caller's stream within the call (event waits only), so a captured
 * call stays a CUDA graph on the caller's stream. */
typedef enum {
    FATHOM_RES_DEVICE = 0,
    FATHOM_RES_HOST_MAPPED = 1
} fathom_residency;

/* A packed K index of one session (one layer).  Plain descriptor; every
 * pointer is caller-owned.  planes is a device pointer (DEVICE) or a pinned,
 * device-mapped host pointer (HOST_MAPPED); the statistics are device
 * pointers.  bits is the code width b: 4 (the 4-bit K cache) or 8 (the
 * 8-plane variant); 0 is read as 4, so a zero-initialised field keeps the
 * 4-bit index. */
typedef struct {
    int32_t n_kv_heads;       /* H */
    int32_t group;            /* G query heads per KV head */
    int32_t head_dim;         /* d */
    int32_t n_keys;           /* n */
    int32_t n_words;          /* words per plane */
    int32_t residency;        /* fathom_residency */
    uint32_t *planes;         /* [H][d][b][n_words] */
    float *mn;                /* [H][d] channel minimum */
    float *scale;             /* [H][d] (max - min) / (2^b - 1), 0 if max == min */
    float *sigma2;            /* [H][d] variance of the dequantised keys */
    int64_t *sum_code;        /* [H][d] sum of codes */
    int64_t *sum_code2;       /* [H][d] sum of squared codes */
    int32_t bits;             /* b: 4 or 8 (0 means 4) */
    int32_t block_keys;       /* 0, or tokens per scale block (a multiple of 2048) */
} fathom_index;

/* Scan flags. */
#define FATHOM_SCAN_DEFAULT 0u
/* Skip the sampled candidate threshold and select every query's top-k with
 * the exact multi-pass radix select (the path the fast path falls back to). */
#define FATHOM_SCAN_FORCE_EXACT 1u
/* Record CUDA events around the dominant work of the call (benchmarking
 * only): for a HOST_MAPPED index the fetch sequence (from the first KV head's
 * fetch to the end of the last one's, on the side stream), else the main
 * scan kernel. */
#define FATHOM_SCAN_PROFILE 2u

/* Words per plane for n keys: n rounded up to 128 keys, i.e. 16-byte rows. */
int32_t fathom_n_words(int32_t n_keys);

/* Human-readable name of a status. */
const char *fathom_status_str(fathom_status status);

/* ---------------------------------------------------------------------- */
/* Storage side.                                                          */
/* ---------------------------------------------------------------------- */

/* Workspace bytes fathom_pack_keys needs for `index` (8*H*d). */
size_t fathom_pack_workspace_bytes(const fathom_index *index);

/* Quantise keys to b bits per (KV head, channel) and write the bit planes
 * and channel statistics into `index` (explainer, 核心方法 / 存储侧).
 * Per (h, c) over all n keys: mn = min, scale = (max-min)/L with
 * L = 2^b - 1 (0 if the channel is constant), code = clamp(floor((k-mn)/scale
 * + 0.5), 0, L) in IEEE float32; sum_code, sum_code2 exact;
 * sigma2 = scale^2*(n*S2-S1^2)/n^2 in fp64 rounded to float32 (the variance
 * of the stored b-bit keys, the
 * importance weight the read side uses).
 * keys: device float32 [H][n][d].  Every output array of `index` is
 * written; planes may be a mapped host pointer (written zero-copy).
 * With grouped scales the min, scale and sums are per (h, block, c), each
 * block over its own keys (the last one may be short), and sigma2 is the
 * variance of all n dequantised keys: each block's mean and squared
 * deviations from its exact sums, combined block by block in fp64 with
 * the pairwise update of Chan, Golub and LeVeque; the workspace is then
 * unused (the accumulators live in mn and scale).
 * A non-finite key sets FATHOM_ERR_NONFINITE in the device status. */
fathom_status fathom_pack_keys(const float *keys, const fathom_index *index,
                               void *workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/* Append m new keys per KV head at positions n..n+m-1 of an index holding
 * n = index->n_keys keys: the decode step's keys entering the b-bit K
 * cache the read side scans (explainer, 核心方法 / 存储侧; the cache comes
 * from the serving stack, 适用边界).  Each new key is quantised with the
 * index's stored mn and scale exactly as fathom_pack_keys quantises, its
 * level clamped to 0..2^b-1 (a key outside the stored range takes the nearest
 * level; a constant channel stores code 0); its bits go to key positions
 * n..n+m-1 of the planes; sum_code, sum_code2 grow by the new codes and
 * sigma2 is recomputed for n+m keys.  Keys inside the stored range give
 * exactly the index that packing all n+m keys would.
 * keys: device float32 [H][m][d].  clamped: optional (may be NULL) device
 * uint32 [H][d], incremented by the number of new keys whose level was
 * clamped (for a constant channel: keys other than mn) -- the range-drift
 * measure; re-pack with fathom_pack_keys when a channel's count passes the
 * caller's tolerance.  Requires n + m <= 32*n_words, with the plane words
 * past key n zero (as fathom_pack_keys and earlier appends leave them);
 * planes may be a mapped host pointer.  On success index->n_keys grows by
 * m (host field).  A non-finite key stores code 0 and sets
 * FATHOM_ERR_NONFINITE in the device status.
 * Grouped scales: n must be a whole number of blocks (the serving stack
 * hands over a block once it is full); the m keys open new blocks, each
 * quantised on its own exactly as fathom_pack_keys would, sigma2 is
 * recombined, and `clamped` is not touched (nothing is clamped). */
fathom_status fathom_append_keys(fathom_index *index, const float *keys, int32_t m,
                                 uint32_t *clamped, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Read side: plans.                                                      */
/* ---------------------------------------------------------------------- */

/* Reverse water-filling (explainer, 核心方法 / 读侧): for each query,
 * w_c = (q_c*q_c)*sigma2_c in float32; channels are visited by w descending
 * (ties to the lower channel) and each takes min(b, remaining budget) bits,
 * so t_c = min(b, max(0, B - b*rank_c)) and sum_c t_c = B.  Also writes the
 * GQA union t_union[h][c] = max over the G queries of KV head h, and the
 * bytes each query (and each KV head's union) reads: sum_c t_c * 4*n_words.
 * q_bf16, budget, t, t_union, bytes: device pointers.
 * A budget outside [0, b*d] sets FATHOM_ERR_INVALID_ARG in the device status
 * (that query reads nothing); a non-finite w sets FATHOM_ERR_NONFINITE. */
fathom_status fathom_plan(const fathom_index *index, const uint16_t *q_bf16,
                          const int32_t *budget, uint8_t *t, uint8_t *t_union,
                          uint64_t *bytes, cudaStream_t stream);

/* Marginal-gain plan, a finer reverse water-filling (the explainer's walk
 * hands out whole 4-bit channels; 核心方法 / 读侧 notes finer handling for
 * continuous importance): bit s+1 of channel c is worth w_c * 4^-s (the
 * distortion a channel read at t bits keeps falls as 4^-t), and each query
 * reads its B most valuable (channel, bit) pairs, ties to the lower channel
 * then the lower bit -- the same as handing the bits out one at a time to
 * the channel of largest w_c * 4^-t_c.  Same arguments, outputs and errors
 * as fathom_plan; sum_c t_c = B and t_c <= b. */
fathom_status fathom_plan_marginal(const fathom_index *index, const uint16_t *q_bf16,
                                   const int32_t *budget, uint8_t *t, uint8_t *t_union,
                                   uint64_t *bytes, cudaStream_t stream);

/* Fixed-width baseline plan (the 136-bit / 68-bit key scans the explainer
 * compares against): the r channels of largest |q_c| (ties to the lower
 * channel) are read at all b bits, the rest at 0.  Same outputs as
 * fathom_plan.  0 <= r <= d. */
fathom_status fathom_fixed_plan(const fathom_index *index, const uint16_t *q_bf16,
                                int32_t r, uint8_t *t, uint8_t *t_union,
                                uint64_t *bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Read side: scan and select.                                            */
/* ---------------------------------------------------------------------- */

/* Workspace bytes fathom_scan_topk needs for `index` and k. */
size_t fathom_scan_workspace_bytes(const fathom_index *index, int32_t k);

/* Score every key for every query from only the planes its plan selects,
 * and select the top-k (explainer, 核心方法 and 解决什么真问题).
 * Each KV head reads the union of its G queries' planes once; query g's
 * score of key j is
 *   s_gj = sum_c q_gc * (mn_c + scale_c*(2^(b-t)*u + (2^(b-t)-1)/2)),
 *   t = t_gc, u = code_cj >> (b-t)
 * (the key rebuilt at the middle of its coarse t-bit bin), accumulated in
 * float32.  Outputs the k keys of largest s, ties to the lower index,
 * listed in ascending key index.
 * An 8-plane index (b = 8) is scored as 2d nibble channels: the high and
 * low nibbles of channel c (planes 0-3 and 4-7, which the layout already
 * stores as two 4-plane channels) with scales 16*scale_c and scale_c and
 * minima mn_c and 0, read to min(t, 4) and max(t - 4, 0) planes -- the
 * same rebuilt key, since the high nibble's bin middle plus the low
 * nibble's is the 8-bit bin middle.  This adds one small launch and
 * (9*H + 3*Q)*2d bytes of workspace (each array rounded up to 16 bytes) for
 * the nibble-channel arguments.
 * All sessions of a batched call have the same b.
 * Grouped scales: key j is scored with mn and scale of its block; extra
 * CTAs of the call's threshold launch compute each (KV head, block, query
 * head) bias, and the workspace holds those H*n_blocks*G floats.  All sessions of a batched
 * call have grouped scales or none have.
 * q_bf16, t, t_union, out_idx, out_score, workspace: device pointers.
 * flags: FATHOM_SCAN_* bits. */
fathom_status fathom_scan_topk(const fathom_index *index, const uint16_t *q_bf16,
                               const uint8_t *t, const uint8_t *t_union, int32_t k,
                               int32_t *out_idx, float *out_score,
                               void *workspace, size_t workspace_bytes,
                               uint32_t flags, cudaStream_t stream);

/* fathom_scan_topk for callers that cannot allocate device memory (the
 * paper has no counterpart: this is an interface convenience).  Some callers
 * are handed only their inputs and outputs and have no allocator to call --
 * e.g. a plugin inside an engine whose memory pool already owns the free HBM,
 * or a decode loop that must not call cudaMalloc because it can synchronise
 * the device.  This call takes no workspace: it runs on an 8 MiB scratch
 * array that the library reserves as a static __device__ variable on every
 * GPU that loads it, held until the process exits.
 *   - Same arguments and results as fathom_scan_topk, minus the workspace.
 *   - A problem needing more than 8 MiB of scratch is rejected with
 *     FATHOM_ERR_WORKSPACE before anything is enqueued; use fathom_scan_topk
 *     for it.  For a device index, a layer of 64 query heads at 1,048,576
 *     keys with k <= 2048 needs 6.3 MiB; a host-resident index also needs
 *     room for its two-slot plane ring, so only small ones fit.
 *   - Every call looks up the scratch array's device address
 *     (cudaGetSymbolAddress) on the current device instead of caching it.
 *     The first call on a device may also load the library's device code
 *     there; make that first call before any stream capture.  Like every
 *     call of this library it must not follow a cudaDeviceReset of that
 *     device (see the conventions above).
 *   - All calls on a device share the one array.  Calls whose kernels overlap
 *     on the GPU (e.g. on two streams at once) race on it: order them.
 *   - Calls or frees no device memory. */
fathom_status fathom_scan_topk_static(const fathom_index *index, const uint16_t *q_bf16,
                                      const uint8_t *t, const uint8_t *t_union, int32_t k,
                                      int32_t *out_idx, float *out_score, uint32_t flags,
                                      cudaStream_t stream);

/* Workspace bytes fathom_scan_topk_batched needs. */
size_t fathom_scan_batched_workspace_bytes(const fathom_index *sessions,
                                           int32_t n_sessions, int32_t k);

/* The same scan over many independent sessions (concurrent agent sessions
 * of the explainer's setting) in one launch per phase.  sessions: host
 * array of n_sessions (1..64) descriptors sharing head_dim and group;
 * q_bf16, t, t_union, out_idx, out_score: host arrays of n_sessions device
 * pointers laid out as for fathom_scan_topk. */
fathom_status fathom_scan_topk_batched(const fathom_index *sessions, int32_t n_sessions,
                                       const uint16_t *const *q_bf16,
                                       const uint8_t *const *t,
                                       const uint8_t *const *t_union, int32_t k,
                                       int32_t *const *out_idx, float *const *out_score,
                                       void *workspace, size_t workspace_bytes,
                                       uint32_t flags, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* One KV head's keys split across devices.                               */
/* ---------------------------------------------------------------------- */

/* Exact top-k over the shards of a key range (explainer, 解决什么真问题:
 * each decode step keeps the top-k of all keys).  Shard s holds the keys
 * [shard_offset[s], shard_offset[s+1]) of every KV head and returned its
 * top-k_shard per query (e.g. from fathom_scan_topk on an index of that
 * range): shard_idx int32 [S][Q][k_shard] local key indices in ascending
 * order, shard_score float32 [S][Q][k_shard] (device pointers, e.g. one
 * all-gathered buffer).  Keys rank by (score descending, global index
 * ascending), the order of the single-device top-k, so the result is the
 * top-k of all the shards' keys: out_idx int32 [Q][k] global indices in
 * ascending order, out_score float32 [Q][k].  Shards that are word ranges
 * of one packed index (same mn, scale, sigma2) score each key exactly as
 * the whole index does, and the merge reproduces the single-device output.
 * shard_offset: host array of S ascending key offsets.  1 <= S <= 64,
 * S*k_shard <= 16384, 1 <= k <= min(S*k_shard, 4096).  A negative index or
 * non-finite score in the lists sets FATHOM_ERR_INVALID_ARG in the device
 * status. */
fathom_status fathom_merge_topk(const int32_t *shard_idx, const float *shard_score,
                                const int64_t *shard_offset, int32_t n_shards, int32_t n_queries,
                                int32_t k_shard, int32_t k, int32_t *out_idx, float *out_score,
                                cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* After the scan: attention over the selected keys.                      */
/* ---------------------------------------------------------------------- */

/* Workspace bytes fathom_sparse_attention needs (0 for invalid sizes). */
size_t fathom_sparse_attention_workspace_bytes(int32_t n_queries, int32_t head_dim, int32_t k);

/* Softmax attention of each query over the k keys its top-k selected (the
 * step after the scan: the explainer's decode step fetches and attends over
 * the selected K/V rows, 解决什么真问题): for query q of KV head q / G,
 *   l_i = softmax_scale * (q . K[h][idx[q][i]]),  p = softmax(l),
 *   out[q] = sum_i p_i * V[h][idx[q][i]],
 * in float32 (q the bf16 query widened exactly).
 * keys, values: float32 [H][n][d], device memory or pinned host memory
 * (read through its device mapping), 16-byte aligned; q_bf16 [Q][d],
 * idx int32 [Q][k] (e.g. fathom_scan_topk's out_idx), out float32 [Q][d]:
 * device pointers.  1 <= k <= n; head_dim a multiple of 32, at most 256;
 * G 1..8.  An index outside [0, n) is skipped and sets
 * FATHOM_ERR_INVALID_ARG in the device status. */
fathom_status fathom_sparse_attention(const float *keys, const float *values, int32_t n_kv_heads,
                                      int32_t group, int32_t head_dim, int32_t n_keys,
                                      const uint16_t *q_bf16, const int32_t *idx, int32_t k,
                                      float softmax_scale, float *out, void *workspace,
                                      size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Status and instrumentation.                                            */
/* ---------------------------------------------------------------------- */

/* Synchronise `stream`, return the first device-side error recorded on the
 * current device since the last call (FATHOM_OK if none) and clear it.
 * A failed synchronisation returns FATHOM_ERR_CUDA. */
fathom_status fathom_last_device_status(cudaStream_t stream);

/* Kernels this library has launched in this process. */
uint64_t fathom_launch_count(void);

/* Time of what FATHOM_SCAN_PROFILE times (the fetch sequence for a
 * host-resident index, else the main scan kernel), recorded with CUDA events:
 * synchronises on the recorded events and returns the summed milliseconds
 * and the number of launches timed, then forgets them.  Not thread-safe;
 * benchmarking only. */
fathom_status fathom_profile_read(double *scan_kernel_ms, uint64_t *scan_kernel_launches);

/* Instrumentation: read `bytes` (>= 16, a multiple of 16 is read in full)
 * of `buffer` -- a pinned, device-mapped host buffer, or device memory --
 * with 16-byte loads from every SM, the access pattern of the host-resident
 * scan, so the zero-copy read bandwidth of the host link can be measured
 * with events around the call.  `sink` is a device word the kernel may
 * increment (keeps the loads).  buffer must be 16-byte aligned. */
fathom_status fathom_link_probe(const void *buffer, size_t bytes, unsigned long long *sink,
                                cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FATHOM_H */
