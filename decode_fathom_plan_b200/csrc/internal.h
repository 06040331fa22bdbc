// Host-side interfaces between the C-ABI layer and the kernel launchers
// (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <nvtx3/nvToolsExt.h>

#include "fathom.h"

namespace fathom {

// Named NVTX range for the lifetime of a scope: marks each C-ABI call and
// each scan phase on a profiler's timeline (Nsight Systems); without a
// profiler attached the calls return at once.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Address of this device's status word (a __device__ int).
int *device_status_ptr();
// Count one kernel launch (for fathom_launch_count).
void note_launch(int n = 1);
// Record the CUDA error of a failed step (reported on stderr once per site
// by the C-ABI layer) and return it.
cudaError_t note_error(cudaError_t e, const char *site);

// Code width b of an index: 4, or 8 for the 8-plane variant (the C ABI
// reads 0 as 4 and rejects anything else before a launcher runs).
inline int index_bits(const fathom_index &ix) { return ix.bits == 8 ? 8 : 4; }
// Statistics rows per KV head: 1, or the blocks the planes can hold when the
// index has grouped per-token-block scales (block_keys > 0).
inline int index_blocks(const fathom_index &ix)
{
    return ix.block_keys ? (int)(((long long)ix.n_words * 32 + ix.block_keys - 1) / ix.block_keys)
                         : 1;
}

// ---- pack.cu
cudaError_t launch_pack(const float *keys, const fathom_index &ix, uint32_t *ws_minmax,
                        cudaStream_t stream);
// sigma^2 of every (head, channel) from its exact sums and the key count n
// (combined over the blocks of a block-scaled index).
cudaError_t launch_channel_stats(const fathom_index &ix, int n, cudaStream_t stream);
// Appends m keys (device float32 [H][m][d]) to a block-scaled index whose
// ix.n_keys is a whole number of blocks: the new blocks are packed on their
// own, sigma^2 is recomputed for ix.n_keys + m keys.
cudaError_t launch_append_blocks(const float *keys, const fathom_index &ix, int m,
                                 cudaStream_t stream);

// ---- append.cu
// Appends m keys (device float32 [H][m][d]) at positions ix.n_keys.. and
// recomputes sigma^2 for ix.n_keys + m keys; clamped may be null.
cudaError_t launch_append(const float *keys, const fathom_index &ix, int m, uint32_t *clamped,
                          cudaStream_t stream);

// ---- plan.cu
cudaError_t launch_plan(const fathom_index &ix, const uint16_t *q, const int32_t *budget,
                        int32_t fixed_r, bool fixed, uint8_t *t, uint8_t *t_union,
                        uint64_t *bytes, cudaStream_t stream);
cudaError_t launch_plan_marginal(const fathom_index &ix, const uint16_t *q, const int32_t *budget,
                                 uint8_t *t, uint8_t *t_union, uint64_t *bytes,
                                 cudaStream_t stream);

// ---- lift.cu
// An 8-plane index's scan arguments rewritten for the 4-plane scan over 2d
// nibble channels (the planes themselves need no change).
struct LiftArgs {
    const float *mn, *scale;     // [stat_rows][d]: one row per (head, scale block)
    const uint16_t *q;           // [Q][d]
    const uint8_t *t, *tu;       // [Q][d], [H][d]
    float *mn2, *scale2;         // [stat_rows][2d]
    uint16_t *q2;                // [Q][2d]
    uint8_t *t2, *tu2;           // [Q][2d], [H][2d]
    int H, Q, d, stat_rows;
};
// Workspace bytes of the primed arrays (each rounded up to 16 bytes).
size_t lift_bytes(int H, int Q, int d, int stat_rows);
// Points the primed arrays of *a into ws (lift_bytes(...) bytes, 16-byte
// aligned) and sets its sizes; the caller sets the inputs.
void lift_carve(void *ws, int H, int Q, int d, int stat_rows, LiftArgs *a);
cudaError_t launch_lift(const LiftArgs &a, cudaStream_t stream);

// ---- fetch.cu
// One host-resident index to fetch: for each of its n_channels = H*d
// (head, channel) pairs, the first t_union[hc] slots of n_words words.
struct FetchJob {
    const uint32_t *src;       // device-mapped host planes [H][d][4][n_words]
    uint32_t *dst;             // device ring slot, same layout
    const uint8_t *t_union;    // [H][d]
    int n_channels;
    int n_words;
};
// CTAs per multiprocessor of a fetch that shares the GPU with the scoring
// kernels of the previous unit (the link needs few SMs to stay busy).
constexpr int kFetchCtasPerSmShared = 2;
cudaError_t launch_fetch(const FetchJob *jobs, int n_jobs, cudaStream_t stream, int ctas_per_sm);

// ---- attention.cu
// Split-K runs per query for k selected keys.
int attention_splits(int k);
// Attention of Q = H*G queries over their k selected keys; part: workspace
// of Q * attention_splits(k) * (d + 2) floats.
cudaError_t launch_attention(const float *keys, const float *values, int H, int G, int d, int n,
                             const uint16_t *q_bf16, const int32_t *idx, int k, float scale,
                             float *out, float *part, cudaStream_t stream);

// ---- merge.cu
constexpr int kMaxMergeShards = 64;
constexpr int kMaxMergeCandidates = 16384;   // S * k_s per query (shared memory)
struct MergeOffsets {
    long long offset[kMaxMergeShards];       // first global key of each shard
};
size_t merge_smem_bytes(int S, int k_s);
cudaError_t launch_merge(const int32_t *idx, const float *score, const MergeOffsets &off, int S,
                         int Q, int k_s, int k, int32_t *out_idx, float *out_score,
                         cudaStream_t stream);

// ---- scan.cu
struct ScanSessionArgs {
    const fathom_index *ix;
    const uint16_t *q;
    const uint8_t *t;
    const uint8_t *t_union;
    int32_t *out_idx;
    float *out_score;
};

// Workspace bytes for a batch of sessions (single call = batch of one).
size_t scan_workspace_bytes(const fathom_index *sessions, int n_sessions, int k);

// Profiling events around the dominant kernel of a scan call
// (FATHOM_SCAN_PROFILE): the fetch sequence when any index is host-resident, else
// the main scan.
struct ScanProfileHook {
    bool enabled;
    cudaEvent_t begin, end;
    bool recorded;   // set when that kernel was launched and timed
};

cudaError_t launch_scan(const ScanSessionArgs *sessions, int n_sessions, int k,
                        void *ws, size_t ws_bytes, uint32_t flags, cudaStream_t stream,
                        ScanProfileHook *hook);

}  // namespace fathom
