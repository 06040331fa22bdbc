// One KV head's keys split across devices: the exact merge of the shards'
// top-k lists.
//
// Source: Fathom explainer (papers.ananclaw.com, arXiv 2609.17652),
// section 解决什么真问题 (each decode step keeps the top-k of all n keys).
// When the keys of a head are split into ranges held by different devices,
// each range's top-k (by score, ties to the lower index) contains every key
// of the global top-k that falls in it, so an exact selection over the
// gathered lists gives the global top-k.  Shards that are word ranges of
// one packed index (shared statistics) score every key exactly as the whole
// index would, so the merge reproduces the single-device result.
//
// One CTA per query: the S*k_s (score, global index) composites go to
// shared memory, the same range-relative radix select as the scan's final
// pass finds the k-th, and a stable compaction in (shard, list position)
// order -- ascending global index, since each list is ascending and the
// shard offsets ascend -- writes the outputs.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace fathom {
namespace {

__global__ void __launch_bounds__(kSelThreads)
merge_kernel(const int32_t *__restrict__ idx, const float *__restrict__ score,
             const __grid_constant__ MergeOffsets off, int S, int Q, int k_s, int k,
             int32_t *out_idx, float *out_score, int *status)
{
    extern __shared__ unsigned long long x[];   // [S * k_s]
    __shared__ SelShared ss;
    const int qq = blockIdx.x;
    const int m = S * k_s;
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    bool bad = false;
    for (int e = threadIdx.x; e < m; e += kSelThreads) {
        const int s = e / k_s, i = e - s * k_s;
        const size_t at = ((size_t)s * Q + qq) * k_s + i;
        const int32_t li = idx[at];
        const float sc = score[at];
        bad |= li < 0 || !isfinite(sc);
        const uint32_t okey = order_key(sc);
        const uint32_t gidx = (uint32_t)(off.offset[s] + (long long)(li < 0 ? 0 : li));
        x[e] = ((unsigned long long)okey << 32) | (0xFFFFFFFFu - gidx);
        lo = min(lo, okey);
        hi = max(hi, okey);
    }
    if (bad) set_status(status, FATHOM_ERR_INVALID_ARG);
    sel_range(ss, lo, hi);
    const unsigned long long base = (unsigned long long)ss.lo << 32;
    const int top = 32 + bit_length(ss.hi - ss.lo);
    sel_run(ss, (unsigned)m, (unsigned)k, top, 0, [&](unsigned i) { return x[i] - base; });
    const int cut = ss.cut;
    const unsigned long long lim = ss.prefix >> cut;
    // stable compaction: each thread a contiguous run of the lists
    const int per = (m + kSelThreads - 1) / kSelThreads;
    const int e0 = threadIdx.x * per, e1 = min(m, e0 + per);
    unsigned mine = 0;
    for (int e = e0; e < e1; ++e) mine += ((x[e] - base) >> cut) >= lim;
    unsigned total;
    unsigned pos = block_exclusive_scan(mine, ss.wsum, &total);
    for (int e = e0; e < e1; ++e) {
        const unsigned long long v = x[e];
        if (((v - base) >> cut) >= lim) {
            if (pos < (unsigned)k) {
                out_idx[(size_t)qq * k + pos] = (int32_t)(0xFFFFFFFFu - (uint32_t)(v & 0xFFFFFFFFull));
                out_score[(size_t)qq * k + pos] = order_key_to_float((uint32_t)(v >> 32));
            }
            ++pos;
        }
    }
}

}  // namespace

size_t merge_smem_bytes(int S, int k_s) { return (size_t)S * k_s * sizeof(unsigned long long); }

cudaError_t launch_merge(const int32_t *idx, const float *score, const MergeOffsets &off, int S,
                         int Q, int k_s, int k, int32_t *out_idx, float *out_score,
                         cudaStream_t stream)
{
    static int smem_set[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!smem_set[dev]) {
        e = cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)merge_smem_bytes(1, kMaxMergeCandidates));
        if (e != cudaSuccess) return e;
        smem_set[dev] = 1;
    }
    merge_kernel<<<Q, kSelThreads, merge_smem_bytes(S, k_s), stream>>>(
        idx, score, off, S, Q, k_s, k, out_idx, out_score, device_status_ptr());
    note_launch(1);
    return cudaGetLastError();
}

}  // namespace fathom
