// Fetch of host-resident planes into device memory.
//
// Source: Fathom explainer (papers.ananclaw.com, arXiv 2609.17652),
// section 核心方法: the 4-bit K index is offloaded (the read side pulls it
// over the host link), and a query reads only its planned planes, so the
// bytes moved are sum_c t_c * bytes_per_plane.  Here a KV head moves the
// union plan's planes once: for channel c the first T_c = t_union[h][c]
// slots, which are adjacent in the channel-major layout [H][d][4][n_words],
// so every (head, channel) pair is one contiguous span of
// T_c * n_words * 4 bytes.  They land at the same offsets of a device ring
// slot laid out like the fetched heads of the index; slots past T_c are
// neither copied nor read afterwards.
//
// The copy streams at the link's rate only while every SM keeps loads in
// flight without pause, so the work is split into 16 KB items (one per CTA
// iteration, 4 independent 16-byte loads per thread) and the plan bytes an
// item needs are fetched 32 items ahead, one per lane, instead of once per
// item: a device-memory load issued behind a deep queue of host-link loads
// waits as long as they do.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace fathom {
namespace {

constexpr int kFetchThreads = 256;
constexpr int kFetchLoads = 4;                                    // per thread per item
constexpr int kFetchItemUnits = kFetchThreads * kFetchLoads;      // 16-byte units per item
constexpr int kFetchCtasPerSm = 6;

struct FetchBatch {
    FetchJob job[kMaxSessions];
    long long item_begin[kMaxSessions + 1];   // prefix of items over jobs
    int n_jobs;
};

// Items of one job: (head*d + channel) major, 16 KB block minor.
__device__ __forceinline__ int blocks_per_channel(int n_words)
{
    return (n_words + kFetchItemUnits - 1) / kFetchItemUnits;   // n_words units per channel
}

__global__ void __launch_bounds__(kFetchThreads, kFetchCtasPerSm)
fetch_kernel(const __grid_constant__ FetchBatch b)
{
    const long long total = b.item_begin[b.n_jobs];
    const int lane = threadIdx.x & 31;
    for (long long base = blockIdx.x; base < total; base += 32ll * gridDim.x) {
        // lane l looks up item base + l*grid: its job, span and depth
        const long long my_item = base + (long long)lane * gridDim.x;
        int my_live = 0;   // 16-byte units to copy in this item
        if (my_item < total) {
            int j = 0;
            while (j + 1 < b.n_jobs && my_item >= b.item_begin[j + 1]) ++j;
            const FetchJob &J = b.job[j];
            const long long local = my_item - b.item_begin[j];
            const int bpc = blocks_per_channel(J.n_words);
            const long long hc = local / bpc;
            const int blk = (int)(local - hc * bpc);
            const int depth = J.t_union[hc];
            const long long live = (long long)depth * (J.n_words / 4) - (long long)blk * kFetchItemUnits;
            my_live = live <= 0 ? 0 : (live >= kFetchItemUnits ? kFetchItemUnits : (int)live);
        }
        for (int l = 0; l < 32; ++l) {
            const long long item = base + (long long)l * gridDim.x;
            if (item >= total) break;
            const int live = __shfl_sync(0xFFFFFFFFu, my_live, l);
            if (live == 0) continue;
            int j = 0;
            while (j + 1 < b.n_jobs && item >= b.item_begin[j + 1]) ++j;
            const FetchJob &J = b.job[j];
            const long long local = item - b.item_begin[j];
            const int bpc = blocks_per_channel(J.n_words);
            const long long hc = local / bpc;
            const int blk = (int)(local - hc * bpc);
            const size_t off = (size_t)hc * (size_t)J.n_words + (size_t)blk * kFetchItemUnits;
            const uint4 *src = reinterpret_cast<const uint4 *>(J.src) + off;
            uint4 *dst = reinterpret_cast<uint4 *>(J.dst) + off;
            uint4 v[kFetchLoads];
#pragma unroll
            for (int i = 0; i < kFetchLoads; ++i) {
                const int u = i * kFetchThreads + threadIdx.x;
                if (u < live) v[i] = __ldcs(src + u);
            }
#pragma unroll
            for (int i = 0; i < kFetchLoads; ++i) {
                const int u = i * kFetchThreads + threadIdx.x;
                if (u < live) dst[u] = v[i];
            }
        }
    }
}

}  // namespace

cudaError_t launch_fetch(const FetchJob *jobs, int n_jobs, cudaStream_t stream, int ctas_per_sm)
{
    if (n_jobs <= 0) return cudaSuccess;
    if (n_jobs > kMaxSessions) return cudaErrorInvalidValue;
    FetchBatch b{};
    b.n_jobs = n_jobs;
    long long items = 0;
    for (int j = 0; j < n_jobs; ++j) {
        b.job[j] = jobs[j];
        b.item_begin[j] = items;
        items += (long long)jobs[j].n_channels *
                 ((jobs[j].n_words + kFetchItemUnits - 1) / kFetchItemUnits);
    }
    b.item_begin[n_jobs] = items;
    if (items == 0) return cudaSuccess;
    int dev = 0, n_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const int per_sm = std::max(1, std::min(ctas_per_sm, kFetchCtasPerSm));
    const long long ctas = std::min<long long>(items, (long long)std::max(1, n_sm) * per_sm);
    fetch_kernel<<<(int)ctas, kFetchThreads, 0, stream>>>(b);
    note_launch(1);
    return cudaGetLastError();
}

}  // namespace fathom
