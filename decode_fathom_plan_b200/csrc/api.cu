// C ABI of the Fathom sm_100a library: argument validation, residency
// resolution, workspace accounting, device status and instrumentation.
// The operations themselves are documented in include/fathom.h.
#include <stdio.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace fathom {

// First device-side error since the last fathom_last_device_status() call
// (one word per device: a module-scope __device__ variable).
__device__ int g_device_status;

namespace {
std::atomic<unsigned long long> g_launches{0};
std::mutex g_mu;
int *g_status_ptr[64] = {nullptr};
struct EventPair {
    cudaEvent_t begin, end;
};
std::vector<EventPair> g_recorded;   // profiled scan launches not read yet
std::vector<EventPair> g_free_events;
}  // namespace

int *device_status_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int *>(p);
    }
    return g_status_ptr[dev];
}

void note_launch(int n) { g_launches.fetch_add((unsigned long long)n); }

cudaError_t note_error(cudaError_t e, const char *site)
{
    if (e != cudaSuccess)
        fprintf(stderr, "fathom: %s failed: %s (%s)\n", site, cudaGetErrorName(e),
                cudaGetErrorString(e));
    return e;
}

}  // namespace fathom

using namespace fathom;

namespace {

fathom_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FATHOM_OK : FATHOM_ERR_CUDA; }

bool index_shape_ok(const fathom_index *ix)
{
    if (!ix) return false;
    if (ix->n_kv_heads < 1 || ix->group < 1 || ix->group > kMaxGroup) return false;
    if (ix->head_dim < 32 || ix->head_dim > kMaxHeadDim || ix->head_dim % 32) return false;
    if (ix->n_keys < 1 || ix->n_words < 4 || ix->n_words % 4) return false;
    if ((long long)ix->n_words * 32 < (long long)ix->n_keys) return false;
    if (ix->residency != FATHOM_RES_DEVICE && ix->residency != FATHOM_RES_HOST_MAPPED) return false;
    if (ix->bits != 0 && ix->bits != 4 && ix->bits != 8) return false;
    // grouped scales: blocks of whole 2048-key scan tiles
    if (ix->block_keys < 0 || ix->block_keys % kTileKeys) return false;
    const int bits = index_bits(*ix);
    // 8 planes: the scan's 2d nibble channels fit its head_dim limit
    if (bits == 8 && 2 * ix->head_dim > kMaxHeadDim) return false;
    // n * sum_code2 <= n^2 * (2^b - 1)^2 must fit in int64
    if ((long long)ix->n_words * 32 > (bits == 8 ? (1ll << 23) : (1ll << 27))) return false;
    // global plane row indices must fit in 32 bits
    if ((long long)ix->n_kv_heads * ix->head_dim * bits >= (1ll << 31)) return false;
    return true;
}

size_t align16(size_t b) { return (b + 15) & ~(size_t)15; }

// The descriptor the 4-plane scan sees: an 8-plane index is 2d nibble
// channels of 4 planes each (same planes; mn and scale are replaced by the
// lifted arrays before a launch).
fathom_index scan_view(const fathom_index &ix)
{
    fathom_index v = ix;
    if (index_bits(ix) == 8) {
        v.head_dim = 2 * ix.head_dim;
        v.bits = 4;
    }
    return v;
}

// Workspace of a scan call: the scan's own part (16-byte rounded), then the
// lifted arrays of every 8-plane session.
size_t scan_part_bytes(const fathom_index *sessions, int n_sessions, int k)
{
    std::vector<fathom_index> views(n_sessions);
    for (int s = 0; s < n_sessions; ++s) views[s] = scan_view(sessions[s]);
    return align16(scan_workspace_bytes(views.data(), n_sessions, k));
}

size_t scan_total_bytes(const fathom_index *sessions, int n_sessions, int k)
{
    size_t total = scan_part_bytes(sessions, n_sessions, k);
    for (int s = 0; s < n_sessions; ++s) {
        const fathom_index &ix = sessions[s];
        if (index_bits(ix) == 8)
            total += lift_bytes(ix.n_kv_heads, ix.n_kv_heads * ix.group, ix.head_dim,
                                ix.n_kv_heads * index_blocks(ix));
    }
    return total;
}

// Resolve the planes pointer to a device address for the residency mode.
fathom_status resolve_planes(const fathom_index *ix, uint32_t **out)
{
    // plane rows are copied 16 bytes at a time
    if (!ix->planes || (reinterpret_cast<uintptr_t>(ix->planes) & 15u)) return FATHOM_ERR_INVALID_ARG;
    if (ix->residency == FATHOM_RES_HOST_MAPPED) {
        void *dptr = nullptr;
        if (cudaHostGetDevicePointer(&dptr, ix->planes, 0) != cudaSuccess || !dptr) {
            cudaGetLastError();
            return FATHOM_ERR_INVALID_ARG;
        }
        *out = static_cast<uint32_t *>(dptr);
        return FATHOM_OK;
    }
    cudaPointerAttributes attr{};
    if (cudaPointerGetAttributes(&attr, ix->planes) != cudaSuccess) {
        cudaGetLastError();
        return FATHOM_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
        return FATHOM_ERR_INVALID_ARG;
    *out = ix->planes;
    return FATHOM_OK;
}

bool stats_ok(const fathom_index *ix)
{
    return ix->mn && ix->scale && ix->sigma2 && ix->sum_code && ix->sum_code2;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

EventPair take_event_pair()
{
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_free_events.empty()) {
        EventPair p = g_free_events.back();
        g_free_events.pop_back();
        return p;
    }
    EventPair p{};
    cudaEventCreate(&p.begin);
    cudaEventCreate(&p.end);
    return p;
}

fathom_status scan_common(const fathom_index *sessions, int n_sessions,
                          const uint16_t *const *q, const uint8_t *const *t,
                          const uint8_t *const *tu, int32_t k, int32_t *const *out_idx,
                          float *const *out_score, void *ws, size_t ws_bytes, uint32_t flags,
                          cudaStream_t stream)
{
    if (!sessions || n_sessions < 1 || n_sessions > kMaxSessions) return FATHOM_ERR_INVALID_ARG;
    if (!q || !t || !tu || !out_idx || !out_score) return FATHOM_ERR_INVALID_ARG;
    if (flags & ~(FATHOM_SCAN_FORCE_EXACT | FATHOM_SCAN_PROFILE)) return FATHOM_ERR_INVALID_ARG;
    if (k < 1 || k > kMaxK) return FATHOM_ERR_INVALID_ARG;
    std::vector<fathom_index> resolved(n_sessions);
    std::vector<ScanSessionArgs> args(n_sessions);
    for (int s = 0; s < n_sessions; ++s) {
        const fathom_index *ix = &sessions[s];
        if (!index_shape_ok(ix) || !ix->mn || !ix->scale) return FATHOM_ERR_INVALID_ARG;
        if (ix->head_dim != sessions[0].head_dim || ix->group != sessions[0].group ||
            index_bits(*ix) != index_bits(sessions[0]) ||
            (ix->block_keys != 0) != (sessions[0].block_keys != 0))
            return FATHOM_ERR_INVALID_ARG;
        if (k > ix->n_keys) return FATHOM_ERR_INVALID_ARG;
        if (!q[s] || !t[s] || !tu[s] || !out_idx[s] || !out_score[s]) return FATHOM_ERR_INVALID_ARG;
        resolved[s] = scan_view(*ix);
        fathom_status st = resolve_planes(ix, &resolved[s].planes);
        if (st != FATHOM_OK) return st;
        args[s] = ScanSessionArgs{&resolved[s], q[s], t[s], tu[s], out_idx[s], out_score[s]};
    }
    const size_t scan_part = scan_part_bytes(sessions, n_sessions, k);
    if (!ws || !aligned16(ws) || ws_bytes < scan_total_bytes(sessions, n_sessions, k))
        return FATHOM_ERR_WORKSPACE;
    if (index_bits(sessions[0]) == 8) {
        // 8-plane sessions: write the nibble-channel arguments behind the
        // scan's own workspace and point the scan at them
        unsigned char *at = static_cast<unsigned char *>(ws) + scan_part;
        for (int s = 0; s < n_sessions; ++s) {
            const fathom_index &ix = sessions[s];
            const int H = ix.n_kv_heads, Q = H * ix.group, d = ix.head_dim;
            const int rows = H * index_blocks(ix);
            LiftArgs la{};
            la.mn = ix.mn;
            la.scale = ix.scale;
            la.q = q[s];
            la.t = t[s];
            la.tu = tu[s];
            lift_carve(at, H, Q, d, rows, &la);
            at += lift_bytes(H, Q, d, rows);
            const cudaError_t e = launch_lift(la, stream);
            if (e != cudaSuccess) return cuda_status(note_error(e, "lift"));
            resolved[s].mn = la.mn2;
            resolved[s].scale = la.scale2;
            args[s].q = la.q2;
            args[s].t = la.t2;
            args[s].t_union = la.tu2;
        }
    }

    ScanProfileHook hook{false, nullptr, nullptr, false};
    EventPair ev{};
    if (flags & FATHOM_SCAN_PROFILE) {
        ev = take_event_pair();
        hook = ScanProfileHook{true, ev.begin, ev.end, false};
    }
    cudaError_t e = launch_scan(args.data(), n_sessions, k, ws, scan_part, flags, stream, &hook);
    if (flags & FATHOM_SCAN_PROFILE) {
        std::lock_guard<std::mutex> lock(g_mu);
        if (hook.recorded)
            g_recorded.push_back(ev);
        else
            g_free_events.push_back(ev);
    }
    return cuda_status(e);
}

// A device-usable address for a K or V array: device or managed memory as
// is, pinned host memory through its device mapping; 16-byte aligned.
fathom_status resolve_kv(const float *p, const float **out)
{
    if (!p || !aligned16(p)) return FATHOM_ERR_INVALID_ARG;
    cudaPointerAttributes attr{};
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return FATHOM_ERR_INVALID_ARG;
    }
    if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) {
        *out = p;
        return FATHOM_OK;
    }
    if (attr.type == cudaMemoryTypeHost) {
        void *dptr = nullptr;
        if (cudaHostGetDevicePointer(&dptr, const_cast<float *>(p), 0) != cudaSuccess || !dptr) {
            cudaGetLastError();
            return FATHOM_ERR_INVALID_ARG;
        }
        *out = static_cast<const float *>(dptr);
        return FATHOM_OK;
    }
    return FATHOM_ERR_INVALID_ARG;
}

size_t attention_bytes(int32_t n_queries, int32_t head_dim, int32_t k)
{
    if (n_queries < 1 || head_dim < 32 || head_dim > kMaxHeadDim || head_dim % 32 || k < 1)
        return 0;
    return (size_t)n_queries * fathom::attention_splits(k) * (size_t)(head_dim + 2) * sizeof(float);
}

}  // namespace

extern "C" {

int32_t fathom_n_words(int32_t n_keys)
{
    if (n_keys < 1) return 0;
    return (int32_t)(((long long)n_keys + 127) / 128 * 4);
}

const char *fathom_status_str(fathom_status status)
{
    switch (status) {
    case FATHOM_OK: return "ok";
    case FATHOM_ERR_INVALID_ARG: return "invalid argument";
    case FATHOM_ERR_CUDA: return "CUDA error";
    case FATHOM_ERR_NONFINITE: return "non-finite key, query or importance";
    case FATHOM_ERR_TIMEOUT: return "device wait timed out";
    case FATHOM_ERR_WORKSPACE: return "workspace missing or too small";
    case FATHOM_ERR_UNIMPLEMENTED: return "unimplemented";
    }
    return "unknown status";
}

size_t fathom_pack_workspace_bytes(const fathom_index *index)
{
    if (!index_shape_ok(index)) return 0;
    return (size_t)8 * index->n_kv_heads * index->head_dim;
}

fathom_status fathom_pack_keys(const float *keys, const fathom_index *index, void *workspace,
                               size_t workspace_bytes, cudaStream_t stream)
{
    NvtxRange range("fathom_pack_keys");
    if (!keys || !index_shape_ok(index) || !stats_ok(index)) return FATHOM_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace) || workspace_bytes < fathom_pack_workspace_bytes(index))
        return FATHOM_ERR_WORKSPACE;
    fathom_index ix = *index;
    fathom_status st = resolve_planes(index, &ix.planes);
    if (st != FATHOM_OK) return st;
    return cuda_status(launch_pack(keys, ix, static_cast<uint32_t *>(workspace), stream));
}

fathom_status fathom_append_keys(fathom_index *index, const float *keys, int32_t m,
                                 uint32_t *clamped, cudaStream_t stream)
{
    NvtxRange range("fathom_append_keys");
    if (!keys || !index_shape_ok(index) || !stats_ok(index) || m < 1) return FATHOM_ERR_INVALID_ARG;
    if ((long long)index->n_keys + m > (long long)index->n_words * 32) return FATHOM_ERR_INVALID_ARG;
    fathom_index ix = *index;
    fathom_status st = resolve_planes(index, &ix.planes);
    if (st != FATHOM_OK) return st;
    if (ix.block_keys) {
        // grouped scales: new keys open new blocks, each quantised on its own
        if (ix.n_keys % ix.block_keys) return FATHOM_ERR_INVALID_ARG;
        st = cuda_status(launch_append_blocks(keys, ix, m, stream));
    } else {
        st = cuda_status(launch_append(keys, ix, m, clamped, stream));
    }
    if (st == FATHOM_OK) index->n_keys += m;
    return st;
}

fathom_status fathom_plan(const fathom_index *index, const uint16_t *q_bf16,
                          const int32_t *budget, uint8_t *t, uint8_t *t_union, uint64_t *bytes,
                          cudaStream_t stream)
{
    NvtxRange range("fathom_plan");
    if (!index_shape_ok(index) || !index->sigma2) return FATHOM_ERR_INVALID_ARG;
    if (!q_bf16 || !budget || !t || !t_union || !bytes) return FATHOM_ERR_INVALID_ARG;
    return cuda_status(launch_plan(*index, q_bf16, budget, 0, false, t, t_union, bytes, stream));
}

fathom_status fathom_plan_marginal(const fathom_index *index, const uint16_t *q_bf16,
                                   const int32_t *budget, uint8_t *t, uint8_t *t_union,
                                   uint64_t *bytes, cudaStream_t stream)
{
    NvtxRange range("fathom_plan_marginal");
    if (!index_shape_ok(index) || !index->sigma2) return FATHOM_ERR_INVALID_ARG;
    if (!q_bf16 || !budget || !t || !t_union || !bytes) return FATHOM_ERR_INVALID_ARG;
    return cuda_status(launch_plan_marginal(*index, q_bf16, budget, t, t_union, bytes, stream));
}

fathom_status fathom_fixed_plan(const fathom_index *index, const uint16_t *q_bf16, int32_t r,
                                uint8_t *t, uint8_t *t_union, uint64_t *bytes,
                                cudaStream_t stream)
{
    NvtxRange range("fathom_fixed_plan");
    if (!index_shape_ok(index)) return FATHOM_ERR_INVALID_ARG;
    if (!q_bf16 || !t || !t_union || !bytes) return FATHOM_ERR_INVALID_ARG;
    if (r < 0 || r > index->head_dim) return FATHOM_ERR_INVALID_ARG;
    return cuda_status(launch_plan(*index, q_bf16, nullptr, r, true, t, t_union, bytes, stream));
}

size_t fathom_scan_workspace_bytes(const fathom_index *index, int32_t k)
{
    if (!index_shape_ok(index) || k < 1 || k > kMaxK) return 0;
    return scan_total_bytes(index, 1, k);
}

fathom_status fathom_scan_topk(const fathom_index *index, const uint16_t *q_bf16,
                               const uint8_t *t, const uint8_t *t_union, int32_t k,
                               int32_t *out_idx, float *out_score, void *workspace,
                               size_t workspace_bytes, uint32_t flags, cudaStream_t stream)
{
    NvtxRange range("fathom_scan_topk");
    return scan_common(index, 1, &q_bf16, &t, &t_union, k, &out_idx, &out_score, workspace,
                       workspace_bytes, flags, stream);
}

size_t fathom_scan_batched_workspace_bytes(const fathom_index *sessions, int32_t n_sessions,
                                           int32_t k)
{
    if (!sessions || n_sessions < 1 || n_sessions > kMaxSessions || k < 1 || k > kMaxK) return 0;
    for (int s = 0; s < n_sessions; ++s)
        if (!index_shape_ok(&sessions[s]) || index_bits(sessions[s]) != index_bits(sessions[0]) ||
            (sessions[s].block_keys != 0) != (sessions[0].block_keys != 0))
            return 0;
    return scan_total_bytes(sessions, n_sessions, k);
}

fathom_status fathom_scan_topk_batched(const fathom_index *sessions, int32_t n_sessions,
                                       const uint16_t *const *q_bf16, const uint8_t *const *t,
                                       const uint8_t *const *t_union, int32_t k,
                                       int32_t *const *out_idx, float *const *out_score,
                                       void *workspace, size_t workspace_bytes, uint32_t flags,
                                       cudaStream_t stream)
{
    NvtxRange range("fathom_scan_topk_batched");
    return scan_common(sessions, n_sessions, q_bf16, t, t_union, k, out_idx, out_score,
                       workspace, workspace_bytes, flags, stream);
}

fathom_status fathom_last_device_status(cudaStream_t stream)
{
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                  stream) != cudaSuccess)
        return FATHOM_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return FATHOM_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                                stream) != cudaSuccess)
        return FATHOM_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return FATHOM_ERR_CUDA;
    return static_cast<fathom_status>(v);
}

uint64_t fathom_launch_count(void) { return (uint64_t)g_launches.load(); }

fathom_status fathom_profile_read(double *scan_kernel_ms, uint64_t *scan_kernel_launches)
{
    std::vector<EventPair> recs;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        recs.swap(g_recorded);
    }
    double total = 0.0;
    fathom_status st = FATHOM_OK;
    for (const EventPair &p : recs) {
        float ms = 0.0f;
        if (cudaEventSynchronize(p.end) != cudaSuccess ||
            cudaEventElapsedTime(&ms, p.begin, p.end) != cudaSuccess) {
            cudaGetLastError();
            st = FATHOM_ERR_CUDA;
            continue;
        }
        total += ms;
    }
    {
        std::lock_guard<std::mutex> lock(g_mu);
        g_free_events.insert(g_free_events.end(), recs.begin(), recs.end());
    }
    if (scan_kernel_ms) *scan_kernel_ms = total;
    if (scan_kernel_launches) *scan_kernel_launches = recs.size();
    return st;
}

fathom_status fathom_merge_topk(const int32_t *shard_idx, const float *shard_score,
                                const int64_t *shard_offset, int32_t n_shards, int32_t n_queries,
                                int32_t k_shard, int32_t k, int32_t *out_idx, float *out_score,
                                cudaStream_t stream)
{
    NvtxRange range("fathom_merge_topk");
    if (!shard_idx || !shard_score || !shard_offset || !out_idx || !out_score)
        return FATHOM_ERR_INVALID_ARG;
    if (n_shards < 1 || n_shards > kMaxMergeShards || n_queries < 1 || k_shard < 1)
        return FATHOM_ERR_INVALID_ARG;
    if ((long long)n_shards * k_shard > kMaxMergeCandidates) return FATHOM_ERR_INVALID_ARG;
    if (k < 1 || k > kMaxK || (long long)k > (long long)n_shards * k_shard)
        return FATHOM_ERR_INVALID_ARG;
    MergeOffsets off{};
    for (int s = 0; s < n_shards; ++s) {
        // ascending shard ranges, each holding at least its k_shard listed keys
        if (shard_offset[s] < 0 || (s > 0 && shard_offset[s] < shard_offset[s - 1] + k_shard))
            return FATHOM_ERR_INVALID_ARG;
        off.offset[s] = shard_offset[s];
    }
    if (shard_offset[n_shards - 1] + k_shard > (1ll << 31)) return FATHOM_ERR_INVALID_ARG;
    return cuda_status(launch_merge(shard_idx, shard_score, off, n_shards, n_queries, k_shard, k,
                                    out_idx, out_score, stream));
}

size_t fathom_sparse_attention_workspace_bytes(int32_t n_queries, int32_t head_dim, int32_t k)
{
    return attention_bytes(n_queries, head_dim, k);
}

fathom_status fathom_sparse_attention(const float *keys, const float *values, int32_t n_kv_heads,
                                      int32_t group, int32_t head_dim, int32_t n_keys,
                                      const uint16_t *q_bf16, const int32_t *idx, int32_t k,
                                      float softmax_scale, float *out, void *workspace,
                                      size_t workspace_bytes, cudaStream_t stream)
{
    NvtxRange range("fathom_sparse_attention");
    if (n_kv_heads < 1 || group < 1 || group > kMaxGroup || n_keys < 1) return FATHOM_ERR_INVALID_ARG;
    if (head_dim < 32 || head_dim > kMaxHeadDim || head_dim % 32) return FATHOM_ERR_INVALID_ARG;
    if (k < 1 || k > n_keys || !q_bf16 || !idx || !out || !isfinite(softmax_scale))
        return FATHOM_ERR_INVALID_ARG;
    const float *kd = nullptr, *vd = nullptr;
    fathom_status st = resolve_kv(keys, &kd);
    if (st != FATHOM_OK) return st;
    if ((st = resolve_kv(values, &vd)) != FATHOM_OK) return st;
    const size_t need = attention_bytes(n_kv_heads * group, head_dim, k);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return FATHOM_ERR_WORKSPACE;
    return cuda_status(fathom::launch_attention(kd, vd, n_kv_heads, group, head_dim, n_keys, q_bf16,
                                                idx, k, softmax_scale, out,
                                                static_cast<float *>(workspace), stream));
}

}  // extern "C"
