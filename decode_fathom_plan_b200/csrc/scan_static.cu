// fathom_scan_topk_static: the scan + top-k of fathom_scan_topk for callers
// that cannot allocate device memory, running on scratch space the library
// reserves itself in a fixed-size file-scope device array.
//
// Who needs it: code that is handed only its inputs and outputs and has no
// allocator to call -- a plugin inside an inference engine whose memory pool
// already owns all free HBM (a cudaMalloc there fails or steals from the KV
// cache), or a decode loop that must not call cudaMalloc/cudaFree because
// they can synchronise the device mid-step.  Such a caller cannot size and
// pass the workspace fathom_scan_topk asks for.
//
// The array below is that workspace: kStaticScratchBytes per GPU, reserved
// on every device that loads this library and kept until the process exits.
// Host code may not pass the array's name to a kernel (on the host it is a
// stand-in, not a device address), so the first call on each device looks up
// the device address with cudaGetSymbolAddress while that device is current,
// and later calls reuse it.
#include <mutex>

#include "common.cuh"
#include "internal.h"

// 8 MiB: one Qwen3-8B-shaped layer (32 query heads) at up to 1,048,576 keys
// with k <= 2048 needs about 7 MiB of per-query state, sampled keys and
// candidates.
static constexpr size_t kStaticScratchBytes = 8u << 20;
static __device__ __align__(256) unsigned char g_scan_scratch[kStaticScratchBytes];

namespace {
std::mutex g_static_mu;
void *g_static_ptr[64] = {nullptr};

// Device address of g_scan_scratch on the current device (looked up once).
fathom_status static_scratch(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return FATHOM_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scan_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return FATHOM_ERR_CUDA;
        }
        g_static_ptr[dev] = p;
    }
    *out = g_static_ptr[dev];
    return FATHOM_OK;
}
}  // namespace

extern "C" fathom_status fathom_scan_topk_static(const fathom_index *index,
                                                 const uint16_t *q_bf16, const uint8_t *t,
                                                 const uint8_t *t_union, int32_t k,
                                                 int32_t *out_idx, float *out_score,
                                                 uint32_t flags, cudaStream_t stream)
{
    fathom::NvtxRange range("fathom_scan_topk_static");
    const size_t need = fathom_scan_workspace_bytes(index, k);
    if (need == 0) return FATHOM_ERR_INVALID_ARG;
    if (need > kStaticScratchBytes) return FATHOM_ERR_WORKSPACE;   // beyond the fixed maximum
    void *scratch = nullptr;
    const fathom_status st = static_scratch(&scratch);
    if (st != FATHOM_OK) return st;
    // Every per-call word of the scratch (threshold, candidate count, fallback
    // flag, sampled keys, candidates) is written by the kernels before it is
    // read, so nothing left over from the previous call needs clearing.
    return fathom_scan_topk(index, q_bf16, t, t_union, k, out_idx, out_score, scratch,
                            kStaticScratchBytes, flags, stream);
}
