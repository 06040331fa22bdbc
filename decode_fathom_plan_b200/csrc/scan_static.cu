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
// stand-in, not a device address), so every call looks up the device address
// with cudaGetSymbolAddress while the call's device is current (a call costs
// little next to the scan's launches, and nothing here goes stale).  The rest
// of the library still keeps per-device state for the life of the process,
// so no call may follow a cudaDeviceReset of the device.
#include "common.cuh"
#include "internal.h"

// 8 MiB: a device index of 64 query heads at 1,048,576 keys with k <= 2048
// needs about 6.3 MiB (per-query state, candidate buffers, per-KV-head scan
// tables).  A host-resident index also needs room for the two-slot ring its
// planes are fetched into, so only small host-resident indices fit.
static constexpr size_t kStaticScratchBytes = 8u << 20;
static __device__ __align__(256) unsigned char g_scan_scratch[kStaticScratchBytes];

namespace {
// Device address of g_scan_scratch on the current device.
fathom_status static_scratch(void **out)
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scan_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return FATHOM_ERR_CUDA;
    }
    *out = p;
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
