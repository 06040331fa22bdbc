// Host-link read probe: reads a pinned, device-mapped host buffer (or any
// device-visible buffer) with 16-byte loads from every SM, the way the scan
// reads host-resident planes, so a benchmark can state the zero-copy read
// bandwidth of the link it measures against.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace fathom {
namespace {

__global__ void __launch_bounds__(256) link_probe_kernel(const uint4 *__restrict__ src,
                                                         size_t n16, unsigned long long *sink)
{
    uint32_t acc = 0;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    // 4 independent loads in flight per thread
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 a = src[i], b = src[i + stride], c = src[i + 2 * stride], d = src[i + 3 * stride];
        acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^
               d.z ^ d.w;
    }
    for (; i < n16; i += stride) {
        const uint4 a = src[i];
        acc ^= a.x ^ a.y ^ a.z ^ a.w;
    }
    if (acc == 0x9E3779B9u) atomicAdd(sink, 1ull);   // keeps the loads; practically never taken
}

}  // namespace
}  // namespace fathom

extern "C" fathom_status fathom_link_probe(const void *buffer, size_t bytes,
                                           unsigned long long *sink, cudaStream_t stream)
{
    if (!buffer || !sink || bytes < 16 || (reinterpret_cast<uintptr_t>(buffer) & 15u))
        return FATHOM_ERR_INVALID_ARG;
    const void *dptr = buffer;
    cudaPointerAttributes attr{};
    if (cudaPointerGetAttributes(&attr, buffer) != cudaSuccess) {
        cudaGetLastError();
        return FATHOM_ERR_INVALID_ARG;
    }
    if (attr.type == cudaMemoryTypeHost) {
        void *p = nullptr;
        if (cudaHostGetDevicePointer(&p, const_cast<void *>(buffer), 0) != cudaSuccess || !p) {
            cudaGetLastError();
            return FATHOM_ERR_INVALID_ARG;
        }
        dptr = p;
    } else if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) {
        return FATHOM_ERR_INVALID_ARG;
    }
    int dev = 0, n_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    fathom::link_probe_kernel<<<std::max(1, n_sm) * 8, 256, 0, stream>>>(
        static_cast<const uint4 *>(dptr), bytes / 16, sink);
    fathom::note_launch(1);
    return cudaGetLastError() == cudaSuccess ? FATHOM_OK : FATHOM_ERR_CUDA;
}
