// Shared device/host definitions of the Fathom sm_100a library (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fathom.h"

namespace fathom {

constexpr int kBits = 4;          // 4-bit K cache: 4 planes per channel
constexpr int kMaxHeadDim = 256;
constexpr int kMaxGroup = 8;
constexpr int kMaxK = 4096;       // largest top-k any path supports
constexpr int kMaxFastK = 2048;   // largest top-k of the sampled-threshold path
constexpr int kMaxSessions = 64;

// Scan tiling: a tile is 64 plane words (2048 keys) of one KV head; a CTA of
// 256 threads gives each thread 8 keys (column = thread/4, key row = thread%4,
// keys 32*column + 4*m + row for m = 0..7).
constexpr int kTileCols = 64;
constexpr int kTileKeys = kTileCols * 32;
constexpr int kScanThreads = 256;
constexpr int kStageChannels = 8;                 // union channels per smem stage
constexpr int kStageRows = kStageChannels * kBits;
constexpr int kStages = 3;

// Sample-threshold sizing (see the scan launcher).
constexpr int kSampleMinKeys = 4096;
constexpr int kSampleMaxKeys = 8192;   // past this the rank is 3k*m/n (see the scan launcher)
constexpr int kSampleTargetRank = 128;

// Per-query state kept in the workspace: threshold, candidate count,
// fallback flag, spare.
constexpr int kQueryStateWords = 4;

// Device error codes written to the status word (first error wins).
__device__ __forceinline__ void set_status(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_to_float(uint16_t b)
{
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Order-preserving map float32 -> uint32 (larger float -> larger key);
// -0 is canonicalised to +0 first so equal scores get equal keys.
__device__ __forceinline__ uint32_t order_key(float f)
{
    f = f + 0.0f;
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float order_key_to_float(uint32_t k)
{
    uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(u);
}

// Composite selection key: score order key in the high word, complemented
// key index in the low word, so larger composite = higher score, then lower
// index.  Unique per key.
__device__ __forceinline__ unsigned long long composite(uint32_t okey, uint32_t j)
{
    return (static_cast<unsigned long long>(okey) << 32) | static_cast<unsigned long long>(~j);
}

// Variance of the stored 4-bit keys of a channel from its exact sums:
// scale^2 * (n*S2 - S1^2) / n^2 in fp64, rounded once to float32 (the
// importance weight of the read side).
__device__ __forceinline__ float channel_sigma2(long long s1, long long s2, float scale, long long n)
{
    const long long num = n * s2 - s1 * s1;
    const double sc = (double)scale;
    const double sc2 = __dmul_rn(sc, sc);
    const double frac = __ddiv_rn((double)num, __dmul_rn((double)n, (double)n));
    return __double2float_rn(__dmul_rn(sc2, frac));
}

}  // namespace fathom
