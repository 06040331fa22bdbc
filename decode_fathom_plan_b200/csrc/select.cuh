// Range-relative radix select of a CTA of kSelThreads threads over a set
// of 64-bit composites held in shared memory (shared by the selection
// kernels of the scan and by the shard merge).
#pragma once

#include "common.cuh"

namespace fathom {
namespace {

// ------------------------------------------------- range-relative radix select
// Selection over a set held in shared memory by a CTA of kSelThreads threads.
// Values are composites x = ((okey - lo) << 32) | low, where lo is the set's
// smallest order key, so the first 11-bit digit already splits the set's own
// range instead of the fixed sign/exponent bits (and bins stay sparse, so
// plain shared-memory atomics rarely collide).
constexpr int kSelThreads = 512;
constexpr int kSelBits = 11;
constexpr int kSelBins = 1 << kSelBits;
constexpr int kSelBinsPerThread = kSelBins / kSelThreads;   // 4

struct SelShared {
    unsigned hist[kSelBins];
    unsigned wsum[kSelThreads / 32];
    unsigned long long prefix;
    unsigned krem, above;
    int bin, cut, done;
    uint32_t lo, hi;
};

__device__ __forceinline__ bool high_bits_match(unsigned long long x, unsigned long long p, int top)
{
    return top >= 64 || ((x ^ p) >> top) == 0ull;
}

// Block-wide min / max of order keys (all kSelThreads threads call it).
__device__ __forceinline__ void sel_range(SelShared &ss, uint32_t lo, uint32_t hi)
{
    lo = __reduce_min_sync(0xFFFFFFFFu, lo);
    hi = __reduce_max_sync(0xFFFFFFFFu, hi);
    if (threadIdx.x == 0) { ss.lo = 0xFFFFFFFFu; ss.hi = 0u; }
    __syncthreads();
    if ((threadIdx.x & 31) == 0) { atomicMin(&ss.lo, lo); atomicMax(&ss.hi, hi); }
    __syncthreads();
}

// Exclusive prefix sum of one value per thread over the block; returns the
// thread's prefix and writes the total to *total (all threads).
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned v, unsigned *wsum, unsigned *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned y = __shfl_up_sync(0xFFFFFFFFu, inc, off);
        if (lane >= off) inc += y;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    unsigned before = inc - v, all = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
        const unsigned ws = wsum[w];
        before += (w < warp) ? ws : 0u;
        all += ws;
    }
    __syncthreads();
    *total = all;
    return before;
}

// Which bin (counting from the top) holds the krem-th largest element:
// above = elements in higher bins < krem <= above + hist[bin].  Thread t
// owns the kSelBinsPerThread bins just below 2048 - t*kSelBinsPerThread.
__device__ __forceinline__ void sel_pick(SelShared &ss)
{
    const int tid = threadIdx.x;
    unsigned h[kSelBinsPerThread], mine = 0;
#pragma unroll
    for (int i = 0; i < kSelBinsPerThread; ++i) {
        h[i] = ss.hist[kSelBins - 1 - kSelBinsPerThread * tid - i];
        mine += h[i];
    }
    unsigned total;
    const unsigned before = block_exclusive_scan(mine, ss.wsum, &total);
    const unsigned krem = ss.krem;
    if (before < krem && krem <= before + mine) {
        unsigned run = before;
#pragma unroll
        for (int i = 0; i < kSelBinsPerThread; ++i) {
            if (run < krem && krem <= run + h[i]) {
                ss.bin = kSelBins - 1 - kSelBinsPerThread * tid - i;
                ss.above = run;
            }
            run += h[i];
        }
    }
    __syncthreads();
}

// Runs the digit passes over `count` elements produced by get(i) until the
// selected set is determined.  Afterwards: selected iff
// (x >> ss.cut) >= (ss.prefix >> ss.cut).  stop_bit: lowest bit examined.
template <class Get>
__device__ void sel_run(SelShared &ss, unsigned count, unsigned k, int top, int stop_bit, Get get)
{
    if (threadIdx.x == 0) {
        ss.prefix = 0ull;
        ss.krem = k;
        ss.done = 0;
        ss.cut = stop_bit;
    }
    for (int hi_bit = top; hi_bit > stop_bit; hi_bit -= kSelBits) {
        const int shift = max(stop_bit, hi_bit - kSelBits);
        const unsigned width_mask = (1u << (hi_bit - shift)) - 1u;
#pragma unroll
        for (int i = 0; i < kSelBinsPerThread; ++i) ss.hist[threadIdx.x + i * kSelThreads] = 0;
        if (threadIdx.x == 0) { ss.bin = 0; ss.above = 0; }
        __syncthreads();
        const unsigned long long pf = ss.prefix;
        for (unsigned i = threadIdx.x; i < count; i += kSelThreads) {
            const unsigned long long x = get(i);
            if (high_bits_match(x, pf, hi_bit)) atomicAdd(&ss.hist[(unsigned)(x >> shift) & width_mask], 1u);
        }
        __syncthreads();
        sel_pick(ss);
        if (threadIdx.x == 0) {
            const unsigned b = (unsigned)ss.bin & (kSelBins - 1);
            ss.krem -= ss.above;
            ss.prefix |= (unsigned long long)b << shift;
            if (ss.hist[b] == ss.krem) {
                ss.done = 1;
                ss.cut = shift;
            }
        }
        __syncthreads();
        if (ss.done) break;
    }
}

__device__ __forceinline__ int bit_length(uint32_t v) { return v ? 32 - __clz(v) : 0; }

}  // namespace
}  // namespace fathom
