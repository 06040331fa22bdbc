// Append path: the decode step's new keys into an existing b-bit K index
// (b = 4, or 8 for the 8-plane variant).
//
// Source: Fathom explainer (papers.ananclaw.com, arXiv 2609.17652),
// section 核心方法 / 存储侧 (per-channel 4-bit quantisation stored as
// MSB-first bit planes) and 适用边界 (the 4-bit K cache comes from the
// serving stack, which grows it by one key per decode step).  A new key is
// quantised with the index's stored min and scale in the quantiser's own
// float32 steps, its level clamped to 0..2^b-1 (a key outside the stored
// range takes the nearest level, and the clamp is counted per channel as
// the measure of range drift), its bits are ORed into the zero padding
// words past the last key, the exact sums S1, S2 grow, and sigma^2 is
// recomputed for the new key count (by the appending thread itself when
// all new keys fall in one plane word, the decode step's case).
//
// One thread per (KV head, plane word, channel), channel fastest: it owns
// the up-to-32 new keys of that word for that channel, so every plane word
// has a single writer and the key loads of a warp are contiguous channels.
#include "common.cuh"
#include "internal.h"

namespace fathom {
namespace {

template <int BITS>
__global__ void __launch_bounds__(256)
append_kernel(const float *__restrict__ keys, int H, int n, int m, int d, int n_words,
              const float *__restrict__ mn, const float *__restrict__ scale, uint32_t *planes,
              int64_t *s1, int64_t *s2, float *sigma2, uint32_t *clamped, int *status)
{
    const int w_first = n >> 5;
    const int words = ((n + m - 1) >> 5) - w_first + 1;
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (tid >= (long long)H * words * d) return;
    const int c = (int)(tid % d);
    const long long rest = tid / d;
    const int wi = (int)(rest % words), h = (int)(rest / words);
    const int w = w_first + wi;
    const int j_lo = max(n, w * 32), j_hi = min(n + m, w * 32 + 32);
    const int hc = h * d + c;
    const float lo = mn[hc], sc = scale[hc];
    constexpr int kLevels = (1 << BITS) - 1;
    uint32_t slot[BITS];
#pragma unroll
    for (int s = 0; s < BITS; ++s) slot[s] = 0u;
    unsigned long long a1 = 0, a2 = 0;
    unsigned n_clamped = 0;
    bool bad = false;
    auto take = [&](int j, float x) {
        int v = 0;
        if (!isfinite(x)) {
            bad = true;
        } else if (sc == 0.0f) {
            n_clamped += (x != lo);
        } else {
            const float level = floorf(__fadd_rn(__fdiv_rn(__fsub_rn(x, lo), sc), 0.5f));
            const bool out = level < 0.0f || level > (float)kLevels;
            n_clamped += out;
            v = level < 0.0f ? 0 : (level > (float)kLevels ? kLevels : static_cast<int>(level));
        }
#pragma unroll
        for (int s = 0; s < BITS; ++s)   // slot s holds bit BITS-1-s
            slot[s] |= (uint32_t)((v >> (BITS - 1 - s)) & 1) << (j & 31);
        a1 += (unsigned long long)v;
        a2 += (unsigned long long)(v * v);
    };
    const float *kc = keys + (size_t)h * m * d + c;   // key j at kc[(j - n) * d]
    if (j_hi - j_lo == 32) {
        // a whole word: 16 independent loads in flight per round
#pragma unroll
        for (int j0 = 0; j0 < 32; j0 += 16) {
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = kc[(size_t)(j_lo + j0 + i - n) * d];
#pragma unroll
            for (int i = 0; i < 16; ++i) take(j_lo + j0 + i, x[i]);
        }
    } else {
        for (int j = j_lo; j < j_hi; ++j) take(j, kc[(size_t)(j - n) * d]);
    }
    uint32_t *pw = planes + (size_t)hc * BITS * n_words + w;
#pragma unroll
    for (int s = 0; s < BITS; ++s)
        if (slot[s]) pw[(size_t)s * n_words] |= slot[s];
    unsigned long long *p1 = reinterpret_cast<unsigned long long *>(&s1[hc]);
    unsigned long long *p2 = reinterpret_cast<unsigned long long *>(&s2[hc]);
    if (words == 1) {
        // all new keys in one word: this thread is the channel's only writer
        // and holds its final sums
        const unsigned long long o1 = atomicAdd(p1, a1), o2 = atomicAdd(p2, a2);
        sigma2[hc] = channel_sigma2((long long)(o1 + a1), (long long)(o2 + a2), sc, n + m);
    } else {
        // several words: the sums only accumulate (no value waited for); a
        // second pass recomputes sigma^2
        atomicAdd(p1, a1);
        atomicAdd(p2, a2);
    }
    if (clamped && n_clamped) atomicAdd(&clamped[hc], n_clamped);
    if (bad) set_status(status, FATHOM_ERR_NONFINITE);
}

}  // namespace

cudaError_t launch_append(const float *keys, const fathom_index &ix, int m, uint32_t *clamped,
                          cudaStream_t stream)
{
    const int H = ix.n_kv_heads, d = ix.head_dim, n = ix.n_keys;
    const int words = ((n + m - 1) >> 5) - (n >> 5) + 1;
    const long long threads = (long long)H * words * d;
    const int block = 256;
    const long long grid = (threads + block - 1) / block;
    auto kern = index_bits(ix) == 8 ? append_kernel<8> : append_kernel<4>;
    kern<<<(unsigned)grid, block, 0, stream>>>(keys, H, n, m, d, ix.n_words, ix.mn, ix.scale,
                                               ix.planes, ix.sum_code, ix.sum_code2, ix.sigma2,
                                               clamped, device_status_ptr());
    note_launch(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || words == 1) return e;
    return launch_channel_stats(ix, n + m, stream);
}

}  // namespace fathom
