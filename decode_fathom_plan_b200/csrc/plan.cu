// Read-side planner of the Fathom scan: per-query reverse water-filling over
// variance-weighted channel importance, the GQA union and byte accounting.
//
// Source: Fathom explainer (papers.ananclaw.com, arXiv 2609.17652),
// section 核心方法 / 读侧: each query holds a total bit budget B; channels get
// bits in order of importance w_c (key-channel variance as the weight), up
// to 4 bits each (8 for the 8-plane variant of 部署前必读 item 3), and
// unimportant channels may get 0; the bytes read are
// sum_c t_c * bytes_per_plane(c).  The explainer's lineage notes suggest
// sharing across a GQA group; here a KV head reads the union of its
// queries' planes.
//
// One CTA per KV head, one warp per query head: the warp sorts the query's
// channels by (w descending, channel ascending) in registers, so channel
// c's position is rank_c and t_c = min(b, max(0, B - b*rank_c)).
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "plan_warp.cuh"

namespace fathom {
namespace {

// One CTA per KV head, one warp per query head.  Each warp sorts its
// query's channels by (key descending, channel ascending) with a warp
// bitonic network; a channel's position in that order is its rank, and
// t_c = min(b, max(0, B - b*rank)) (or b for the first r under the fixed
// plan).  E = padded head_dim / 32.
template <bool kFixed, int E>
__global__ void __launch_bounds__(kMaxGroup * 32)
plan_kernel(const uint16_t *__restrict__ q, const int32_t *__restrict__ budget, int32_t fixed_r,
            const float *__restrict__ sigma2, int G, int d, int bits, int n_words, uint8_t *t,
            uint8_t *t_union, uint64_t *bytes, int Q, int *status)
{
    __shared__ uint8_t tt[kMaxGroup][kMaxHeadDim];
    const int h = blockIdx.x;
    const int g = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned long long plane_bytes = 4ull * (unsigned long long)n_words;
    const int qi = h * G + g;
    warp_plan<kFixed, E>(q + (size_t)qi * d, sigma2 + h * d, d, bits, kFixed ? 0 : budget[qi],
                         fixed_r, tt[g], status);
    __syncwarp();
    unsigned long long my_bytes = 0;
    for (int c = lane; c < d; c += 32) {
        t[(size_t)qi * d + c] = tt[g][c];
        my_bytes += (unsigned long long)tt[g][c] * plane_bytes;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) my_bytes += __shfl_xor_sync(0xFFFFFFFFu, my_bytes, off);
    if (lane == 0) bytes[qi] = my_bytes;
    __syncthreads();
    // GQA union, one warp per 32 channels
    if (g == 0) {
        unsigned long long ub = 0;
        for (int c = lane; c < d; c += 32) {
            uint8_t m = 0;
            for (int gg = 0; gg < G; ++gg) m = max(m, tt[gg][c]);
            t_union[h * d + c] = m;
            ub += (unsigned long long)m * plane_bytes;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ub += __shfl_xor_sync(0xFFFFFFFFu, ub, off);
        if (lane == 0) bytes[Q + h] = ub;
    }
}

// Marginal-gain plan (a finer reverse water-filling; the explainer's walk
// hands out whole 4-bit channels, 核心方法 / 读侧): bit s+1 of channel c is
// worth w_c * 4^-s, the B most valuable (channel, bit) pairs are read, ties
// to the lower channel then the lower bit.  A warp sorts the b*d pairs of
// its query (value as an order key, then ~(b*c + s)); since a channel's
// values fall with s, the selected bits of a channel are a prefix and t_c is
// one past its deepest selected bit.  4^-s is a power of two, so the values
// are exact.  E = padded head_dim / 32; BITS = b, the cap per channel.
template <int E, int BITS>
__global__ void __launch_bounds__(kMaxGroup * 32)
plan_marginal_kernel(const uint16_t *__restrict__ q, const int32_t *__restrict__ budget,
                     const float *__restrict__ sigma2, int G, int d, int n_words, uint8_t *t,
                     uint8_t *t_union, uint64_t *bytes, int Q, int *status)
{
    constexpr int E4 = BITS * E;
    __shared__ int tt[kMaxGroup][kMaxHeadDim];
    const int h = blockIdx.x;
    const int g = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned long long plane_bytes = 4ull * (unsigned long long)n_words;
    const int qi = h * G + g;
    unsigned long long key[E4];
    bool bad = false;
#pragma unroll
    for (int i = 0; i < E; ++i) {
        const int c = lane * E + i;
        float w = 0.0f;
        if (c < d) {
            const float qf = bf16_to_float(q[(size_t)qi * d + c]);
            w = __fmul_rn(__fmul_rn(qf, qf), sigma2[h * d + c]);
            bad |= !isfinite(w);
            tt[g][c] = 0;
        }
#pragma unroll
        for (int s = 0; s < BITS; ++s) {
            const float gain = __fmul_rn(w, 1.0f / (float)(1 << (2 * s)));   // exact
            key[i * BITS + s] = (c < d) ? (((unsigned long long)order_key(gain) << 32) |
                                           (0xFFFFFFFFu - (uint32_t)(c * BITS + s)))
                                        : 0ull;
        }
    }
    bad = __any_sync(0xFFFFFFFFu, bad);
    int B = budget[qi];
    if (B < 0 || B > BITS * d) {
        if (lane == 0) set_status(status, FATHOM_ERR_INVALID_ARG);
        B = 0;
    }
    if (bad) {
        if (lane == 0) set_status(status, FATHOM_ERR_NONFINITE);
        B = 0;
    }
    __syncwarp();
    warp_sort_desc<E4>(key);
#pragma unroll
    for (int i = 0; i < E4; ++i) {
        const int rank = lane * E4 + i;
        if (rank < B && key[i] != 0ull) {
            const uint32_t cs = 0xFFFFFFFFu - (uint32_t)(key[i] & 0xFFFFFFFFull);
            atomicMax(&tt[g][cs / BITS], (int)(cs % BITS) + 1);
        }
    }
    __syncwarp();
    unsigned long long my_bytes = 0;
#pragma unroll
    for (int i = 0; i < E; ++i) {
        const int c = lane * E + i;
        if (c < d) {
            t[(size_t)qi * d + c] = (uint8_t)tt[g][c];
            my_bytes += (unsigned long long)tt[g][c] * plane_bytes;
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) my_bytes += __shfl_xor_sync(0xFFFFFFFFu, my_bytes, off);
    if (lane == 0) bytes[qi] = my_bytes;
    __syncthreads();
    if (g == 0) {   // GQA union, one warp
        unsigned long long ub = 0;
        for (int c = lane; c < d; c += 32) {
            int m = 0;
            for (int gg = 0; gg < G; ++gg) m = max(m, tt[gg][c]);
            t_union[h * d + c] = (uint8_t)m;
            ub += (unsigned long long)m * plane_bytes;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ub += __shfl_xor_sync(0xFFFFFFFFu, ub, off);
        if (lane == 0) bytes[Q + h] = ub;
    }
}

template <bool kFixed>
void launch_plan_kernel(int E, dim3 grid, int threads, cudaStream_t stream, const uint16_t *q,
                        const int32_t *budget, int32_t fixed_r, const float *sigma2, int G, int d,
                        int bits, int n_words, uint8_t *t, uint8_t *t_union, uint64_t *bytes,
                        int Q, int *status)
{
    switch (E) {
    case 1: plan_kernel<kFixed, 1><<<grid, threads, 0, stream>>>(q, budget, fixed_r, sigma2, G, d, bits, n_words, t, t_union, bytes, Q, status); break;
    case 2: plan_kernel<kFixed, 2><<<grid, threads, 0, stream>>>(q, budget, fixed_r, sigma2, G, d, bits, n_words, t, t_union, bytes, Q, status); break;
    case 4: plan_kernel<kFixed, 4><<<grid, threads, 0, stream>>>(q, budget, fixed_r, sigma2, G, d, bits, n_words, t, t_union, bytes, Q, status); break;
    default: plan_kernel<kFixed, 8><<<grid, threads, 0, stream>>>(q, budget, fixed_r, sigma2, G, d, bits, n_words, t, t_union, bytes, Q, status); break;
    }
}

template <int BITS>
void launch_marginal_kernel(int E, dim3 grid, int threads, cudaStream_t stream,
                            const uint16_t *q, const int32_t *budget, const float *sigma2, int G,
                            int d, int n_words, uint8_t *t, uint8_t *t_union, uint64_t *bytes,
                            int Q, int *status)
{
    switch (E) {
    case 1: plan_marginal_kernel<1, BITS><<<grid, threads, 0, stream>>>(q, budget, sigma2, G, d, n_words, t, t_union, bytes, Q, status); break;
    case 2: plan_marginal_kernel<2, BITS><<<grid, threads, 0, stream>>>(q, budget, sigma2, G, d, n_words, t, t_union, bytes, Q, status); break;
    case 4: plan_marginal_kernel<4, BITS><<<grid, threads, 0, stream>>>(q, budget, sigma2, G, d, n_words, t, t_union, bytes, Q, status); break;
    default:
        if constexpr (BITS == 4)   // head_dim <= 128 when b = 8
            plan_marginal_kernel<8, BITS><<<grid, threads, 0, stream>>>(q, budget, sigma2, G, d, n_words, t, t_union, bytes, Q, status);
        break;
    }
}

}  // namespace

cudaError_t launch_plan_marginal(const fathom_index &ix, const uint16_t *q, const int32_t *budget,
                                 uint8_t *t, uint8_t *t_union, uint64_t *bytes, cudaStream_t stream)
{
    const int H = ix.n_kv_heads, G = ix.group, d = ix.head_dim;
    const int Q = H * G;
    int *status = device_status_ptr();
    int E = 1;
    while (32 * E < d) E <<= 1;
    const dim3 grid(H);
    const int threads = G * 32;
    if (index_bits(ix) == 8)
        launch_marginal_kernel<8>(E, grid, threads, stream, q, budget, ix.sigma2, G, d,
                                  ix.n_words, t, t_union, bytes, Q, status);
    else
        launch_marginal_kernel<4>(E, grid, threads, stream, q, budget, ix.sigma2, G, d,
                                  ix.n_words, t, t_union, bytes, Q, status);
    note_launch(1);
    return cudaGetLastError();
}

cudaError_t launch_plan(const fathom_index &ix, const uint16_t *q, const int32_t *budget,
                        int32_t fixed_r, bool fixed, uint8_t *t, uint8_t *t_union,
                        uint64_t *bytes, cudaStream_t stream)
{
    const int H = ix.n_kv_heads, G = ix.group, d = ix.head_dim;
    const int Q = H * G;
    int *status = device_status_ptr();
    int E = 1;
    while (32 * E < d) E <<= 1;   // head_dim padded to a power of two
    const int bits = index_bits(ix);
    if (fixed)
        launch_plan_kernel<true>(E, dim3(H), G * 32, stream, q, budget, fixed_r, ix.sigma2, G, d,
                                 bits, ix.n_words, t, t_union, bytes, Q, status);
    else
        launch_plan_kernel<false>(E, dim3(H), G * 32, stream, q, budget, fixed_r, ix.sigma2, G, d,
                                  bits, ix.n_words, t, t_union, bytes, Q, status);
    note_launch(1);
    return cudaGetLastError();
}

}  // namespace fathom
