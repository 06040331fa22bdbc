// Reverse water-filling of one query by one warp (the plan kernels' core).
//
// Source: Fathom explainer (papers.ananclaw.com, arXiv 2609.17652),
// section 核心方法 / 读侧: channels are visited in order of importance
// w_c = q_c^2 sigma_c^2 and each takes min(b, remaining budget) bits (b = 4;
// 8 for the 8-plane variant), so with rank_c the position of channel c in
// (w descending, channel ascending) order, t_c = min(b, max(0, B - b*rank_c)).
// The fixed-width baselines instead read the top-r channels by |q_c| at all
// b bits.
#pragma once

#include "common.cuh"

namespace fathom {
namespace {

// Sort N composite keys held E = N/32 per lane (element e = lane*E + i)
// in descending order: bitonic network, strides below E inside the lane,
// the rest by warp shuffles.
template <int E>
__device__ __forceinline__ void warp_sort_desc(unsigned long long (&key)[E])
{
    const int lane = threadIdx.x & 31;
    constexpr int N = 32 * E;
#pragma unroll
    for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
        for (int j = size >> 1; j > 0; j >>= 1) {
            if (j < E) {
#pragma unroll
                for (int i = 0; i < E; ++i) {
                    if ((i & j) == 0) {
                        const int e = lane * E + i;
                        const bool desc = (e & size) == 0;
                        const unsigned long long a = key[i], b = key[i ^ j];
                        if ((a < b) == desc) {
                            key[i] = b;
                            key[i ^ j] = a;
                        }
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < E; ++i) {
                    const unsigned long long other = __shfl_xor_sync(0xFFFFFFFFu, key[i], j / E);
                    const int e = lane * E + i;
                    const bool desc = (e & size) == 0, low = (e & j) == 0;
                    key[i] = (low == desc) ? max(key[i], other) : min(key[i], other);
                }
            }
        }
    }
}

// One warp plans query row q_row of a KV head whose channel variances are
// sigma2_h: writes t_c to tt_row[c] for c < d (shared or global memory).
// E = head_dim padded to a power of two, / 32; bits = b.  A budget outside
// [0, b*d] sets FATHOM_ERR_INVALID_ARG (the query reads nothing); a
// non-finite importance (or |q|) sets FATHOM_ERR_NONFINITE (likewise).
template <bool kFixed, int E>
__device__ __forceinline__ void warp_plan(const uint16_t *q_row, const float *sigma2_h, int d,
                                          int bits, int B, int fixed_r, uint8_t *tt_row,
                                          int *status)
{
    const int lane = threadIdx.x & 31;
    unsigned long long key[E];
    bool bad = false;
#pragma unroll
    for (int i = 0; i < E; ++i) {
        const int c = lane * E + i;
        key[i] = 0ull;                                   // padding sorts last
        if (c < d) {
            const float qf = bf16_to_float(q_row[c]);
            float k;
            if (kFixed) {
                k = fabsf(qf);
                bad |= !isfinite(qf);
            } else {
                k = __fmul_rn(__fmul_rn(qf, qf), sigma2_h[c]);
                bad |= !isfinite(k);
            }
            key[i] = ((unsigned long long)order_key(k) << 32) | (0xFFFFFFFFu - (uint32_t)c);
        }
    }
    bad = __any_sync(0xFFFFFFFFu, bad);
    if (!kFixed && (B < 0 || B > bits * d)) {
        if (lane == 0) set_status(status, FATHOM_ERR_INVALID_ARG);
        B = 0;
    }
    if (bad && lane == 0) set_status(status, FATHOM_ERR_NONFINITE);
    warp_sort_desc<E>(key);
#pragma unroll
    for (int i = 0; i < E; ++i) {
        const int rank = lane * E + i;
        const uint32_t c = 0xFFFFFFFFu - (uint32_t)(key[i] & 0xFFFFFFFFull);
        if (key[i] != 0ull && c < (uint32_t)d) {
            int tc = kFixed ? (rank < fixed_r ? bits : 0) : min(bits, max(0, B - bits * rank));
            if (bad) tc = 0;
            tt_row[c] = (uint8_t)tc;
        }
    }
}

}  // namespace
}  // namespace fathom
