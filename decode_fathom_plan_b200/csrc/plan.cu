// Read-side planner of the Fathom scan: per-query reverse water-filling over
// variance-weighted channel importance, the GQA union and byte accounting.
//
// Source: Fathom explainer (papers.ananclaw.com, arXiv 2609.17652),
// section 核心方法 / 读侧: each query holds a total bit budget B; channels get
// bits in order of importance w_c (key-channel variance as the weight), up
// to 4 bits each, and unimportant channels may get 0; the bytes read are
// sum_c t_c * bytes_per_plane(c).  The explainer's lineage notes suggest
// sharing across a GQA group; here a KV head reads the union of its
// queries' planes.
//
// One CTA per KV head, one warp per query head; d <= 256 channels, so each
// lane owns d/32 channels.  Ranks come from counting (w' > w, or w' == w and
// c' < c) over the d importances in shared memory, which gives
// t_c = min(4, max(0, B - 4*rank_c)) without a sort.
#include "common.cuh"
#include "internal.h"

namespace fathom {
namespace {

template <bool kFixed>
__global__ void plan_kernel(const uint16_t *__restrict__ q, const int32_t *__restrict__ budget,
                            int32_t fixed_r, const float *__restrict__ sigma2, int G, int d,
                            int n_words, uint8_t *t, uint8_t *t_union, uint64_t *bytes, int Q,
                            int *status)
{
    __shared__ float key[kMaxGroup][kMaxHeadDim];
    __shared__ uint8_t tt[kMaxGroup][kMaxHeadDim];
    __shared__ unsigned long long union_bytes;
    const int h = blockIdx.x;
    const int g = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qi = h * G + g;
    const int per = d >> 5;
    const unsigned long long plane_bytes = 4ull * (unsigned long long)n_words;
    if (threadIdx.x == 0) union_bytes = 0;

    bool bad = false;
    for (int i = 0; i < per; ++i) {
        const int c = lane + 32 * i;
        const float qf = bf16_to_float(q[(size_t)qi * d + c]);
        float k;
        if (kFixed) {
            k = fabsf(qf);
            bad |= !isfinite(qf);
        } else {
            k = __fmul_rn(__fmul_rn(qf, qf), sigma2[h * d + c]);
            bad |= !isfinite(k);
        }
        key[g][c] = k;
    }
    bad = __any_sync(0xFFFFFFFFu, bad);
    int B = 0;
    if (!kFixed) {
        B = budget[qi];
        if (B < 0 || B > kBits * d) {
            set_status(status, FATHOM_ERR_INVALID_ARG);
            B = 0;
        }
    }
    if (bad) set_status(status, FATHOM_ERR_NONFINITE);
    __syncwarp();

    unsigned long long my_bytes = 0;
    for (int i = 0; i < per; ++i) {
        const int c = lane + 32 * i;
        const float kc = key[g][c];
        int rank = 0;
        for (int c2 = 0; c2 < d; ++c2) {
            const float k2 = key[g][c2];
            rank += (k2 > kc) || (k2 == kc && c2 < c);
        }
        int tc;
        if (kFixed)
            tc = rank < fixed_r ? kBits : 0;
        else
            tc = min(kBits, max(0, B - kBits * rank));
        if (bad) tc = 0;
        tt[g][c] = (uint8_t)tc;
        t[(size_t)qi * d + c] = (uint8_t)tc;
        my_bytes += (unsigned long long)tc * plane_bytes;
    }
    for (int off = 16; off > 0; off >>= 1) my_bytes += __shfl_xor_sync(0xFFFFFFFFu, my_bytes, off);
    if (lane == 0) bytes[qi] = my_bytes;
    __syncthreads();

    unsigned long long ub = 0;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        uint8_t m = 0;
        for (int gg = 0; gg < G; ++gg) m = max(m, tt[gg][c]);
        t_union[h * d + c] = m;
        ub += (unsigned long long)m * plane_bytes;
    }
    atomicAdd(&union_bytes, ub);
    __syncthreads();
    if (threadIdx.x == 0) bytes[Q + h] = union_bytes;
}

}  // namespace

cudaError_t launch_plan(const fathom_index &ix, const uint16_t *q, const int32_t *budget,
                        int32_t fixed_r, bool fixed, uint8_t *t, uint8_t *t_union,
                        uint64_t *bytes, cudaStream_t stream)
{
    const int H = ix.n_kv_heads, G = ix.group, d = ix.head_dim;
    const int Q = H * G;
    int *status = device_status_ptr();
    if (fixed)
        plan_kernel<true><<<H, G * 32, 0, stream>>>(q, budget, fixed_r, ix.sigma2, G, d,
                                                    ix.n_words, t, t_union, bytes, Q, status);
    else
        plan_kernel<false><<<H, G * 32, 0, stream>>>(q, budget, fixed_r, ix.sigma2, G, d,
                                                     ix.n_words, t, t_union, bytes, Q, status);
    note_launch(1);
    return cudaGetLastError();
}

}  // namespace fathom
