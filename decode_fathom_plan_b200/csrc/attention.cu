// Attention over the keys the scan selected: the step after the scan.
//
// Source: Fathom explainer (papers.ananclaw.com, arXiv 2609.17652),
// section 解决什么真问题: each decode step scores the keys to decide which
// K/V rows of the offloaded cache to fetch, then attends over those; its
// experiments report the resulting attention error.  Here query g of KV
// head h attends over the k keys of its top-k: logits l_i = scale *
// (q . K[h][idx_i]), p = softmax(l), out = sum_i p_i V[h][idx_i], in fp32
// with the running-max (online) softmax.
//
// Split-K: a query's k keys are cut into runs of kKeysPerSplit, one CTA each
// (so a layer's 32 queries x k = 2048 keys fill the GPU); warp w of a CTA
// takes every 8th key of the run, 4 K and 4 V rows in flight, lane l holding
// channels [l*E, l*E + E) of d = 32*E.  Each CTA writes its (max, sum,
// partial output); the combine kernel rescales and adds them per query.
// K and V may be device memory or pinned, mapped host memory.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace fathom {
namespace {

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kKeysPerSplit = 128;
constexpr int kRowsInFlight = 4;

template <int E>
struct Row {
    float v[E];
};

// A lane's E channels of one row: 16-byte loads when E is a multiple of 4
// (the lane's offset is then 16-byte aligned), 8-byte when even, else 4.
template <int E>
__device__ __forceinline__ Row<E> load_row(const float *p)
{
    Row<E> r;
    if constexpr (E % 4 == 0) {
#pragma unroll
        for (int e = 0; e < E; e += 4) {
            const float4 a = *reinterpret_cast<const float4 *>(p + e);
            r.v[e] = a.x; r.v[e + 1] = a.y; r.v[e + 2] = a.z; r.v[e + 3] = a.w;
        }
    } else if constexpr (E % 2 == 0) {
#pragma unroll
        for (int e = 0; e < E; e += 2) {
            const float2 a = *reinterpret_cast<const float2 *>(p + e);
            r.v[e] = a.x; r.v[e + 1] = a.y;
        }
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) r.v[e] = p[e];
    }
    return r;
}

// grid (splits, Q).  part: [Q][splits][d + 2] = partial output, max, sum.
template <int E>
__global__ void __launch_bounds__(kAttnThreads)
attention_split_kernel(const float *__restrict__ keys, const float *__restrict__ values, int G,
                       int n, const uint16_t *__restrict__ q_bf16,
                       const int32_t *__restrict__ idx, int k, float scale, float *part,
                       int *status)
{
    constexpr int d = 32 * E;
    __shared__ float s_m[kAttnWarps], s_l[kAttnWarps];
    __shared__ float s_o[kAttnWarps][d];
    const int qq = blockIdx.y, split = blockIdx.x, splits = gridDim.x;
    const int h = qq / G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *kh = keys + (size_t)h * n * d + lane * E;
    const float *vh = values + (size_t)h * n * d + lane * E;
    float q[E];
#pragma unroll
    for (int e = 0; e < E; ++e) q[e] = bf16_to_float(q_bf16[(size_t)qq * d + lane * E + e]);
    const int i0 = split * kKeysPerSplit, i1 = min(k, i0 + kKeysPerSplit);
    const int32_t *ix = idx + (size_t)qq * k;
    float m = -INFINITY, l = 0.0f, o[E];
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = 0.0f;
    bool bad = false;
    for (int base = i0 + warp; base < i1; base += kAttnWarps * kRowsInFlight) {
        int j[kRowsInFlight];
        Row<E> kr[kRowsInFlight], vr[kRowsInFlight];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            const int i = base + u * kAttnWarps;
            j[u] = (i < i1) ? ix[i] : -1;
            if (i < i1 && (j[u] < 0 || j[u] >= n)) { bad = true; j[u] = -1; }
            if (j[u] >= 0) {
                kr[u] = load_row<E>(kh + (size_t)j[u] * d);
                vr[u] = load_row<E>(vh + (size_t)j[u] * d);
            }
        }
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            if (j[u] < 0) continue;   // warp-uniform: every lane holds the same j
            float dot = 0.0f;
#pragma unroll
            for (int e = 0; e < E; ++e) dot = fmaf(q[e], kr[u].v[e], dot);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, off);
            const float logit = scale * dot;
            const float m_new = fmaxf(m, logit);
            const float corr = expf(m - m_new);
            const float p = expf(logit - m_new);
            l = l * corr + p;
#pragma unroll
            for (int e = 0; e < E; ++e) o[e] = o[e] * corr + p * vr[u].v[e];
            m = m_new;
        }
    }
    if (bad && lane == 0) set_status(status, FATHOM_ERR_INVALID_ARG);
    if (lane == 0) { s_m[warp] = m; s_l[warp] = l; }
#pragma unroll
    for (int e = 0; e < E; ++e) s_o[warp][lane * E + e] = o[e];
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_m[w]);
    float *pq = part + ((size_t)qq * splits + split) * (d + 2);
    for (int c = threadIdx.x; c < d; c += kAttnThreads) {
        float acc = 0.0f;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w)
            if (s_m[w] != -INFINITY) acc += s_o[w][c] * expf(s_m[w] - M);
        pq[c] = acc;
    }
    if (threadIdx.x == 0) {
        float L = 0.0f;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w)
            if (s_m[w] != -INFINITY) L += s_l[w] * expf(s_m[w] - M);
        pq[d] = M;
        pq[d + 1] = L;
    }
}

// One CTA per query: out = sum_s o_s e^(m_s - M) / sum_s l_s e^(m_s - M).
__global__ void __launch_bounds__(kAttnThreads)
attention_combine_kernel(const float *part, int splits, int d, float *out)
{
    const int qq = blockIdx.x;
    const float *pq = part + (size_t)qq * splits * (d + 2);
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, pq[(size_t)s * (d + 2) + d]);
    float L = 0.0f;
    for (int s = 0; s < splits; ++s) {
        const float ms = pq[(size_t)s * (d + 2) + d];
        if (ms != -INFINITY) L += pq[(size_t)s * (d + 2) + d + 1] * expf(ms - M);
    }
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float acc = 0.0f;
        for (int s = 0; s < splits; ++s) {
            const float ms = pq[(size_t)s * (d + 2) + d];
            if (ms != -INFINITY) acc += pq[(size_t)s * (d + 2) + c] * expf(ms - M);
        }
        out[(size_t)qq * d + c] = acc / L;
    }
}

}  // namespace

int attention_splits(int k) { return (k + kKeysPerSplit - 1) / kKeysPerSplit; }

cudaError_t launch_attention(const float *keys, const float *values, int H, int G, int d, int n,
                             const uint16_t *q_bf16, const int32_t *idx, int k, float scale,
                             float *out, float *part, cudaStream_t stream)
{
    const int Q = H * G, splits = attention_splits(k);
    const dim3 grid(splits, Q);
    int *status = device_status_ptr();
    switch (d / 32) {
    case 1: attention_split_kernel<1><<<grid, kAttnThreads, 0, stream>>>(keys, values, G, n, q_bf16, idx, k, scale, part, status); break;
    case 2: attention_split_kernel<2><<<grid, kAttnThreads, 0, stream>>>(keys, values, G, n, q_bf16, idx, k, scale, part, status); break;
    case 3: attention_split_kernel<3><<<grid, kAttnThreads, 0, stream>>>(keys, values, G, n, q_bf16, idx, k, scale, part, status); break;
    case 4: attention_split_kernel<4><<<grid, kAttnThreads, 0, stream>>>(keys, values, G, n, q_bf16, idx, k, scale, part, status); break;
    case 5: attention_split_kernel<5><<<grid, kAttnThreads, 0, stream>>>(keys, values, G, n, q_bf16, idx, k, scale, part, status); break;
    case 6: attention_split_kernel<6><<<grid, kAttnThreads, 0, stream>>>(keys, values, G, n, q_bf16, idx, k, scale, part, status); break;
    case 7: attention_split_kernel<7><<<grid, kAttnThreads, 0, stream>>>(keys, values, G, n, q_bf16, idx, k, scale, part, status); break;
    default: attention_split_kernel<8><<<grid, kAttnThreads, 0, stream>>>(keys, values, G, n, q_bf16, idx, k, scale, part, status); break;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attention_combine_kernel<<<Q, 128, 0, stream>>>(part, splits, d, out);
    note_launch(2);
    return cudaGetLastError();
}

}  // namespace fathom
