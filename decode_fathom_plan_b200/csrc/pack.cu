// Storage side of the Fathom scan: per-channel b-bit min/max quantisation
// (b = 4, or 8 for the 8-plane variant), channel-major MSB-first bit planes
// and exact channel statistics.
//
// Source: Fathom explainer (papers.ananclaw.com, arXiv 2609.17652),
// section 核心方法 / 存储侧: the K cache is quantised to 4 bits, laid out
// channel-major, and each channel's 4 bits are split into bit planes so that
// the first t planes of a channel are its t-bit quantiser; 部署前必读 item 3:
// an 8-bit upstream K cache needs the index adapted to 8 planes.
//
// Four small kernels (the index build is off the decode path):
//   init    ordered-key min/max accumulators, zero the integer sums
//   minmax  per (h, c) min and max over all n keys (exact, via atomics on
//           order-preserving integer keys)
//   range   mn and scale = (max - min) / (2^b - 1) per (h, c)
//   quant   codes -> b ballots per 32-key word -> plane rows staged in shared
//           memory and written 128 bytes at a time; code sums from popcounts
//   stats   sigma^2 = scale^2 * (n*S2 - S1^2) / n^2 in fp64
#include "common.cuh"
#include "internal.h"

namespace fathom {
namespace {

constexpr int kMinMaxKeysPerBlock = 1024;
constexpr int kQuantWordsPerBlock = 32;   // 1024 keys, 128-byte plane rows
constexpr int kQuantThreads = 256;

__global__ void pack_init_kernel(uint32_t *ws_min, uint32_t *ws_max, int64_t *s1, int64_t *s2,
                                 int count)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < count) {
        ws_min[i] = 0xFFFFFFFFu;
        ws_max[i] = 0u;
        s1[i] = 0;
        s2[i] = 0;
    }
}

// grid (ceil(n / 1024), H), block d threads: thread c owns channel c.
__global__ void pack_minmax_kernel(const float *__restrict__ keys, int n, int d,
                                   uint32_t *ws_min, uint32_t *ws_max, int *status)
{
    const int h = blockIdx.y;
    const int c = threadIdx.x;
    const int j0 = blockIdx.x * kMinMaxKeysPerBlock;
    const int j1 = min(n, j0 + kMinMaxKeysPerBlock);
    const float *kh = keys + (size_t)h * n * d;
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    bool bad = false;
    for (int j = j0; j < j1; ++j) {
        float x = kh[(size_t)j * d + c];
        bad |= !isfinite(x);
        uint32_t o = order_key(x);
        lo = min(lo, o);
        hi = max(hi, o);
    }
    if (bad) set_status(status, FATHOM_ERR_NONFINITE);
    if (j0 < j1) {
        atomicMin(&ws_min[h * d + c], lo);
        atomicMax(&ws_max[h * d + c], hi);
    }
}

__global__ void pack_range_kernel(const uint32_t *ws_min, const uint32_t *ws_max, float *mn,
                                  float *scale, int count, int levels)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count) return;
    float lo = order_key_to_float(ws_min[i]);
    float hi = order_key_to_float(ws_max[i]);
    mn[i] = lo;
    scale[i] = (hi == lo) ? 0.0f : __fdiv_rn(__fsub_rn(hi, lo), (float)levels);
}

template <int BITS>
__device__ __forceinline__ uint32_t quantize_code(float x, float lo, float sc)
{
    constexpr int kLevels = (1 << BITS) - 1;
    if (sc == 0.0f) return 0u;
    float ratio = __fdiv_rn(__fsub_rn(x, lo), sc);
    float level = floorf(__fadd_rn(ratio, 0.5f));
    int v = static_cast<int>(level);
    v = v < 0 ? 0 : (v > kLevels ? kLevels : v);
    return static_cast<uint32_t>(v);
}

// grid (ceil(n_words / 32), H), block 256 = 8 warps; a warp quantises one
// 32-key word at a time (lane = key) over all d channels; dynamic shared
// memory holds the CTA's 32-word slice of every plane row (d*BITS rows).
template <int BITS>
__global__ void __launch_bounds__(kQuantThreads)
pack_quant_kernel(const float *__restrict__ keys, int n, int d, int n_words,
                  const float *__restrict__ mn, const float *__restrict__ scale,
                  uint32_t *planes, int64_t *s1, int64_t *s2)
{
    extern __shared__ uint32_t rows[];               // [d*BITS][32]
    __shared__ unsigned long long sum1[kMaxHeadDim], sum2[kMaxHeadDim];
    const int h = blockIdx.y;
    const int w0 = blockIdx.x * kQuantWordsPerBlock;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int c = threadIdx.x; c < d; c += blockDim.x) { sum1[c] = 0; sum2[c] = 0; }
    __syncthreads();

    const float *kh = keys + (size_t)h * n * d;
    const float *mnh = mn + h * d;
    const float *sch = scale + h * d;
    for (int wl = warp; wl < kQuantWordsPerBlock; wl += kQuantThreads / 32) {
        const int j = (w0 + wl) * 32 + lane;
        const bool live = j < n;
        const float *krow = kh + (size_t)(live ? j : 0) * d;
        for (int c = 0; c < d; ++c) {
            const uint32_t code = live ? quantize_code<BITS>(krow[c], mnh[c], sch[c]) : 0u;
            uint32_t b[BITS];   // b[p]: ballot of bit p
#pragma unroll
            for (int p = 0; p < BITS; ++p) b[p] = __ballot_sync(0xFFFFFFFFu, (code >> p) & 1u);
            // slot s holds bit BITS-1-s (slot 0 = most significant)
            if (lane < BITS) {
                uint32_t word = 0u;
#pragma unroll
                for (int p = 0; p < BITS; ++p)
                    if (lane == BITS - 1 - p) word = b[p];
                rows[(c * BITS + lane) * kQuantWordsPerBlock + wl] = word;
            }
            if (lane == (c & 31)) {
                // sum code = sum_p 2^p popc(b_p); sum code^2 = sum_{p,p'} 2^(p+p') popc(b_p & b_p')
                unsigned long long a1 = 0, a2 = 0;
#pragma unroll
                for (int p = 0; p < BITS; ++p) {
                    a1 += (unsigned long long)__popc(b[p]) << p;
#pragma unroll
                    for (int pp = 0; pp < BITS; ++pp)
                        a2 += (unsigned long long)__popc(b[p] & b[pp]) << (p + pp);
                }
                atomicAdd(&sum1[c], a1);
                atomicAdd(&sum2[c], a2);
            }
        }
    }
    __syncthreads();
    // 128-byte row segments: thread -> (row, word)
    const int n_rows = d * BITS;
    for (int e = threadIdx.x; e < n_rows * kQuantWordsPerBlock; e += blockDim.x) {
        const int row = e / kQuantWordsPerBlock, wl = e % kQuantWordsPerBlock;
        const int w = w0 + wl;
        if (w < n_words)
            planes[((size_t)h * n_rows + row) * n_words + w] = rows[row * kQuantWordsPerBlock + wl];
    }
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        atomicAdd(reinterpret_cast<unsigned long long *>(&s1[h * d + c]), sum1[c]);
        atomicAdd(reinterpret_cast<unsigned long long *>(&s2[h * d + c]), sum2[c]);
    }
}

__global__ void pack_stats_kernel(const int64_t *s1, const int64_t *s2, const float *scale,
                                  float *sigma2, int n, int count)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count) return;
    sigma2[i] = channel_sigma2(s1[i], s2[i], scale[i], n);
}

}  // namespace

cudaError_t launch_pack(const float *keys, const fathom_index &ix, uint32_t *ws_minmax,
                        cudaStream_t stream)
{
    const int H = ix.n_kv_heads, d = ix.head_dim, n = ix.n_keys, n_words = ix.n_words;
    const int bits = index_bits(ix);
    const int count = H * d;
    uint32_t *ws_min = ws_minmax, *ws_max = ws_minmax + count;
    int *status = device_status_ptr();
    const int eb = 256, eg = (count + eb - 1) / eb;

    pack_init_kernel<<<eg, eb, 0, stream>>>(ws_min, ws_max, ix.sum_code, ix.sum_code2, count);
    dim3 g1((n + kMinMaxKeysPerBlock - 1) / kMinMaxKeysPerBlock, H);
    pack_minmax_kernel<<<g1, d, 0, stream>>>(keys, n, d, ws_min, ws_max, status);
    pack_range_kernel<<<eg, eb, 0, stream>>>(ws_min, ws_max, ix.mn, ix.scale, count,
                                             (1 << bits) - 1);
    const size_t smem = (size_t)d * bits * kQuantWordsPerBlock * sizeof(uint32_t);
    auto kern = bits == 8 ? pack_quant_kernel<8> : pack_quant_kernel<4>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 g2((n_words + kQuantWordsPerBlock - 1) / kQuantWordsPerBlock, H);
    kern<<<g2, kQuantThreads, smem, stream>>>(keys, n, d, n_words, ix.mn, ix.scale, ix.planes,
                                              ix.sum_code, ix.sum_code2);
    note_launch(4);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_channel_stats(ix, n, stream);
}

cudaError_t launch_channel_stats(const fathom_index &ix, int n, cudaStream_t stream)
{
    const int count = ix.n_kv_heads * ix.head_dim;
    const int eb = 256, eg = (count + eb - 1) / eb;
    pack_stats_kernel<<<eg, eb, 0, stream>>>(ix.sum_code, ix.sum_code2, ix.scale, ix.sigma2, n,
                                             count);
    note_launch(1);
    return cudaGetLastError();
}

}  // namespace fathom
