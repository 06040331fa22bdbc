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
// Grouped per-token-block scales (block_keys > 0, a multiple of 2048): each
// block of block_keys tokens is quantised on its own, so every statistic
// below is per (h, block, c) instead of per (h, c), except sigma^2, which
// stays per (h, c): the variance of all dequantised keys, combined from the
// blocks' exact sums (pairwise update of Chan, Golub and LeVeque).  A pack
// CTA covers 1024 keys and blocks hold whole multiples of 2048, so each CTA
// works inside one block.
//
// Small kernels (the index build is off the decode path):
//   init    ordered-key min/max accumulators, zero the integer sums
//   minmax  per (h, block, c) min and max (exact, via atomics on
//           order-preserving integer keys)
//   range   mn and scale = (max - min) / (2^b - 1) per (h, block, c)
//   quant   codes -> b ballots per 32-key word -> plane rows staged in shared
//           memory and written 128 bytes at a time; code sums from popcounts
//   stats   sigma^2 = scale^2 * (n*S2 - S1^2) / n^2 in fp64 (one block), or
//           the blocks' pairwise combination
// The same kernels append whole blocks to a block-scaled index (keys
// starting at position j_base, a block boundary).
#include "common.cuh"
#include "internal.h"

namespace fathom {
namespace {

constexpr int kMinMaxKeysPerBlock = 1024;
constexpr int kQuantWordsPerBlock = 32;   // 1024 keys, 128-byte plane rows
constexpr int kQuantThreads = 256;

// Where the input keys go: input key i (of n_in per head) is index key
// j_base + i; statistics rows are [H][nb][d] (nb = 1 without blocks).
struct PackGeom {
    int H, d, n_in, j_base, n_words;
    int words_out;    // plane words written from j_base/32 on (zeros past the input)
    int block_keys;   // 0: one block over all keys
    int nb;           // statistics rows per head
    int b0, n_touch;  // blocks written by this pack: b0 .. b0 + n_touch - 1
};

__device__ __forceinline__ int stat_row(const PackGeom &g, int h, int j)
{
    return h * g.nb + (g.block_keys ? j / g.block_keys : 0);
}

// (h, touched block, c) entries: accumulators and integer sums.
__global__ void pack_init_kernel(uint32_t *ws_min, uint32_t *ws_max, int64_t *s1, int64_t *s2,
                                 PackGeom g)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= g.H * g.n_touch * g.d) return;
    const int c = i % g.d, r = i / g.d;
    const int h = r / g.n_touch, bi = r % g.n_touch;
    const int e = (h * g.nb + g.b0 + bi) * g.d + c;
    ws_min[e] = 0xFFFFFFFFu;
    ws_max[e] = 0u;
    s1[e] = 0;
    s2[e] = 0;
}

// grid (ceil(n_in / 1024), H), block d threads: thread c owns channel c.
__global__ void pack_minmax_kernel(const float *__restrict__ keys, PackGeom g, uint32_t *ws_min,
                                   uint32_t *ws_max, int *status)
{
    const int h = blockIdx.y;
    const int c = threadIdx.x, d = g.d;
    const int j0 = blockIdx.x * kMinMaxKeysPerBlock;
    const int j1 = min(g.n_in, j0 + kMinMaxKeysPerBlock);
    const float *kh = keys + (size_t)h * g.n_in * d;
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
        const int e = stat_row(g, h, g.j_base + j0) * d + c;
        atomicMin(&ws_min[e], lo);
        atomicMax(&ws_max[e], hi);
    }
}

// mn, scale of the touched entries; ws_min / ws_max may alias mn / scale
// (each thread reads its entry before writing it).
__global__ void pack_range_kernel(const uint32_t *ws_min, const uint32_t *ws_max, float *mn,
                                  float *scale, PackGeom g, int levels)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= g.H * g.n_touch * g.d) return;
    const int c = i % g.d, r = i / g.d;
    const int h = r / g.n_touch, bi = r % g.n_touch;
    const int e = (h * g.nb + g.b0 + bi) * g.d + c;
    float lo = order_key_to_float(ws_min[e]);
    float hi = order_key_to_float(ws_max[e]);
    mn[e] = lo;
    scale[e] = (hi == lo) ? 0.0f : __fdiv_rn(__fsub_rn(hi, lo), (float)levels);
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

// grid (ceil(words of the input / 32), H), block 256 = 8 warps; a warp
// quantises one 32-key word at a time (lane = key) over all d channels;
// dynamic shared memory holds the CTA's 32-word slice of every plane row
// (d*BITS rows).  Plane words j_base/32 .. j_base/32 + words_out - 1 are
// written (zeros past the input's last key).
template <int BITS>
__global__ void __launch_bounds__(kQuantThreads)
pack_quant_kernel(const float *__restrict__ keys, PackGeom g, const float *__restrict__ mn,
                  const float *__restrict__ scale, uint32_t *planes, int64_t *s1, int64_t *s2)
{
    extern __shared__ uint32_t rows[];               // [d*BITS][32]
    __shared__ unsigned long long sum1[kMaxHeadDim], sum2[kMaxHeadDim];
    const int h = blockIdx.y, d = g.d, n_words = g.n_words;
    const int w0 = g.j_base / 32 + blockIdx.x * kQuantWordsPerBlock;   // first plane word
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int c = threadIdx.x; c < d; c += blockDim.x) { sum1[c] = 0; sum2[c] = 0; }
    __syncthreads();

    const float *kh = keys + (size_t)h * g.n_in * d;
    const int row0 = stat_row(g, h, w0 * 32);         // the CTA's keys share one block
    const float *mnh = mn + (size_t)row0 * d;
    const float *sch = scale + (size_t)row0 * d;
    for (int wl = warp; wl < kQuantWordsPerBlock; wl += kQuantThreads / 32) {
        const int jl = (w0 + wl) * 32 + lane - g.j_base;   // input key of this lane
        const bool live = jl < g.n_in;
        const float *krow = kh + (size_t)(live ? jl : 0) * d;
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
        if (w < n_words && w < g.j_base / 32 + g.words_out)
            planes[((size_t)h * n_rows + row) * n_words + w] = rows[row * kQuantWordsPerBlock + wl];
    }
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        atomicAdd(reinterpret_cast<unsigned long long *>(&s1[(size_t)row0 * d + c]), sum1[c]);
        atomicAdd(reinterpret_cast<unsigned long long *>(&s2[(size_t)row0 * d + c]), sum2[c]);
    }
}

__global__ void pack_stats_kernel(const int64_t *s1, const int64_t *s2, const float *scale,
                                  float *sigma2, int n, int count)
{
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count) return;
    sigma2[i] = channel_sigma2(s1[i], s2[i], scale[i], n);
}

// sigma^2 of (h, c) over n keys in blocks of block_keys: each block's mean
// and sum of squared deviations from its exact sums, combined block by block
// in order (Chan, Golub and LeVeque's pairwise update), all in fp64 with
// no fused operations.
__global__ void pack_blocked_stats_kernel(const float *mn, const float *scale, const int64_t *s1,
                                          const int64_t *s2, float *sigma2, int H, int d, int nb,
                                          int n, int block_keys)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= H * d) return;
    const int h = i / d, c = i % d;
    const int n_filled = (n + block_keys - 1) / block_keys;
    double N = 0.0, mean = 0.0, M2 = 0.0;
    for (int b = 0; b < n_filled; ++b) {
        const long long nbk = (b + 1) * (long long)block_keys <= n ? block_keys
                                                                    : n - (long long)b * block_keys;
        const size_t e = ((size_t)h * nb + b) * d + c;
        const double nbd = (double)nbk;
        const double sc = (double)scale[e];
        const double mean_b = __dadd_rn((double)mn[e], __dmul_rn(sc, __ddiv_rn((double)s1[e], nbd)));
        const long long num = nbk * s2[e] - s1[e] * s1[e];
        const double m2_b = __dmul_rn(__dmul_rn(sc, sc), __ddiv_rn((double)num, nbd));
        const double Nn = __dadd_rn(N, nbd);
        const double delta = __dsub_rn(mean_b, mean);
        mean = __dadd_rn(mean, __dmul_rn(delta, __ddiv_rn(nbd, Nn)));
        M2 = __dadd_rn(__dadd_rn(M2, m2_b),
                       __dmul_rn(__dmul_rn(delta, delta), __ddiv_rn(__dmul_rn(N, nbd), Nn)));
        N = Nn;
    }
    sigma2[h * d + c] = __double2float_rn(__ddiv_rn(M2, (double)n));
}

// The kernels of one pack over geometry g; ws_min / ws_max index like the
// statistics rows.
cudaError_t run_pack(const float *keys, const fathom_index &ix, const PackGeom &g,
                     uint32_t *ws_min, uint32_t *ws_max, cudaStream_t stream)
{
    const int bits = index_bits(ix);
    int *status = device_status_ptr();
    const int count = g.H * g.n_touch * g.d;
    const int eb = 256, eg = (count + eb - 1) / eb;
    pack_init_kernel<<<eg, eb, 0, stream>>>(ws_min, ws_max, ix.sum_code, ix.sum_code2, g);
    dim3 g1((g.n_in + kMinMaxKeysPerBlock - 1) / kMinMaxKeysPerBlock, g.H);
    pack_minmax_kernel<<<g1, g.d, 0, stream>>>(keys, g, ws_min, ws_max, status);
    pack_range_kernel<<<eg, eb, 0, stream>>>(ws_min, ws_max, ix.mn, ix.scale, g, (1 << bits) - 1);
    const size_t smem = (size_t)g.d * bits * kQuantWordsPerBlock * sizeof(uint32_t);
    auto kern = bits == 8 ? pack_quant_kernel<8> : pack_quant_kernel<4>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 g2((g.words_out + kQuantWordsPerBlock - 1) / kQuantWordsPerBlock, g.H);
    kern<<<g2, kQuantThreads, smem, stream>>>(keys, g, ix.mn, ix.scale, ix.planes, ix.sum_code,
                                              ix.sum_code2);
    note_launch(4);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_channel_stats(ix, g.j_base + g.n_in, stream);
}

PackGeom geometry(const fathom_index &ix, int j_base, int n_in, int words_out)
{
    PackGeom g{};
    g.words_out = words_out;
    g.H = ix.n_kv_heads;
    g.d = ix.head_dim;
    g.n_in = n_in;
    g.j_base = j_base;
    g.n_words = ix.n_words;
    g.block_keys = ix.block_keys;
    g.nb = index_blocks(ix);
    g.b0 = ix.block_keys ? j_base / ix.block_keys : 0;
    g.n_touch = ix.block_keys ? (j_base + n_in - 1) / ix.block_keys - g.b0 + 1 : 1;
    return g;
}

}  // namespace

cudaError_t launch_pack(const float *keys, const fathom_index &ix, uint32_t *ws_minmax,
                        cudaStream_t stream)
{
    // every word of the planes: zero padding past the keys, for appends
    const PackGeom g = geometry(ix, 0, ix.n_keys, ix.n_words);
    if (ix.block_keys) {   // the min/max accumulators live in mn and scale themselves
        return run_pack(keys, ix, g, reinterpret_cast<uint32_t *>(ix.mn),
                        reinterpret_cast<uint32_t *>(ix.scale), stream);
    }
    const int count = ix.n_kv_heads * ix.head_dim;
    return run_pack(keys, ix, g, ws_minmax, ws_minmax + count, stream);
}

cudaError_t launch_append_blocks(const float *keys, const fathom_index &ix, int m,
                                 cudaStream_t stream)
{
    const PackGeom g = geometry(ix, ix.n_keys, m, (m + 31) / 32);
    return run_pack(keys, ix, g, reinterpret_cast<uint32_t *>(ix.mn),
                    reinterpret_cast<uint32_t *>(ix.scale), stream);
}

cudaError_t launch_channel_stats(const fathom_index &ix, int n, cudaStream_t stream)
{
    const int count = ix.n_kv_heads * ix.head_dim;
    const int eb = 256, eg = (count + eb - 1) / eb;
    if (ix.block_keys)
        pack_blocked_stats_kernel<<<eg, eb, 0, stream>>>(ix.mn, ix.scale, ix.sum_code,
                                                         ix.sum_code2, ix.sigma2, ix.n_kv_heads,
                                                         ix.head_dim, index_blocks(ix), n,
                                                         ix.block_keys);
    else
        pack_stats_kernel<<<eg, eb, 0, stream>>>(ix.sum_code, ix.sum_code2, ix.scale, ix.sigma2,
                                                 n, count);
    note_launch(1);
    return cudaGetLastError();
}

}  // namespace fathom
