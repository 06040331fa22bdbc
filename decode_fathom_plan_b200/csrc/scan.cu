// Read side of the Fathom scan: fetch the selected bit planes, score every
// key from them, and select the top-k.
//
// Source: Fathom explainer (papers.ananclaw.com, arXiv 2609.17652),
// section 核心方法: the first t planes of a channel are its t-bit quantiser,
// so a query that plans t_c bits for channel c reads planes 0..t_c-1 (most
// significant first) and scores the key rebuilt from that coarser
// quantiser; section 解决什么真问题: each decode step ranks the n keys and
// keeps the top-k.
//
// Score decomposition used on the GPU.  With v = code with the low 4-t bits
// cleared (the t most significant bits in place) and off(t) = (2^(4-t)-1)/2,
// the coarse-bin midpoint is mn + scale*(v + off(t)), so
//   s_gj = bias_g + sum_c W_gc * v_gcj,   W_gc = q_gc*scale_c,
//   bias_g = sum_c q_gc*(mn_c + scale_c*off(t_gc))   (fp64, rounded once).
// v is an integer 0..15, so the hot loop is "nibble -> float, then one fma
// per query head", with no per-bit work.
//
// Data path (one CTA = one KV head x one 2048-key tile):
//   * the union plan T_c = max_g t_gc of the KV head's G query heads decides
//     which plane rows are read; each row slice is 256 contiguous bytes
//     (64 words) and is copied into shared memory with 16-byte cp.async,
//     three stages of up to 8 channels (32 rows) in flight;
//   * thread (column, row r) owns keys 32*column + 4m + r, m = 0..7: a
//     funnel-shift rotate and a mask move bit 4m+r of each plane word to bit
//     4m+p, so one register holds the thread's 8 nibbles; each nibble
//     becomes a float by OR-ing it under the mantissa of a power of two and
//     subtracting that power (exact), two at a time with __fadd2_rn;
//   * each query head reading the channel adds W*v with __ffma2_rn (two keys
//     per instruction); a head reading fewer planes than the union masks
//     its nibbles first.
// No tensor cores: this is a sparse binary-weighted reduction.
//
// Selection without materialising n scores per query:
//   1. sample:   score a few evenly spaced tiles (about 3% of the keys) and
//                write their order keys to the workspace;
//   2. theta:    per query, theta = the r-th largest sampled key, with r
//                about 2*k*m/n, so ~2k keys are expected to pass;
//   3. filter:   the full scan appends (key, index) of every key scoring
//                >= theta to a per-query candidate buffer;
//   4. final:    if k <= candidates <= capacity, an exact radix select over
//                the unique composite (order key, ~index) and a bitonic sort
//                give the top-k; otherwise the query is flagged;
//   5. fallback: a flagged query is redone exactly by one CTA that
//                recomputes its scores once per radix digit (no score
//                buffer), so results never depend on the sample.
// Every key of the sampled pass is recomputed by the full scan with the same
// arithmetic, so a key's score is the same in both passes.
#include <math.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace fathom {
namespace {

struct SessionDesc {
    const uint32_t *planes;      // device address of [H][d][4][n_words]
    const float *mn;
    const float *scale;
    const uint16_t *q;           // [Q][d]
    const uint8_t *t;            // [Q][d]
    const uint8_t *tu;           // [H][d]
    int32_t *out_idx;            // [Q][k]
    float *out_score;            // [Q][k]
    uint32_t *qstate;            // [Q][4]: theta, count, fallback flag, spare
    uint32_t *sample;            // [Q][m_keys]
    unsigned long long *cand;    // [Q][cap]
    int H, n, n_words, n_cols, n_tiles;
    int m_tiles, sample_stride, m_keys, sample_rank, exact_only;
    int item_begin, sample_item_begin, q_begin;
};

template <int NS>
struct Batch {
    int n_sessions, G, d, k, cap, kpad;
    SessionDesc s[NS];
};

template <int GP>
struct alignas(16) ScanSmem {
    alignas(16) uint32_t stage[kStages][kStageRows][kTileCols];   // cp.async needs 16-byte rows
    uint32_t row_g[kBits * kMaxHeadDim];         // global plane row of each union row
    float W[kMaxHeadDim][GP];                    // q*scale per (union channel, query)
    uint8_t tq[kMaxHeadDim][GP];                 // planes read per (union channel, query)
    uint8_t uT[kMaxHeadDim];                     // union depth
    uint8_t uro[kMaxHeadDim];                    // first row of the channel inside its stage
    uint16_t stage_row0[kMaxHeadDim / kStageChannels + 1];
    float bias[GP];
    int U, P, n_stages;
    int part[2][kScanThreads / 32];
};

// ------------------------------------------------------------ small helpers
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, int src_bytes)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// 8 nibbles of a word -> 8 exact floats, paired (m, m+4).  A nibble at bit
// 4m is OR-ed under the mantissa of 2^(23-4m), whose unit in the last place
// there is 1, so the float is 2^(23-4m) + v; subtracting the power leaves v.
// Nibbles 5..7 are shifted down by 20 bits first (bits 20..31 would reach
// the exponent).
__device__ __forceinline__ void nibbles_to_floats(uint32_t nib, float2 (&v)[4])
{
    const uint32_t hi = nib >> 20;
    const float f0 = __uint_as_float((nib & 0x0000000Fu) | 0x4B000000u);   // 2^23
    const float f1 = __uint_as_float((nib & 0x000000F0u) | 0x49000000u);   // 2^19
    const float f2 = __uint_as_float((nib & 0x00000F00u) | 0x47000000u);   // 2^15
    const float f3 = __uint_as_float((nib & 0x0000F000u) | 0x45000000u);   // 2^11
    const float f4 = __uint_as_float((nib & 0x000F0000u) | 0x43000000u);   // 2^7
    const float f5 = __uint_as_float((hi & 0x0000000Fu) | 0x4B000000u);
    const float f6 = __uint_as_float((hi & 0x000000F0u) | 0x49000000u);
    const float f7 = __uint_as_float((hi & 0x00000F00u) | 0x47000000u);
    v[0] = __fadd2_rn(make_float2(f0, f4), make_float2(-8388608.0f, -128.0f));
    v[1] = __fadd2_rn(make_float2(f1, f5), make_float2(-524288.0f, -8388608.0f));
    v[2] = __fadd2_rn(make_float2(f2, f6), make_float2(-32768.0f, -524288.0f));
    v[3] = __fadd2_rn(make_float2(f3, f7), make_float2(-2048.0f, -32768.0f));
}

// Offset of the coarse-bin middle: (2^(4-t) - 1) / 2.
__device__ __forceinline__ double bin_offset(int t)
{
    return (double)((1 << (kBits - t)) - 1) * 0.5;
}

// ------------------------------------------------------- per-head set-up
// Builds the union channel list, plane-row table, weights and biases for
// query heads q_rows[0..G) of KV head h.  tu_row: the union plan to read;
// t_rows: each query's own plan.  256 threads, d <= 256.
template <int GP>
__device__ void setup_head(ScanSmem<GP> &sm, int h, int G, int d, const uint8_t *tu_row,
                           const uint8_t *t_rows, const uint16_t *q_rows, const float *mn_h,
                           const float *sc_h)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int T = (tid < d) ? min((int)tu_row[tid], kBits) : 0;
    const int has = T > 0;
    int inc_u = has, inc_p = T;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int a = __shfl_up_sync(0xFFFFFFFFu, inc_u, off);
        const int b = __shfl_up_sync(0xFFFFFFFFu, inc_p, off);
        if (lane >= off) { inc_u += a; inc_p += b; }
    }
    if (lane == 31) { sm.part[0][warp] = inc_u; sm.part[1][warp] = inc_p; }
    __syncthreads();
    int base_u = 0, base_p = 0, U = 0, P = 0;
#pragma unroll
    for (int w = 0; w < kScanThreads / 32; ++w) {
        if (w < warp) { base_u += sm.part[0][w]; base_p += sm.part[1][w]; }
        U += sm.part[0][w];
        P += sm.part[1][w];
    }
    const int u = base_u + inc_u - has;
    const int prow = base_p + inc_p - T;
    if (has) {
        const int c = tid;
        sm.uT[u] = (uint8_t)T;
        if ((u % kStageChannels) == 0) sm.stage_row0[u / kStageChannels] = (uint16_t)prow;
        for (int s = 0; s < T; ++s) sm.row_g[prow + s] = (uint32_t)((h * d + c) * kBits + s);
        const float sc = sc_h[c];
#pragma unroll
        for (int g = 0; g < GP; ++g) {
            if (g < G) {
                sm.W[u][g] = __fmul_rn(bf16_to_float(q_rows[g * d + c]), sc);
                sm.tq[u][g] = (uint8_t)min((int)t_rows[g * d + c], T);
            } else {
                sm.W[u][g] = 0.0f;
                sm.tq[u][g] = 0;
            }
        }
    }
    if (tid == 0) {
        sm.U = U;
        sm.P = P;
        sm.n_stages = (U + kStageChannels - 1) / kStageChannels;
        sm.stage_row0[(U + kStageChannels - 1) / kStageChannels] = (uint16_t)P;
    }
    // bias_g over every channel, each at its own (clamped) depth
    if (warp < GP) {
        double acc = 0.0;
        if (warp < G) {
            for (int c = lane; c < d; c += 32) {
                const int tg = min((int)t_rows[warp * d + c], min((int)tu_row[c], kBits));
                const double qf = (double)bf16_to_float(q_rows[warp * d + c]);
                acc += qf * ((double)mn_h[c] + (double)sc_h[c] * bin_offset(tg));
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
        if (lane == 0) sm.bias[warp] = (float)acc;
    }
    __syncthreads();
    if (has) sm.uro[u] = (uint8_t)(prow - sm.stage_row0[u / kStageChannels]);
    __syncthreads();
}

// ------------------------------------------------------------- tile scan
template <int GP>
__device__ __forceinline__ void load_stage(ScanSmem<GP> &sm, int st, int buf,
                                           const uint32_t *planes, int n_words, int n_cols,
                                           int col0)
{
    const int r0 = sm.stage_row0[st];
    const int R = sm.stage_row0[st + 1] - r0;
    const int chunk = threadIdx.x & 15;
    const int col = col0 + chunk * 4;
    const bool ok = col < n_cols;
    for (int row = threadIdx.x >> 4; row < R; row += kScanThreads / 16) {
        const uint32_t *src = planes + (size_t)sm.row_g[r0 + row] * (size_t)n_words + (ok ? col : 0);
        cp_async16(&sm.stage[buf][row][chunk * 4], src, ok ? 16 : 0);
    }
}

template <int GP>
__device__ __forceinline__ void compute_stage(const ScanSmem<GP> &sm, int st, int buf, int col,
                                              int r, float2 (&acc)[GP][4])
{
    const int u0 = st * kStageChannels;
    const int u1 = min(u0 + kStageChannels, sm.U);
    for (int u = u0; u < u1; ++u) {
        const int T = sm.uT[u];
        const int ro = sm.uro[u];
        uint32_t nib = 0;
#pragma unroll
        for (int s = 0; s < kBits; ++s) {
            if (s < T) {
                const uint32_t x = sm.stage[buf][ro + s][col];
                const int p = kBits - 1 - s;   // slot s holds bit 3-s
                nib |= __funnelshift_r(x, x, (r - p) & 31) & (0x11111111u << p);
            }
        }
        float2 v[4];
        nibbles_to_floats(nib, v);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
            const int tg = sm.tq[u][g];
            if (tg == 0) continue;
            const float w = sm.W[u][g];
            const float2 w2 = make_float2(w, w);
            if (tg == T) {
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[g][i] = __ffma2_rn(v[i], w2, acc[g][i]);
            } else {
                const uint32_t keep = ((0xFu << (kBits - tg)) & 0xFu) * 0x11111111u;
                float2 vm[4];
                nibbles_to_floats(nib & keep, vm);
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[g][i] = __ffma2_rn(vm[i], w2, acc[g][i]);
            }
        }
    }
}

// Scores of the thread's 8 keys of tile `tile` for every query head:
// score(g, m) = bias_g + acc[g][m % 4].{x if m < 4 else y}.
template <int GP>
__device__ void scan_tile(ScanSmem<GP> &sm, const uint32_t *planes, int n_words, int n_cols,
                          int tile, float2 (&acc)[GP][4])
{
    const int col = threadIdx.x >> 2, r = threadIdx.x & 3;
    const int col0 = tile * kTileCols;
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[g][i] = make_float2(0.0f, 0.0f);
    const int n_stages = sm.n_stages;
    __syncthreads();   // stage buffers may still be read by a previous tile
#pragma unroll
    for (int st = 0; st < kStages - 1; ++st) {
        if (st < n_stages) load_stage(sm, st, st, planes, n_words, n_cols, col0);
        cp_async_commit();
    }
    for (int st = 0; st < n_stages; ++st) {
        cp_async_wait<kStages - 2>();
        __syncthreads();
        const int nx = st + kStages - 1;
        if (nx < n_stages) load_stage(sm, nx, nx % kStages, planes, n_words, n_cols, col0);
        cp_async_commit();
        compute_stage(sm, st, st % kStages, col, r, acc);
    }
    cp_async_wait<0>();
}

__device__ __forceinline__ float score_of(const float2 (&a)[4], int m, float bias)
{
    const float2 p = a[m & 3];
    return bias + ((m < 4) ? p.x : p.y);
}

template <int NS>
__device__ __forceinline__ int find_session_by_item(const Batch<NS> &b, int item, bool sample)
{
    int si = 0;
    for (int s = 1; s < b.n_sessions; ++s)
        if ((sample ? b.s[s].sample_item_begin : b.s[s].item_begin) <= item) si = s;
    return si;
}

template <int NS>
__device__ __forceinline__ int find_session_by_query(const Batch<NS> &b, int gq)
{
    int si = 0;
    for (int s = 1; s < b.n_sessions; ++s)
        if (b.s[s].q_begin <= gq) si = s;
    return si;
}

// ------------------------------------------------- sampled / filtered scan
// kSample: grid over (session, head, sample tile); writes order keys of the
// sampled keys.  Otherwise grid over (session, head, tile); appends keys
// scoring >= theta to the candidate buffer.
template <int NS, int GP, bool kSample>
__global__ void __launch_bounds__(kScanThreads, (GP >= 8) ? 2 : 3)
scan_kernel(const __grid_constant__ Batch<NS> b)
{
    __shared__ ScanSmem<GP> sm;
    const int item = blockIdx.x;
    const int si = find_session_by_item(b, item, kSample);
    const SessionDesc &S = b.s[si];
    const int local = item - (kSample ? S.sample_item_begin : S.item_begin);
    const int per_head = kSample ? S.m_tiles : S.n_tiles;
    const int h = local / per_head;
    const int ti = local - h * per_head;
    const int tile = kSample ? ti * S.sample_stride : ti;
    const int G = b.G, d = b.d;
    const int q0 = h * G;

    setup_head<GP>(sm, h, G, d, S.tu + h * d, S.t + (size_t)q0 * d, S.q + (size_t)q0 * d,
                   S.mn + h * d, S.scale + h * d);
    float2 acc[GP][4];
    scan_tile<GP>(sm, S.planes, S.n_words, S.n_cols, tile, acc);

    const int col = threadIdx.x >> 2, r = threadIdx.x & 3, lane = threadIdx.x & 31;
    const int key0 = (tile * kTileCols + col) * 32 + r;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
        if (g >= G) break;
        const int qq = q0 + g;
        const float bias = sm.bias[g];
        if (kSample) {
            uint32_t *dst = S.sample + (size_t)qq * S.m_keys + (size_t)ti * kTileKeys + col * 32 + r;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int j = key0 + 4 * m;
                dst[4 * m] = (j < S.n) ? order_key(score_of(acc[g], m, bias)) : 0u;
            }
        } else {
            const uint32_t theta = S.qstate[qq * kQueryStateWords + 0];
            uint32_t ok[8];
            unsigned pass = 0;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int j = key0 + 4 * m;
                ok[m] = order_key(score_of(acc[g], m, bias));
                if (j < S.n && ok[m] >= theta) pass |= 1u << m;
            }
            const int cnt = __popc(pass);
            int inc = cnt;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, inc, off);
                if (lane >= off) inc += y;
            }
            const int total = __shfl_sync(0xFFFFFFFFu, inc, 31);
            if (total == 0) continue;
            unsigned base = 0;
            if (lane == 31) base = atomicAdd(&S.qstate[qq * kQueryStateWords + 1], (unsigned)total);
            base = __shfl_sync(0xFFFFFFFFu, base, 31);
            unsigned pos = base + (unsigned)(inc - cnt);
            unsigned long long *cq = S.cand + (size_t)qq * b.cap;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                if (pass & (1u << m)) {
                    if (pos < (unsigned)b.cap) cq[pos] = composite(ok[m], (uint32_t)(key0 + 4 * m));
                    ++pos;
                }
            }
        }
    }
}

// ------------------------------------------------------- radix selection
// Warp 0 finds, in a 256-bin histogram, the bin holding the krem-th largest
// element: above = elements in higher bins < krem <= above + hist[bin].
__device__ __forceinline__ void pick_bin(const unsigned *hist, unsigned krem, int *out_bin,
                                         unsigned *out_above)
{
    const int lane = threadIdx.x & 31;
    // lane l owns bins 255-8l .. 248-8l (descending)
    unsigned h8[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        h8[i] = hist[255 - 8 * lane - i];
        local += h8[i];
    }
    unsigned inc = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned y = __shfl_up_sync(0xFFFFFFFFu, inc, off);
        if (lane >= off) inc += y;
    }
    const unsigned before = inc - local;
    if (before < krem && krem <= inc) {
        unsigned run = before;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (run < krem && krem <= run + h8[i]) {
                *out_bin = 255 - 8 * lane - i;
                *out_above = run;
            }
            run += h8[i];
        }
    }
}

struct SelectState {
    unsigned hist[256];
    unsigned long long prefix, pmask;
    unsigned krem;
    int bin, shift, done;
    unsigned above;
    unsigned nsel;
};

// One radix pass over a stream of composites (values already folded into
// hist by the caller); updates prefix/krem and decides whether the selected
// set is already determined.  Called by all threads after hist is complete.
__device__ __forceinline__ void select_step(SelectState &ss, int digit)
{
    if (threadIdx.x < 32) pick_bin(ss.hist, ss.krem, &ss.bin, &ss.above);
    __syncthreads();
    if (threadIdx.x == 0) {
        const int b = ss.bin & 0xFF;
        ss.krem -= ss.above;
        ss.prefix |= (unsigned long long)b << (8 * digit);
        ss.pmask |= 0xFFull << (8 * digit);
        if (ss.hist[b] == ss.krem) {
            ss.done = 1;
            ss.shift = 8 * digit;
        }
    }
    __syncthreads();
}

__device__ __forceinline__ void select_reset(SelectState &ss, unsigned k)
{
    if (threadIdx.x == 0) {
        ss.prefix = 0;
        ss.pmask = 0;
        ss.krem = k;
        ss.done = 0;
        ss.shift = 0;
        ss.nsel = 0;
        ss.bin = 0;
        ss.above = 0;
    }
}

// Sort kpad composites in shared memory, descending (bitonic network).
__device__ void bitonic_sort_desc(unsigned long long *x, int kpad)
{
    for (int size = 2; size <= kpad; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < (kpad >> 1); i += blockDim.x) {
                const int lo = 2 * stride * (i / stride) + (i % stride);
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const unsigned long long a = x[lo], c = x[hi];
                if ((a < c) == desc) {
                    x[lo] = c;
                    x[hi] = a;
                }
            }
            __syncthreads();
        }
    }
}

__device__ void write_outputs(const unsigned long long *sel, int k, int32_t *out_idx,
                              float *out_score)
{
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        const unsigned long long x = sel[i];
        out_idx[i] = (int32_t)(~(uint32_t)(x & 0xFFFFFFFFull));
        out_score[i] = order_key_to_float((uint32_t)(x >> 32));
    }
}

// ---------------------------------------------------------------- theta
// One CTA per query: theta = the sample_rank-th largest sampled order key
// (4 radix passes over the sample held in shared memory), and reset the
// candidate count and fallback flag.
template <int NS>
__global__ void __launch_bounds__(1024) theta_kernel(const __grid_constant__ Batch<NS> b,
                                                     uint32_t force_exact)
{
    extern __shared__ uint32_t vals[];
    __shared__ SelectState ss;
    const int gq = blockIdx.x;
    const int si = find_session_by_query(b, gq);
    const SessionDesc &S = b.s[si];
    const int qq = gq - S.q_begin;
    uint32_t *st = S.qstate + qq * kQueryStateWords;
    if (force_exact || S.exact_only) {
        if (threadIdx.x == 0) { st[0] = 0xFFFFFFFFu; st[1] = 0; st[2] = 1; }
        return;
    }
    if (S.m_tiles == 0) {   // few keys: every key is a candidate
        if (threadIdx.x == 0) { st[0] = 0; st[1] = 0; st[2] = 0; }
        return;
    }
    const int m = S.m_keys;
    const uint32_t *src = S.sample + (size_t)qq * m;
    for (int i = threadIdx.x; i < m; i += blockDim.x) vals[i] = src[i];
    select_reset(ss, (unsigned)S.sample_rank);
    __syncthreads();
    for (int digit = 3; digit >= 0; --digit) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) ss.hist[i] = 0;
        __syncthreads();
        const uint32_t pm = (uint32_t)ss.pmask, pf = (uint32_t)ss.prefix;
        for (int i = threadIdx.x; i < m; i += blockDim.x) {
            const uint32_t v = vals[i];
            if ((v & pm) == pf) atomicAdd(&ss.hist[(v >> (8 * digit)) & 0xFFu], 1u);
        }
        __syncthreads();
        select_step(ss, digit);
    }
    if (threadIdx.x == 0) { st[0] = (uint32_t)ss.prefix; st[1] = 0; st[2] = 0; }
}

// ---------------------------------------------------------------- final
// One CTA per query: exact top-k of the candidates when k <= count <= cap.
template <int NS>
__global__ void __launch_bounds__(1024) final_kernel(const __grid_constant__ Batch<NS> b)
{
    extern __shared__ unsigned long long dyn[];
    __shared__ SelectState ss;
    const int gq = blockIdx.x;
    const int si = find_session_by_query(b, gq);
    const SessionDesc &S = b.s[si];
    const int qq = gq - S.q_begin;
    uint32_t *st = S.qstate + qq * kQueryStateWords;
    if (st[2]) return;
    const unsigned cnt = st[1];
    const int k = b.k;
    if (cnt < (unsigned)k || cnt > (unsigned)b.cap) {
        __syncthreads();
        if (threadIdx.x == 0) st[2] = 1;
        return;
    }
    unsigned long long *x = dyn;              // [cap]
    unsigned long long *sel = dyn + b.cap;    // [kpad]
    const unsigned long long *cq = S.cand + (size_t)qq * b.cap;
    for (unsigned i = threadIdx.x; i < cnt; i += blockDim.x) x[i] = cq[i];
    select_reset(ss, (unsigned)k);
    __syncthreads();
    for (int digit = 7; digit >= 0; --digit) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) ss.hist[i] = 0;
        __syncthreads();
        const unsigned long long pm = ss.pmask, pf = ss.prefix;
        for (unsigned i = threadIdx.x; i < cnt; i += blockDim.x) {
            const unsigned long long v = x[i];
            if ((v & pm) == pf) atomicAdd(&ss.hist[(unsigned)(v >> (8 * digit)) & 0xFFu], 1u);
        }
        __syncthreads();
        select_step(ss, digit);
        if (ss.done) break;
    }
    const int shift = ss.shift;
    const unsigned long long lim = ss.prefix >> shift;
    for (unsigned i = threadIdx.x; i < cnt; i += blockDim.x) {
        const unsigned long long v = x[i];
        if ((v >> shift) >= lim) {
            const unsigned slot = atomicAdd(&ss.nsel, 1u);
            if (slot < (unsigned)k) sel[slot] = v;
        }
    }
    for (int i = k + threadIdx.x; i < b.kpad; i += blockDim.x) sel[i] = 0ull;
    __syncthreads();
    bitonic_sort_desc(sel, b.kpad);
    write_outputs(sel, k, S.out_idx + (size_t)qq * k, S.out_score + (size_t)qq * k);
}

// ------------------------------------------------------------- fallback
// One CTA per flagged query: exact top-k by radix select over the composite
// (order key, ~index), recomputing the query's scores from its own plan on
// every pass.  Slow, rare, and independent of the sample.
template <int NS>
__global__ void __launch_bounds__(kScanThreads) fallback_kernel(const __grid_constant__ Batch<NS> b)
{
    __shared__ ScanSmem<1> sm;
    __shared__ SelectState ss;
    extern __shared__ unsigned long long sel[];   // [kpad]
    const int gq = blockIdx.x;
    const int si = find_session_by_query(b, gq);
    const SessionDesc &S = b.s[si];
    const int qq = gq - S.q_begin;
    if (!S.qstate[qq * kQueryStateWords + 2]) return;
    const int d = b.d, k = b.k;
    const int h = qq / b.G;
    const uint8_t *trow = S.t + (size_t)qq * d;
    setup_head<1>(sm, h, 1, d, trow, trow, S.q + (size_t)qq * d, S.mn + h * d, S.scale + h * d);
    select_reset(ss, (unsigned)k);
    const int col = threadIdx.x >> 2, r = threadIdx.x & 3;
    const float bias = sm.bias[0];
    float2 acc[1][4];
    for (int digit = 7; digit >= 0; --digit) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) ss.hist[i] = 0;
        __syncthreads();
        const unsigned long long pm = ss.pmask, pf = ss.prefix;
        for (int tile = 0; tile < S.n_tiles; ++tile) {
            scan_tile<1>(sm, S.planes, S.n_words, S.n_cols, tile, acc);
            const int key0 = (tile * kTileCols + col) * 32 + r;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int j = key0 + 4 * m;
                if (j < S.n) {
                    const unsigned long long v =
                        composite(order_key(score_of(acc[0], m, bias)), (uint32_t)j);
                    if ((v & pm) == pf) atomicAdd(&ss.hist[(unsigned)(v >> (8 * digit)) & 0xFFu], 1u);
                }
            }
        }
        __syncthreads();
        select_step(ss, digit);
        if (ss.done) break;
    }
    const int shift = ss.shift;
    const unsigned long long lim = ss.prefix >> shift;
    for (int tile = 0; tile < S.n_tiles; ++tile) {
        scan_tile<1>(sm, S.planes, S.n_words, S.n_cols, tile, acc);
        const int key0 = (tile * kTileCols + col) * 32 + r;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int j = key0 + 4 * m;
            if (j < S.n) {
                const unsigned long long v = composite(order_key(score_of(acc[0], m, bias)), (uint32_t)j);
                if ((v >> shift) >= lim) {
                    const unsigned slot = atomicAdd(&ss.nsel, 1u);
                    if (slot < (unsigned)k) sel[slot] = v;
                }
            }
        }
    }
    for (int i = k + threadIdx.x; i < b.kpad; i += blockDim.x) sel[i] = 0ull;
    __syncthreads();
    bitonic_sort_desc(sel, b.kpad);
    write_outputs(sel, k, S.out_idx + (size_t)qq * k, S.out_score + (size_t)qq * k);
}

// ------------------------------------------------------------- host side
inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
inline int next_pow2(int x)
{
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

inline int capacity_for(int k) { return std::max(6 * k, 8192); }

struct Sizing {
    int n_cols, n_tiles, m_tiles, stride, m_keys, rank, exact_only;
};

// Sample sizing: m sampled keys (whole tiles, evenly strided) with
// m ~ 128*n/(2k) clamped to [4096, 32768] and to a quarter of the tiles;
// theta is the r-th largest sampled key, r = ceil(f*k*m/n) with f = 2 (or 3
// when f = 2 would give r < 128), so about f*k keys pass the filter.
Sizing size_session(int n, int n_words, int k)
{
    Sizing z{};
    z.n_cols = std::min(n_words, ceil_div(ceil_div(n, 32), 4) * 4);
    z.n_tiles = ceil_div(z.n_cols, kTileCols);
    const int cap = capacity_for(std::min(k, kMaxFastK));
    z.exact_only = (k > kMaxFastK) ? 1 : 0;
    if (z.exact_only || n <= cap) return z;
    const double target = (double)kSampleTargetRank * (double)n / (2.0 * (double)k);
    int m = (int)std::min<double>(std::max<double>(target, kSampleMinKeys), kSampleMaxKeys);
    int mt = ceil_div(m, kTileKeys);
    mt = std::min(mt, std::max(1, z.n_tiles / 4));
    z.m_tiles = mt;
    z.stride = z.n_tiles / mt;
    z.m_keys = mt * kTileKeys;
    const double r2 = 2.0 * (double)k * (double)z.m_keys / (double)n;
    const double f = (r2 >= kSampleTargetRank) ? 2.0 : 3.0;
    z.rank = (int)std::ceil(f * (double)k * (double)z.m_keys / (double)n);
    z.rank = std::max(1, std::min(z.rank, z.m_keys));
    return z;
}

struct WsLayout {
    size_t qstate, sample, cand, total;
};

WsLayout layout_session(const fathom_index &ix, int k, size_t at)
{
    const int Q = ix.n_kv_heads * ix.group;
    const Sizing z = size_session(ix.n_keys, ix.n_words, k);
    const int cap = capacity_for(std::min(k, kMaxFastK));
    WsLayout L{};
    L.qstate = at;
    at += align256((size_t)Q * kQueryStateWords * sizeof(uint32_t));
    L.sample = at;
    at += align256((size_t)Q * z.m_keys * sizeof(uint32_t));
    L.cand = at;
    at += align256((size_t)Q * cap * sizeof(unsigned long long));
    L.total = at;
    return L;
}

template <int NS, int GP>
cudaError_t run_batch(const Batch<NS> &bt, int total_items, int total_sample_items,
                      int total_queries, int max_m_keys, uint32_t flags, cudaStream_t stream,
                      ScanProfileHook *hook)
{
    cudaError_t e;
    const bool force = (flags & FATHOM_SCAN_FORCE_EXACT) != 0;
    int launches = 0;
    if (!force && total_sample_items > 0) {
        scan_kernel<NS, GP, true><<<total_sample_items, kScanThreads, 0, stream>>>(bt);
        ++launches;
    }
    const size_t theta_smem = (size_t)max_m_keys * sizeof(uint32_t);
    e = cudaFuncSetAttribute(theta_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)std::max<size_t>(theta_smem, 1));
    if (e != cudaSuccess) return e;
    theta_kernel<NS><<<total_queries, 1024, theta_smem, stream>>>(bt, force ? 1u : 0u);
    ++launches;
    if (!force && total_items > 0) {
        if (hook && hook->enabled) cudaEventRecord(hook->begin, stream);
        scan_kernel<NS, GP, false><<<total_items, kScanThreads, 0, stream>>>(bt);
        if (hook && hook->enabled) {
            cudaEventRecord(hook->end, stream);
            hook->recorded = true;
        }
        ++launches;
    }
    const size_t final_smem = ((size_t)bt.cap + bt.kpad) * sizeof(unsigned long long);
    e = cudaFuncSetAttribute(final_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)final_smem);
    if (e != cudaSuccess) return e;
    final_kernel<NS><<<total_queries, 1024, final_smem, stream>>>(bt);
    const size_t fb_smem = (size_t)bt.kpad * sizeof(unsigned long long);
    e = cudaFuncSetAttribute(fallback_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)fb_smem);
    if (e != cudaSuccess) return e;
    fallback_kernel<NS><<<total_queries, kScanThreads, fb_smem, stream>>>(bt);
    launches += 2;
    note_launch(launches);
    return cudaGetLastError();
}

template <int NS>
cudaError_t build_and_run(const ScanSessionArgs *ss, int n_sessions, int k, void *ws,
                          uint32_t flags, cudaStream_t stream, ScanProfileHook *hook)
{
    static_assert(sizeof(Batch<NS>) < 32000, "kernel parameter block too large");
    Batch<NS> bt{};
    const fathom_index &ix0 = *ss[0].ix;
    bt.n_sessions = n_sessions;
    bt.G = ix0.group;
    bt.d = ix0.head_dim;
    bt.k = k;
    bt.cap = capacity_for(std::min(k, kMaxFastK));
    bt.kpad = next_pow2(k);
    int items = 0, sitems = 0, queries = 0, max_m = 0;
    size_t at = 0;
    char *base = static_cast<char *>(ws);
    for (int s = 0; s < n_sessions; ++s) {
        const fathom_index &ix = *ss[s].ix;
        const Sizing z = size_session(ix.n_keys, ix.n_words, k);
        const WsLayout L = layout_session(ix, k, at);
        at = L.total;
        SessionDesc &D = bt.s[s];
        D.planes = ix.planes;
        D.mn = ix.mn;
        D.scale = ix.scale;
        D.q = ss[s].q;
        D.t = ss[s].t;
        D.tu = ss[s].t_union;
        D.out_idx = ss[s].out_idx;
        D.out_score = ss[s].out_score;
        D.qstate = reinterpret_cast<uint32_t *>(base + L.qstate);
        D.sample = reinterpret_cast<uint32_t *>(base + L.sample);
        D.cand = reinterpret_cast<unsigned long long *>(base + L.cand);
        D.H = ix.n_kv_heads;
        D.n = ix.n_keys;
        D.n_words = ix.n_words;
        D.n_cols = z.n_cols;
        D.n_tiles = z.n_tiles;
        D.m_tiles = z.m_tiles;
        D.sample_stride = z.stride;
        D.m_keys = z.m_keys;
        D.sample_rank = z.rank;
        D.exact_only = z.exact_only;
        D.item_begin = items;
        D.sample_item_begin = sitems;
        D.q_begin = queries;
        items += D.H * D.n_tiles;
        sitems += D.H * D.m_tiles;
        queries += D.H * bt.G;
        max_m = std::max(max_m, z.m_keys);
    }
    const int G = bt.G;
    if (G <= 1) return run_batch<NS, 1>(bt, items, sitems, queries, max_m, flags, stream, hook);
    if (G <= 2) return run_batch<NS, 2>(bt, items, sitems, queries, max_m, flags, stream, hook);
    if (G <= 4) return run_batch<NS, 4>(bt, items, sitems, queries, max_m, flags, stream, hook);
    return run_batch<NS, 8>(bt, items, sitems, queries, max_m, flags, stream, hook);
}

}  // namespace

size_t scan_workspace_bytes(const fathom_index *sessions, int n_sessions, int k)
{
    size_t at = 0;
    for (int s = 0; s < n_sessions; ++s) at = layout_session(sessions[s], k, at).total;
    return at;
}

cudaError_t launch_scan(const ScanSessionArgs *sessions, int n_sessions, int k, void *ws,
                        size_t ws_bytes, uint32_t flags, cudaStream_t stream,
                        ScanProfileHook *hook)
{
    (void)ws_bytes;
    if (n_sessions == 1) return build_and_run<1>(sessions, 1, k, ws, flags, stream, hook);
    return build_and_run<kMaxSessions>(sessions, n_sessions, k, ws, flags, stream, hook);
}

}  // namespace fathom
