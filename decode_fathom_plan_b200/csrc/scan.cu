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
// Data path.  A KV head reads the union plan T_c = max_g t_gc of its G query
// heads once.  The threshold kernel builds each KV head's tables once (union
// channel list, plane rows, weights, biases); every scanning CTA copies them.  Union
// channels are listed by the set of query heads reading them at full depth,
// and an 8-channel stage runs a body specialised to its set, so a query head
// that does not read a channel issues no fma for it.  A stage is 8 union
// channels x 4 plane rows x a chunk of up to 64 plane words (2048 keys);
// rows past a channel's depth are zero-filled in shared memory with no
// global read.  Stages are copied with 16-byte cp.async, 3 buffers deep.
// Thread (column, row r) owns keys 32*column + 4m + r, m = 0..7: a
// funnel-shift rotate and a mask move bit 4m+r of each plane word to bit
// 4m+p, so one register holds the thread's 8 nibbles; each nibble becomes a
// float by OR-ing it under the mantissa of a power of two and subtracting
// that power (exact), two at a time with __fadd2_rn; each reading query head
// adds W*v with __ffma2_rn (two keys per instruction).  One CTA per 64-word
// chunk of a KV head; host-resident planes are fetched a unit of KV heads at
// a time into a two-slot device ring (fetch.cu) and read from there.
//
// No tensor cores: this is a sparse binary-weighted reduction.
//
// Selection without materialising n scores per query:
//   1. threshold: per query, score evenly strided whole tiles (4096 to 8192
//                 keys) from the query's own plan, and take theta = the r-th
//                 largest sampled key, r about 2*k*m/n (3*k*m/n for large n),
//                 so ~2k (3k) keys are expected to pass;
//   2. filter:    the full scan appends (key, index) of every key scoring
//                 >= theta to a per-query candidate buffer;
//   3. final:     if k <= candidates <= capacity, an exact radix select over
//                 the unique composite (order key, ~index) gives the top-k,
//                 listed in ascending key index; otherwise the same CTA
//                 redoes the query exactly, recomputing its scores once per
//                 radix digit (no score buffer), so results never depend on
//                 the sample.
// Correctness needs only that every key scoring at least the k-th largest
// score is a candidate, which "count >= k" guarantees for any theta.
#include <math.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace fathom {
namespace {

constexpr int kTileGroups = kTileCols / 4;   // 16-byte column groups per 64-word chunk
constexpr int kMainStages = 3;
constexpr int kMaskOrderValues = 16;   // reader sets of up to 4 query heads
constexpr int kMinChunkGroups = 8;     // smallest chunk of the main scan: 32 words
// Sampled tiles of a session with grouped per-token-block scales (Qwen3-8B
// layer, 128K keys in 2048-key blocks: 2 tiles sent some queries to the
// exact path, 4 kept all on the fast path, 8 and 16 cost more threshold
// passes than the exact paths they saved).
constexpr int kBlockedSampleTiles = 4;

struct SessionDesc {
    const uint32_t *planes;      // device address of [H][d][4][n_words]
    const float *mn;
    const float *scale;
    const uint16_t *q;           // [Q][d]
    const uint8_t *t;            // [Q][d]
    const uint8_t *tu;           // [H][d]
    int32_t *out_idx;            // [Q][k]
    float *out_score;            // [Q][k]
    uint32_t *qstate;            // [Q][4]: theta, count, exact-path flag, spare
    unsigned long long *cand;    // [Q][cap]
    unsigned char *tables;       // [H] per-head scan tables (ScanMeta of the batch's GP)
    float *bias_blk;             // grouped scales: [H][nb][G] bias per (head, block, query)
    int block_words;             // grouped scales: plane words per scale block (0: none)
    int nb, n_filled;            // statistics rows per head; blocks holding keys
    int blk_begin;               // first of this session's (KV head, block) bias CTAs
    int H, n, n_words, n_cols, col_groups;
    int m_tiles, sample_stride, m_keys, sample_rank, exact_only;
    int chunks, chunk_begin;   // main-scan chunks per KV head, first chunk's CTA
    int chunk_q, chunk_rem;    // col_groups = chunks * chunk_q + chunk_rem (one scale per channel)
    int q_begin, head_begin;
};

template <int NS>
struct Batch {
    int n_sessions, G, d, k, cap, kpad;
    SessionDesc s[NS];
};

// Per-head tables of a scanning CTA (the stage buffers live in dynamic
// shared memory).
template <int GP>
struct alignas(16) ScanMeta {
    alignas(16) float2 W2[kMaxHeadDim][GP];   // (w, w), w = q*scale if the query reads all T
                                              // planes of the union channel, else (0, 0)
    float Wp[kMaxHeadDim][GP];                // w = q*scale (partial-depth readers)
    uint32_t row_g[kBits * kMaxHeadDim];      // plane row of (union channel, slot); ~0u = zero fill
    uint32_t meta[kMaxHeadDim];               // bits 0-7: queries reading all T planes;
                                              // bits 16-23: queries reading 0 < t < T planes
    uint8_t tq[kMaxHeadDim][GP];              // planes read per (union channel, query)
    uint8_t stage_partial[kMaxHeadDim / kStageChannels];   // a query reads 0 < t < T in the stage
    unsigned stage_mask[kMaxHeadDim / kStageChannels];     // queries reading a stage's channel at
                                                           // full union depth (OR over the stage)
    float bias[GP];
    int U, n_stages;
    int part[kScanThreads / 32];
    int order[kScanThreads / 32][kMaskOrderValues];       // channel-order offsets per (warp, mask)
};

typedef uint32_t (*StageBuf)[kStageRows][kTileCols];

// Query groups of up to 4 heads list a KV head's union channels by the set
// of queries that read them at full union depth (then by channel), so that
// a stage of 8 channels is mostly read by one set and its FMAs can be
// specialised to that set.  Larger groups keep channel order.
template <int GP>
constexpr bool mask_ordered() { return GP <= 4; }

// Position of each reader set in the channel order, 4 bits per set: the
// sets run 0, 1, 3, 2, 6, 4, 12, 8, 9, 11, 10, 14, 15, 13, 5, 7, so that
// neighbouring sets share readers and an 8-channel stage that straddles two
// of them adds few query heads to its fma set (on the synthetic Qwen3-8B
// plans: 14 % fewer fma bodies than numeric order).
constexpr unsigned long long kReaderSetRank = 0xcbd69a87f4e52310ull;
__device__ __forceinline__ unsigned reader_set_rank(unsigned set)
{
    return (unsigned)(kReaderSetRank >> (4 * set)) & 0xFu;
}

// ------------------------------------------------------------ small helpers
// Plain 16-byte copy (no source-size operand).
__device__ __forceinline__ void cp_async16_full(void *smem, const void *gmem)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
// 16 bytes of plane data, or zeros where there is none (a row past the
// channel's depth, or a column past the chunk): a plain copy for live data,
// a shared-memory store of zeros otherwise, so no global request is issued
// for zero rows.  The zeros are visible after the stage's barrier.
__device__ __forceinline__ void copy_or_zero16(void *smem, const void *gmem, bool live)
{
    if (live)
        cp_async16_full(smem, gmem);
    else
        *reinterpret_cast<uint4 *>(smem) = make_uint4(0u, 0u, 0u, 0u);
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

// (a & b) | c in one logic op.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// 8 nibbles of a word -> 8 exact floats, paired (m, m+4).  A nibble at bit
// 4m is OR-ed under the mantissa of 2^(23-4m), whose unit in the last place
// there is 1, so the float is 2^(23-4m) + v; subtracting the power leaves v.
// Nibble m+4 sits at bit 4m of nib >> 16, so both halves of pair m use the
// same mask and power: one fused and/or per key and one paired add
// (add.rn.f32x2) per two keys.  neg[m] = -2^(23-4m).
__device__ __forceinline__ void nibbles_to_floats(uint32_t nib, const float (&neg)[4],
                                                  float2 (&v)[4])
{
    const uint32_t hi = nib >> 16;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const uint32_t mask = 0xFu << (4 * m);
        const uint32_t magic = (150u - 4u * (uint32_t)m) << 23;   // 2^(23-4m)
        const float a = __uint_as_float(and_or(nib, mask, magic));
        const float b = __uint_as_float(and_or(hi, mask, magic));
        v[m] = __fadd2_rn(make_float2(a, b), make_float2(neg[m], neg[m]));
    }
}

// -2^(23-4m), m = 0..3.
__device__ __forceinline__ void magic_negatives(float (&neg)[4])
{
#pragma unroll
    for (int m = 0; m < 4; ++m) neg[m] = -__uint_as_float((150u - 4u * (uint32_t)m) << 23);
}

// Offset of the coarse-bin middle: (2^(4-t) - 1) / 2.
__device__ __forceinline__ double bin_offset(int t)
{
    return (double)((1 << (kBits - t)) - 1) * 0.5;
}

// ------------------------------------------------------- per-head set-up
// Builds the union channel list (by reader set, then channel, for groups of
// up to 4 query heads; channel order otherwise), plane-row table, weights
// (zero for a query that does not read the channel at full union depth) and
// biases for query heads q_rows[0..G) of KV head h.
// tu_row: the union plan to read; t_rows: each query's own plan.  With
// mn_h and sc_h null (grouped per-token-block scales) the tables hold the
// unscaled weights w = q and the bias of mn = 0, scale = 1; each scanning
// CTA then applies its own block's scales.
// Thread c handles channel c: at least 256 threads, d <= 256.  Ends with a
// barrier.
template <int GP>
__device__ void setup_head(ScanMeta<GP> &sm, int h, int G, int d, const uint8_t *tu_row,
                           const uint8_t *t_rows, const uint16_t *q_rows, const float *mn_h,
                           const float *sc_h)
{
    __shared__ double bias_part[kScanThreads / 32][GP];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = tid;
    const bool in = c < d;
    // every input of channel c, loaded at once
    int T = 0;
    float sc = 0.0f, mn = 0.0f;
    int tg[GP];
    float qf[GP];
    if (in) {
        T = min((int)tu_row[c], kBits);
        sc = sc_h ? sc_h[c] : 1.0f;
        mn = mn_h ? mn_h[c] : 0.0f;
    }
#pragma unroll
    for (int g = 0; g < GP; ++g) {
        const bool live = in && g < G;
        tg[g] = live ? (int)t_rows[g * d + c] : 0;
        qf[g] = live ? bf16_to_float(q_rows[g * d + c]) : 0.0f;
    }
    const bool has = T > 0;
    // reader sets of this channel: full = queries reading all T planes,
    // partial = queries reading 0 < t < T of them; each query's bias term
    // q_gc * (mn_c + scale_c * (2^(4-t) - 1) / 2) at its own clamped depth
    unsigned full = 0, partial = 0;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
        tg[g] = min(tg[g], T);
        if (has && tg[g] == T) full |= 1u << g;
        else if (tg[g] > 0) partial |= 1u << g;
        double term = in ? (double)qf[g] * ((double)mn + (double)sc * bin_offset(tg[g])) : 0.0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) term += __shfl_xor_sync(0xFFFFFFFFu, term, off);
        if (lane == 0 && warp < kScanThreads / 32) bias_part[warp][g] = term;
    }
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, has);
    if (lane == 0 && warp < kScanThreads / 32) sm.part[warp] = __popc(bal);
    if (tid < kMaxHeadDim / kStageChannels) {
        sm.stage_partial[tid] = 0;
        sm.stage_mask[tid] = 0u;
    }
    // position among the lanes of this warp with the same ordering key
    const unsigned key = mask_ordered<GP>() ? reader_set_rank(full) : 0u;
    int lane_rank = __popc(bal & ((1u << lane) - 1u));
    if (mask_ordered<GP>()) {
#pragma unroll
        for (unsigned v = 0; v < (1u << GP); ++v) {
            const unsigned b = __ballot_sync(0xFFFFFFFFu, has && key == v);
            if (lane == 0 && warp < kScanThreads / 32) sm.order[warp][v] = __popc(b);
            if (key == v) lane_rank = __popc(b & ((1u << lane) - 1u));
        }
    }
    __syncthreads();
    int U = 0;
#pragma unroll
    for (int w = 0; w < kScanThreads / 32; ++w) U += sm.part[w];
    if (tid < GP) {
        double acc = 0.0;
#pragma unroll
        for (int w = 0; w < kScanThreads / 32; ++w) acc += bias_part[w][tid];
        sm.bias[tid] = (float)acc;
    }
    if (mask_ordered<GP>()) {
        // warp 0 turns the (warp, key) counts into exclusive offsets in
        // (key, warp) order
        if (warp == 0) {
            const unsigned v = (unsigned)lane;
            int tot = 0, cnt[kScanThreads / 32];
#pragma unroll
            for (int w = 0; w < kScanThreads / 32; ++w) {
                cnt[w] = (v < (1u << GP)) ? sm.order[w][v] : 0;
                tot += cnt[w];
            }
            int incl = tot;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off) incl += y;
            }
            int at = incl - tot;
            if (v < (1u << GP)) {
#pragma unroll
                for (int w = 0; w < kScanThreads / 32; ++w) {
                    sm.order[w][v] = at;
                    at += cnt[w];
                }
            }
        }
        __syncthreads();
    }
    int base = 0;
    if (mask_ordered<GP>()) {
        base = has ? sm.order[warp][key] : 0;
    } else {
#pragma unroll
        for (int w = 0; w < kScanThreads / 32; ++w) base += (w < warp) ? sm.part[w] : 0;
    }
    const int n_stages = (U + kStageChannels - 1) / kStageChannels;
    if (has) {
        const int u = base + lane_rank;
#pragma unroll
        for (int g = 0; g < GP; ++g) {
            const float w = __fmul_rn(qf[g], sc);
            // full-depth readers use W2 in the unconditional fma; others add 0
            // there and, if partial, their own masked term
            sm.W2[u][g] = (tg[g] == T) ? make_float2(w, w) : make_float2(0.0f, 0.0f);
            sm.Wp[u][g] = w;
            sm.tq[u][g] = (uint8_t)tg[g];
        }
        sm.meta[u] = full | (partial << 16);
        if (partial) sm.stage_partial[u / kStageChannels] = 1;
        atomicOr(&sm.stage_mask[u / kStageChannels], full);
#pragma unroll
        for (int s2 = 0; s2 < kBits; ++s2)
            sm.row_g[u * kBits + s2] = (s2 < T) ? (uint32_t)((h * d + c) * kBits + s2) : 0xFFFFFFFFu;
    }
    for (int i = U * kBits + tid; i < n_stages * kStageRows; i += blockDim.x) sm.row_g[i] = 0xFFFFFFFFu;
    if (tid == 0) {
        sm.U = U;
        sm.n_stages = n_stages;
    }
    __syncthreads();
}

// Per-head tables are built once per (session, KV head) by threshold_kernel
// and copied by every CTA that scans the head: one round trip instead of the
// dependent loads, barriers and fp64 bias sums of setup_head.  Ends with a
// barrier; completes every cp.async group in flight.
template <int GP>
__device__ __forceinline__ void load_head(ScanMeta<GP> &sm, const unsigned char *tables, int h)
{
    constexpr int kUnits = (int)(sizeof(ScanMeta<GP>) / 16);
    const uint4 *src = reinterpret_cast<const uint4 *>(tables + (size_t)h * sizeof(ScanMeta<GP>));
    uint4 *dst = reinterpret_cast<uint4 *>(&sm);
    for (int i = threadIdx.x; i < kUnits; i += blockDim.x) cp_async16_full(dst + i, src + i);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
}

// ------------------------------------------------------------- chunk scan
// Copy stage st (32 plane rows x the chunk's 16-byte column groups in
// [col_lo, col_hi)) into stage buffer buf.  Rows past a channel's depth and
// columns past col_hi are zero-filled with no global read.
template <int GP>
__device__ __forceinline__ void load_stage(const ScanMeta<GP> &sm, StageBuf stage, int st,
                                           int buf, const uint32_t *planes, int n_words,
                                           int col_lo, int col_hi)
{
    if (threadIdx.x >= kScanThreads) return;   // a larger CTA's extra threads copy nothing
    const int chunk = threadIdx.x & 15;
    const int col = col_lo + chunk * 4;
    const bool ok = col < col_hi;
    const uint32_t *rows = &sm.row_g[st * kStageRows];
#pragma unroll
    for (int row = threadIdx.x >> 4; row < kStageRows; row += kScanThreads / 16) {
        const uint32_t g = rows[row];
        const bool live = ok && g != 0xFFFFFFFFu;
        copy_or_zero16(&stage[buf][row][chunk * 4], planes + (size_t)g * (size_t)n_words + col, live);
    }
}

// The thread's 8 nibbles of one channel: bit 4m+r of the word in slot s
// (bit 3-s of the code) moves to bit 4m+(3-s) by a rotate and a mask.
// sh[p] = (r - p) mod 32.
template <int COLS = kTileCols>
__device__ __forceinline__ uint32_t gather_nibbles(const uint32_t (*rows)[COLS], int col,
                                                   const uint32_t (&sh)[4])
{
    const uint32_t x0 = rows[0][col], x1 = rows[1][col], x2 = rows[2][col], x3 = rows[3][col];
    uint32_t nib = __funnelshift_r(x0, x0, sh[3]) & 0x88888888u;
    nib |= __funnelshift_r(x1, x1, sh[2]) & 0x44444444u;
    nib |= __funnelshift_r(x2, x2, sh[1]) & 0x22222222u;
    nib |= __funnelshift_r(x3, x3, sh[0]) & 0x11111111u;
    return nib;
}

// Queries reading fewer planes than the union drop the low bits first.
template <int GP>
__device__ __forceinline__ void fma_partial(unsigned pmask, uint32_t nib, int u,
                                            const ScanMeta<GP> &sm,
                                            const float (&neg)[4],
                                            float2 (&acc)[GP][4])
{
#pragma unroll
    for (int g = 0; g < GP; ++g) {
        if (pmask & (1u << g)) {
            const int tg = sm.tq[u][g];
            const uint32_t keep = ((0xFu << (kBits - tg)) & 0xFu) * 0x11111111u;
            float2 vm[4];
            nibbles_to_floats(nib & keep, neg, vm);
            const float w = sm.Wp[u][g];
            const float2 w2 = make_float2(w, w);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[g][i] = __ffma2_rn(vm[i], w2, acc[g][i]);
        }
    }
}

// One union channel: gather the thread's 8 nibbles, convert, and add
// W2[u][g] * v for every query head (W2 is zero for heads that do not read
// the channel at full union depth).
template <int GP, bool kPartial, int COLS = kTileCols>
__device__ __forceinline__ void channel(const ScanMeta<GP> &sm, const uint32_t (*rows)[COLS],
                                        int u, int col, const uint32_t (&sh)[4],
                                        const float (&neg)[4], float2 (&acc)[GP][4])
{
    const uint32_t nib = gather_nibbles<COLS>(rows, col, sh);
    float2 v[4];
    nibbles_to_floats(nib, neg, v);
#pragma unroll
    for (int g = 0; g < GP; ++g) {
        const float2 w = sm.W2[u][g];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[g][i] = __ffma2_rn(v[i], w, acc[g][i]);
    }
    if (kPartial) {
        const uint32_t meta = sm.meta[u];
        if (meta >> 16) fma_partial<GP>(meta >> 16, nib, u, sm, neg, acc);
    }
}

// One union channel read at full union depth by exactly the queries in
// MASK (and by no query at a partial depth): FMAs for those queries only.
// rp: the thread's word of slot 0 of the channel in the stage buffer (the
// other slots follow COLS words apart); w2: the channel's weights.
template <int GP, unsigned MASK, int COLS>
__device__ __forceinline__ void channel_masked(const float2 (&w2)[GP], const uint32_t *rp,
                                               const uint32_t (&sh)[4], const float (&neg)[4],
                                               float2 (&acc)[GP][4])
{
    const uint32_t x0 = rp[0], x1 = rp[COLS], x2 = rp[2 * COLS], x3 = rp[3 * COLS];
    uint32_t nib = __funnelshift_r(x0, x0, sh[3]) & 0x88888888u;
    nib |= __funnelshift_r(x1, x1, sh[2]) & 0x44444444u;
    nib |= __funnelshift_r(x2, x2, sh[1]) & 0x22222222u;
    nib |= __funnelshift_r(x3, x3, sh[0]) & 0x11111111u;
    float2 v[4];
    nibbles_to_floats(nib, neg, v);
#pragma unroll
    for (int g = 0; g < GP; ++g) {
        if ((MASK >> g) & 1u) {
            const float2 w = w2[g];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[g][i] = __ffma2_rn(v[i], w, acc[g][i]);
        }
    }
}

template <int GP, unsigned MASK, int COLS>
__device__ __forceinline__ void stage_masked(const ScanMeta<GP> &sm, const uint32_t (*rows)[COLS],
                                             int u0, int col, const uint32_t (&sh)[4],
                                             const float (&neg)[4],
                                             float2 (&acc)[GP][4])
{
    if constexpr (MASK < (1u << GP)) {
        // stage-local bases: every load below is a constant offset from them
        const float2(*W)[GP] = sm.W2 + u0;
        const uint32_t *rp = &rows[0][col];
        // unrolled by 2 only: 16 specialised bodies unrolled 8 times miss in
        // the instruction cache
#pragma unroll 2
        for (int j = 0; j < kStageChannels; ++j)
            channel_masked<GP, MASK, COLS>(W[j], rp + kBits * COLS * j, sh, neg, acc);
    }
}

// A full stage with no partial-depth reader, specialised to the set of
// queries that read its channels (a query outside the set multiplies zeros).
template <int GP, int COLS>
__device__ __forceinline__ void stage_dispatch(unsigned mask, const ScanMeta<GP> &sm,
                                               const uint32_t (*rows)[COLS], int u0, int col,
                                               const uint32_t (&sh)[4],
                                               const float (&neg)[4],
                                               float2 (&acc)[GP][4])
{
    switch (mask) {
    case 1: stage_masked<GP, 1, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 2: stage_masked<GP, 2, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 3: stage_masked<GP, 3, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 4: stage_masked<GP, 4, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 5: stage_masked<GP, 5, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 6: stage_masked<GP, 6, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 7: stage_masked<GP, 7, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 8: stage_masked<GP, 8, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 9: stage_masked<GP, 9, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 10: stage_masked<GP, 10, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 11: stage_masked<GP, 11, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 12: stage_masked<GP, 12, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 13: stage_masked<GP, 13, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    case 14: stage_masked<GP, 14, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    default: stage_masked<GP, 15, COLS>(sm, rows, u0, col, sh, neg, acc); break;
    }
}

// Channels [u0, u1) of the stage held in `rows` (channel u0 in rows 0..3).
template <int GP, int COLS = kTileCols>
__device__ __forceinline__ void compute_stage(const ScanMeta<GP> &sm, int st,
                                              const uint32_t (*rows)[COLS], int u0, int u1,
                                              int col, const uint32_t (&sh)[4],
                                              const float (&neg)[4],
                                              float2 (&acc)[GP][4])
{
    if (u1 - u0 == kStageChannels && !sm.stage_partial[st]) {
        if constexpr (mask_ordered<GP>()) {
            stage_dispatch<GP, COLS>(sm.stage_mask[st], sm, rows, u0, col, sh, neg, acc);
        } else {
#pragma unroll
            for (int j = 0; j < kStageChannels; ++j)
                channel<GP, false, COLS>(sm, rows + kBits * j, u0 + j, col, sh, neg, acc);
        }
    } else {
        for (int u = u0; u < u1; ++u)
            channel<GP, true, COLS>(sm, rows + kBits * (u - u0), u, col, sh, neg, acc);
    }
}

// Scores of the thread's 8 keys of the chunk of plane words [col_lo, col_hi)
// (at most 64 words) for every query head:
// score(g, m) = bias_g + acc[g][m % 4].{x if m < 4 else y}.
// Warps whose 8 columns lie past col_hi only take part in the copies and
// barriers.  Starts with a barrier (stage buffers may still be in use).
template <int GP, int STAGES>
__device__ void scan_chunk(const ScanMeta<GP> &sm, StageBuf stage, const uint32_t *planes,
                           int n_words, int col_lo, int col_hi, float2 (&acc)[GP][4])
{
    const int col = threadIdx.x >> 2, r = threadIdx.x & 3;
    const bool busy = col_lo + ((threadIdx.x >> 5) << 3) < col_hi;   // warp-uniform
    uint32_t sh[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) sh[p] = (uint32_t)(r - p) & 31u;
    float neg[4];
    magic_negatives(neg);
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[g][i] = make_float2(0.0f, 0.0f);
    const int n_stages = sm.n_stages;
    const int U = sm.U;
    __syncthreads();
#pragma unroll
    for (int st = 0; st < STAGES - 1; ++st) {
        if (st < n_stages) load_stage(sm, stage, st, st, planes, n_words, col_lo, col_hi);
        cp_async_commit();
    }
    for (int st = 0; st < n_stages; ++st) {
        cp_async_wait<STAGES - 2>();
        __syncthreads();
        const int nx = st + STAGES - 1;
        if (nx < n_stages) load_stage(sm, stage, nx, nx % STAGES, planes, n_words, col_lo, col_hi);
        cp_async_commit();
        if (busy) {
            const int u0 = st * kStageChannels;
            compute_stage<GP>(sm, st, stage[st % STAGES], u0, min(u0 + kStageChannels, U), col, sh,
                              neg, acc);
        }
    }
    cp_async_wait<0>();
}

__device__ __forceinline__ float score_of(const float2 (&a)[4], int m, float bias)
{
    const float2 p = a[m & 3];
    return bias + ((m < 4) ? p.x : p.y);
}

template <int NS>
__device__ __forceinline__ int find_session_by_chunk(const Batch<NS> &b, int ci)
{
    int si = 0;
    for (int s = 1; s < b.n_sessions; ++s)
        if (b.s[s].chunk_begin <= ci) si = s;
    return si;
}

template <int NS>
__device__ __forceinline__ int find_session_by_head(const Batch<NS> &b, int gh)
{
    int si = 0;
    for (int s = 1; s < b.n_sessions; ++s)
        if (b.s[s].head_begin <= gh) si = s;
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

template <int NS>
__device__ __forceinline__ int find_session_by_block(const Batch<NS> &b, int gi)
{
    int si = 0;
    for (int s = 1; s < b.n_sessions; ++s)
        if (b.s[s].blk_begin <= gi) si = s;
    return si;
}

// ------------------------------------------------ grouped per-block biases
// The CTA of (session, KV head, scale block holding keys) number gi: the
// bias of each query head of the KV head with that block's scales,
//   bias_g = sum_c q_gc * (mn_bc + scale_bc * (2^(4-t)-1)/2),
// t the query's depth clamped to the union, summed exactly as setup_head
// sums the bias of a one-block index (fp64 terms, warp shuffles, the first
// kScanThreads / 32 warps in order).  Thread c handles channel c; a CTA of
// more threads leaves the rest idle.  Runs as extra CTAs of the threshold
// launch, for the scan and the exact path.
template <int NS>
__device__ void block_bias_cta(const Batch<NS> &b, int gi)
{
    __shared__ double part[kScanThreads / 32][kMaxGroup];
    const SessionDesc &S = b.s[find_session_by_block(b, gi)];
    const int local = gi - S.blk_begin;
    const int h = local / S.n_filled, blk = local - h * S.n_filled;
    const int G = b.G, d = b.d;
    const int c = threadIdx.x, lane = c & 31, warp = c >> 5;
    const bool in = c < d;
    int T = 0;
    float mn = 0.0f, sc = 0.0f;
    if (in) {
        T = min((int)S.tu[h * d + c], kBits);
        const size_t e = ((size_t)h * S.nb + blk) * d + c;
        mn = S.mn[e];
        sc = S.scale[e];
    }
    for (int g = 0; g < G; ++g) {
        double term = 0.0;
        if (in) {
            const int tg = min((int)S.t[(size_t)(h * G + g) * d + c], T);
            const float qf = bf16_to_float(S.q[(size_t)(h * G + g) * d + c]);
            term = (double)qf * ((double)mn + (double)sc * bin_offset(tg));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) term += __shfl_xor_sync(0xFFFFFFFFu, term, off);
        if (lane == 0 && warp < kScanThreads / 32) part[warp][g] = term;
    }
    __syncthreads();
    if (c < G) {
        double acc = 0.0;
#pragma unroll
        for (int w = 0; w < kScanThreads / 32; ++w) acc += part[w][c];
        S.bias_blk[((size_t)h * S.nb + blk) * G + c] = (float)acc;
    }
}

// The CTA's block: scale the unscaled weights of the head's tables by the
// block's channel scales and take the block's biases.  Ends with a barrier.
template <int GP>
__device__ __forceinline__ void apply_block(ScanMeta<GP> &sm, const SessionDesc &S, int h, int blk,
                                            int G, int d)
{
    const int U = sm.U;
    const float *sc_row = S.scale + ((size_t)h * S.nb + blk) * d;
    for (int i = threadIdx.x; i < U * GP; i += blockDim.x) {
        const int u = i / GP, g = i - u * GP;
        const int c = (int)(sm.row_g[u * kBits] / kBits) - h * d;   // slot 0 of every union channel
        const float sc = sc_row[c];
        const float2 w2 = sm.W2[u][g];
        sm.W2[u][g] = make_float2(__fmul_rn(w2.x, sc), __fmul_rn(w2.y, sc));
        sm.Wp[u][g] = __fmul_rn(sm.Wp[u][g], sc);
    }
    if (threadIdx.x < GP)
        sm.bias[threadIdx.x] =
            (threadIdx.x < G) ? S.bias_blk[((size_t)h * S.nb + blk) * G + threadIdx.x] : 0.0f;
    __syncthreads();
}

// ------------------------------------------------------- filtered scan
// CTA i owns column groups [i*per_cta, (i+1)*per_cta) of the linear
// (session, KV head, column group) space (one 64-word chunk, or two pieces
// where the range crosses a KV head's end) and appends the keys scoring
// >= theta to their query's candidate buffer.
template <int NS, int GP, int STAGES, bool kBlocked>
__global__ void __launch_bounds__(kScanThreads, (GP >= 8) ? 2 : 4)
scan_kernel(const __grid_constant__ Batch<NS> b)
{
    __shared__ ScanMeta<GP> sm;
    __shared__ float s_theta_f[GP];
    extern __shared__ __align__(16) uint32_t scan_dyn[];
    StageBuf stage = reinterpret_cast<StageBuf>(scan_dyn);
    const int G = b.G;
    const int col = threadIdx.x >> 2, r = threadIdx.x & 3, lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    {
        // this CTA's chunk: chunk c of the KV head's S.chunks equal parts of
        // its column groups (at most 16 groups = 64 words each)
        const int si = find_session_by_chunk(b, (int)blockIdx.x);
        const SessionDesc &S = b.s[si];
        const int local = (int)blockIdx.x - S.chunk_begin;
        const int h = local / S.chunks;
        const int c = local - h * S.chunks;
        int g0, g1, blk = 0;
        if constexpr (kBlocked) {
            // S.chunks / S.n_filled equal chunks per scale block: a chunk
            // never spans two blocks
            const int cpb = S.chunks / S.n_filled;
            blk = c / cpb;
            const int sub = c - blk * cpb;
            const int gb0 = blk * (S.block_words / 4);
            const int gbn = min(S.col_groups, gb0 + S.block_words / 4) - gb0;
            g0 = gb0 + (int)((long long)sub * gbn / cpb);
            g1 = gb0 + (int)((long long)(sub + 1) * gbn / cpb);
        } else {
            // the first chunk_rem chunks take one column group more
            g0 = c * S.chunk_q + min(c, S.chunk_rem);
            g1 = g0 + S.chunk_q + (c < S.chunk_rem ? 1 : 0);
        }
        const int col_lo = g0 * 4;
        const int width = (g1 - g0) * 4;               // plane words owned by this chunk
        const int col_hi = min(S.n_cols, col_lo + width);
        const int q0 = h * G;
        if (threadIdx.x < GP) {
            // order_key(s) >= theta  <=>  s >= theta's float (up to the sign of
            // zero, which can only add a candidate); theta 0 passes every key
            const uint32_t theta = (threadIdx.x < G)
                                       ? S.qstate[(q0 + threadIdx.x) * kQueryStateWords + 0]
                                       : 0xFFFFFFFFu;
            s_theta_f[threadIdx.x] = theta == 0u ? -INFINITY : order_key_to_float(theta);
        }
        load_head<GP>(sm, S.tables, h);   // ends with a barrier
        if constexpr (kBlocked) apply_block<GP>(sm, S, h, blk, G, b.d);
        float2 acc[GP][4];
        scan_chunk<GP, STAGES>(sm, stage, S.planes, S.n_words, col_lo, col_hi, acc);

        // keys scoring >= theta: each warp reserves room for its own keys in
        // each query's candidate buffer (one atomic per query with any such
        // key; no CTA-wide step), then writes them
        if (col_lo + (warp << 3) >= col_hi) return;   // no keys in this warp
        const bool mine = col < width && col_lo + col < col_hi;
        const int key0 = (col_lo + col) * 32 + r;
        // keys key0 + 4m for m < live are real keys (the rest pad the last word)
        const int live = mine ? max(0, min(8, (S.n - key0 + 3) >> 2)) : 0;
        const unsigned live_mask = (1u << live) - 1u;
#pragma unroll
        for (int gg = 0; gg < GP; ++gg) {
            if (gg >= G) break;
            const float bias = sm.bias[gg];
            const float th = s_theta_f[gg];
            // first the thread's best key: most warps hold no key >= theta
            float mx = fmaxf(fmaxf(acc[gg][0].x, acc[gg][0].y), fmaxf(acc[gg][1].x, acc[gg][1].y));
            mx = fmaxf(mx, fmaxf(fmaxf(acc[gg][2].x, acc[gg][2].y), fmaxf(acc[gg][3].x, acc[gg][3].y)));
            if (!__any_sync(0xFFFFFFFFu, live > 0 && bias + mx >= th)) continue;
            unsigned pass = 0u;
#pragma unroll
            for (int m = 0; m < 8; ++m)
                pass |= (score_of(acc[gg], m, bias) >= th) ? (1u << m) : 0u;
            pass &= live_mask;
            const int cnt = __popc(pass);
            int inc = cnt;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, inc, off);
                if (lane >= off) inc += y;
            }
            unsigned at = 0;
            if (lane == 31 && inc) at = atomicAdd(&S.qstate[(q0 + gg) * kQueryStateWords + 1], (unsigned)inc);
            at = __shfl_sync(0xFFFFFFFFu, at, 31);
            unsigned pos = at + (unsigned)(inc - cnt);
            unsigned long long *cq = S.cand + (size_t)(q0 + gg) * b.cap;
            while (pass) {   // the set bits only
                const int m = __ffs(pass) - 1;
                pass &= pass - 1u;
                const float2 p01 = (m & 1) ? acc[gg][1] : acc[gg][0];
                const float2 p23 = (m & 1) ? acc[gg][3] : acc[gg][2];
                const float2 p = (m & 2) ? p23 : p01;
                const float sc = bias + ((m & 4) ? p.y : p.x);
                if (pos < (unsigned)b.cap)
                    cq[pos] = composite(order_key(sc), (uint32_t)(key0 + 4 * m));
                ++pos;
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

// Writes the k selected composites `sel` (okey << 32 | ~index, kpad slots,
// kpad a power of two >= k) to the outputs in ascending key index by sorting
// them on the index (bitonic network); for any number of keys.
__device__ void emit_sorted_by_index(unsigned long long *sel, int k, int kpad, int32_t *out_idx,
                                     float *out_score)
{
    for (int i = threadIdx.x; i < k; i += blockDim.x) sel[i] = (sel[i] << 32) | (sel[i] >> 32);
    for (int i = k + threadIdx.x; i < kpad; i += blockDim.x) sel[i] = 0ull;
    __syncthreads();
    bitonic_sort_desc(sel, kpad);
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        const unsigned long long v = sel[i];
        out_idx[i] = (int32_t)(~(uint32_t)(v >> 32));
        out_score[i] = order_key_to_float((uint32_t)(v & 0xFFFFFFFFull));
    }
}

// Writes the k <= kMaxFastK selected composites `sel` (okey << 32 | ~index)
// to the outputs in ascending key index, for any number of keys n: the keys
// are counted into at most kSelBins buckets of consecutive indices, the
// buckets' exclusive prefix gives each bucket its output range, every key is
// scattered into its bucket's range (`tmp`, k slots), and each key's place
// inside its bucket is the number of keys there with a smaller index (the
// buckets hold about one key each).  The cost follows k, not n.
// Called by all kSelThreads threads; uses ss.hist and ss.wsum.
constexpr int kEmitPerThread = kMaxFastK / kSelThreads;   // 4
__device__ void emit_by_buckets(const unsigned long long *sel, int k, int n,
                                unsigned long long *tmp, SelShared &ss, int32_t *out_idx,
                                float *out_score)
{
    const int shift = max(0, bit_length((uint32_t)max(n - 1, 1)) - kSelBits);
    unsigned *cnt = ss.hist;
#pragma unroll
    for (int i = 0; i < kSelBinsPerThread; ++i) cnt[threadIdx.x + i * kSelThreads] = 0u;
    __syncthreads();
    unsigned slot[kEmitPerThread];
#pragma unroll
    for (int e = 0; e < kEmitPerThread; ++e) {
        const int i = threadIdx.x + e * kSelThreads;
        if (i < k) {
            const uint32_t j = ~(uint32_t)(sel[i] & 0xFFFFFFFFull);
            slot[e] = atomicAdd(&cnt[j >> shift], 1u);
        }
    }
    __syncthreads();
    // thread t owns bins 4t .. 4t+3: their exclusive prefix, in place
    unsigned c4[kSelBinsPerThread], mine = 0;
#pragma unroll
    for (int i = 0; i < kSelBinsPerThread; ++i) {
        c4[i] = cnt[kSelBinsPerThread * threadIdx.x + i];
        mine += c4[i];
    }
    unsigned total;
    unsigned run = block_exclusive_scan(mine, ss.wsum, &total);
#pragma unroll
    for (int i = 0; i < kSelBinsPerThread; ++i) {
        cnt[kSelBinsPerThread * threadIdx.x + i] = run;
        run += c4[i];
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kEmitPerThread; ++e) {
        const int i = threadIdx.x + e * kSelThreads;
        if (i < k) {
            const uint32_t j = ~(uint32_t)(sel[i] & 0xFFFFFFFFull);
            tmp[cnt[j >> shift] + slot[e]] = sel[i];
        }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kEmitPerThread; ++e) {
        const int i = threadIdx.x + e * kSelThreads;
        if (i < k) {
            const unsigned long long v = sel[i];
            const uint32_t j = ~(uint32_t)(v & 0xFFFFFFFFull);
            const unsigned bk = j >> shift;
            const unsigned lo = cnt[bk];
            const unsigned hi = (bk + 1 < (unsigned)kSelBins) ? cnt[bk + 1] : (unsigned)k;
            unsigned pos = lo;
            for (unsigned x = lo; x < hi; ++x)
                pos += (~(uint32_t)(tmp[x] & 0xFFFFFFFFull) < j) ? 1u : 0u;
            out_idx[pos] = (int32_t)j;
            out_score[pos] = order_key_to_float((uint32_t)(v >> 32));
        }
    }
}

// ------------------------------------------------------- sampled threshold
// One CTA per query: score the query's sampled keys (m_tiles whole 64-word
// tiles, evenly strided) from its own plan, then theta = the lower edge of a
// 2^-22-of-the-range bin holding the sample_rank-th largest sampled order key
// (two 11-bit radix passes; any theta is correct, it only sizes the candidate
// set).  The query's channels, weights and bias come straight from its plan
// and the index statistics; H further CTAs of the same launch build each KV
// head's scan tables for the filtering pass.  Stages of 8 own
// channels x 2 tiles are copied with cp.async, three in flight; every query of
// a KV head reads its sampled rows itself (a few tens of KB, mostly L2 hits).
// A pass scores 2 tiles (one per thread) or, with more than 2 sampled tiles,
// 4 (two per thread), so a sample of up to 4 tiles takes one pass.
constexpr int kThetaThreadTiles = kSelThreads / kScanThreads;             // 2
constexpr int kThetaTilesPerPass = 2 * kThetaThreadTiles;                 // 4
constexpr int kThetaCols = kThetaTilesPerPass * kTileCols;                // 256 words
typedef uint32_t (*ThetaBuf)[kStageRows][kThetaCols];
constexpr size_t kThetaStageBytes = (size_t)kStageRows * kThetaCols * sizeof(uint32_t);
constexpr int kThetaResolutionBits = 2 * kSelBits;
constexpr int kThetaBufs = 3;   // stages in flight

template <int NS, int GP, bool kBlocked>
__global__ void __launch_bounds__(kSelThreads) threshold_kernel(const __grid_constant__ Batch<NS> b,
                                                                uint32_t force_exact,
                                                                int total_queries, int table_ctas)
{
    extern __shared__ __align__(16) uint32_t th_dyn[];
    __shared__ ScanMeta<GP> sm;
    __shared__ SelShared ss;
    __shared__ uint16_t own_c[kMaxHeadDim];   // the query's channels (t > 0) ...
    __shared__ uint8_t own_t[kMaxHeadDim];    // ... their depths ...
    __shared__ float own_w[kMaxHeadDim];      // ... and weights q*scale (q with grouped scales)
    __shared__ double bias_part[kSelThreads / 32];
    __shared__ float bias_s;
    // grouped scales: the weights and bias of the pass's tiles' blocks
    __shared__ float tile_w[kBlocked ? kThetaTilesPerPass : 1][kBlocked ? kMaxHeadDim : 1];
    __shared__ float tile_bias[kThetaTilesPerPass];
    __shared__ float tile_bias_part[kBlocked ? kSelThreads / 32 : 1][kThetaTilesPerPass];
    ThetaBuf stage = reinterpret_cast<ThetaBuf>(th_dyn);
    uint32_t *vals = th_dyn + kThetaBufs * kStageRows * kThetaCols;
    const int G = b.G, d = b.d;
    if constexpr (kBlocked) {
        if (blockIdx.x >= total_queries + table_ctas) {   // a (KV head, block)'s biases
            block_bias_cta(b, blockIdx.x - total_queries - table_ctas);
            return;
        }
    }
    if (blockIdx.x >= total_queries) {   // a KV head's tables for the filtering pass
        const int gh = blockIdx.x - total_queries;
        const SessionDesc &S = b.s[find_session_by_head(b, gh)];
        const int h = gh - S.head_begin;
        setup_head<GP>(sm, h, G, d, S.tu + h * d, S.t + (size_t)h * G * d, S.q + (size_t)h * G * d,
                       kBlocked ? nullptr : S.mn + h * d, kBlocked ? nullptr : S.scale + h * d);
        constexpr int kUnits = (int)(sizeof(ScanMeta<GP>) / 16);
        const uint4 *src = reinterpret_cast<const uint4 *>(&sm);
        uint4 *dst = reinterpret_cast<uint4 *>(S.tables + (size_t)h * sizeof(ScanMeta<GP>));
        for (int i = threadIdx.x; i < kUnits; i += blockDim.x) dst[i] = src[i];
        return;
    }
    const int gq = blockIdx.x;
    const int si = find_session_by_query(b, gq);
    const SessionDesc &S = b.s[si];
    const int qq = gq - S.q_begin;
    const int h = qq / G;
    uint32_t *st = S.qstate + qq * kQueryStateWords;
    if (force_exact || S.exact_only) {
        if (threadIdx.x == 0) { st[0] = 0xFFFFFFFFu; st[1] = 0; st[2] = 1; }
        return;
    }
    if (S.m_tiles == 0) {   // few keys: every key is a candidate
        if (threadIdx.x == 0) { st[0] = 0; st[1] = 0; st[2] = 0; }
        return;
    }
    // the query's own plan: channel c on thread c, depth clamped to the union
    {
        const int c = threadIdx.x, lane = c & 31, warp = c >> 5;
        int tq = 0;
        float w = 0.0f;
        double term = 0.0;
        if (c < d) {
            const int T = min((int)S.tu[h * d + c], kBits);
            tq = min((int)S.t[(size_t)qq * d + c], T);
            const float qf = bf16_to_float(S.q[(size_t)qq * d + c]);
            if constexpr (kBlocked) {
                w = qf;   // scaled per sampled tile below; the bias is per block
            } else {
                const float sc = S.scale[h * d + c];
                w = __fmul_rn(qf, sc);
                term = (double)qf * ((double)S.mn[h * d + c] + (double)sc * bin_offset(tq));
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) term += __shfl_xor_sync(0xFFFFFFFFu, term, off);
        if (lane == 0) bias_part[warp] = term;
        unsigned n_own;
        const unsigned pos = block_exclusive_scan(tq > 0 ? 1u : 0u, ss.wsum, &n_own);
        if (tq > 0) {
            own_c[pos] = (uint16_t)c;
            own_t[pos] = (uint8_t)tq;
            own_w[pos] = w;
        }
        if (threadIdx.x == 0) {
            double acc = 0.0;
            for (int w2 = 0; w2 < kSelThreads / 32; ++w2) acc += bias_part[w2];
            bias_s = (float)acc;
            ss.krem = n_own;   // parked until the barrier below
        }
        __syncthreads();
    }
    const int n_own = (int)ss.krem;
    const int n_stages = (n_own + kStageChannels - 1) / kStageChannels;
    // tiles per pass, and per thread (tiles sub and sub + kThetaThreadTiles)
    const int pass_tiles = S.m_tiles > kThetaThreadTiles ? kThetaTilesPerPass : kThetaThreadTiles;
    const int thread_tiles = pass_tiles / kThetaThreadTiles;
    const int sub = threadIdx.x / kScanThreads;             // first tile of the pass
    const int lt = threadIdx.x - sub * kScanThreads;
    const int col = lt >> 2, r = lt & 3;
    uint32_t sh[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) sh[p] = (uint32_t)(r - p) & 31u;
    float neg[4];
    magic_negatives(neg);
    const float bias = bias_s;
    const size_t head_row0 = (size_t)h * d * kBits;
    // A stage: plane rows of own channels 8s..8s+7 (4 slots each, zeros past
    // the channel's depth), pass_tiles tiles x 16 column groups per row.
    // Thread copies e = tid + i*kSelThreads: row e >> lg_groups, 16-byte
    // group e & (groups - 1); the part that does not depend on the stage is
    // worked out once per pass.
    constexpr int kLoadIters = kStageRows * kThetaCols / 4 / kSelThreads;   // 4
    const int lg_groups = (pass_tiles == kThetaTilesPerPass) ? 6 : 5;       // 16 * pass_tiles
    const int n_copies = kStageRows << lg_groups;
    int l_wcol[kLoadIters];   // source column of copy i; -1: past the sample
    auto load = [&](int s, int bufi) {
#pragma unroll
        for (int i = 0; i < kLoadIters; ++i) {
            const int e = threadIdx.x + i * kSelThreads;
            if (e < n_copies) {
                const int row = e >> lg_groups, part = e & ((1 << lg_groups) - 1);
                const int j = s * kStageChannels + (row >> 2), slot = row & 3;
                const bool live = l_wcol[i] >= 0 && j < n_own && slot < own_t[min(j, kMaxHeadDim - 1)];
                const size_t grow = live ? head_row0 + (size_t)own_c[j] * kBits + slot : 0;
                copy_or_zero16(&stage[bufi][row][part * 4],
                               S.planes + grow * (size_t)S.n_words + max(l_wcol[i], 0), live);
            }
        }
        cp_async_commit();
    };
    for (int t0 = 0; t0 < S.m_tiles; t0 += pass_tiles) {
#pragma unroll
        for (int i = 0; i < kLoadIters; ++i) {
            const int part = (threadIdx.x + i * kSelThreads) & ((1 << lg_groups) - 1);
            const int tile = t0 + (part >> 4);
            const int wcol = tile * S.sample_stride * kTileCols + (part & 15) * 4;
            l_wcol[i] = (tile < S.m_tiles && wcol < S.n_cols) ? wcol : -1;
        }
        float2 acc[2][4];
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[k2][i] = make_float2(0.0f, 0.0f);
        __syncthreads();   // the buffers are free
        if constexpr (kBlocked) {
            // each sampled tile lies in one scale block (blocks hold whole tiles)
            for (int e = threadIdx.x; e < pass_tiles * kMaxHeadDim; e += kSelThreads) {
                const int tsub = e / kMaxHeadDim, j = e - tsub * kMaxHeadDim;
                const int tile = t0 + tsub;
                const int wcol = tile * S.sample_stride * kTileCols;
                if (j < n_own && tile < S.m_tiles && wcol < S.n_cols) {
                    const int blk = wcol / S.block_words;
                    tile_w[tsub][j] = __fmul_rn(
                        own_w[j], S.scale[((size_t)h * S.nb + blk) * d + own_c[j]]);
                }
            }
            // and the query's bias with each tile's block scales, summed here
            // in float (the threshold only sizes the candidate set; the scan
            // uses the biases the bias CTAs of this launch write)
            {
                const int c = threadIdx.x, lane = c & 31, warp = c >> 5;
                float qf = 0.0f;
                int tq = 0;
                if (c < d) {
                    qf = bf16_to_float(S.q[(size_t)qq * d + c]);
                    tq = min((int)S.t[(size_t)qq * d + c], min((int)S.tu[h * d + c], kBits));
                }
                for (int tsub = 0; tsub < pass_tiles; ++tsub) {
                    const int tile = t0 + tsub;
                    const int wcol = tile * S.sample_stride * kTileCols;
                    float term = 0.0f;
                    if (c < d && tile < S.m_tiles && wcol < S.n_cols) {
                        const size_t e = ((size_t)h * S.nb + wcol / S.block_words) * d + c;
                        term = qf * (S.mn[e] + S.scale[e] * (float)bin_offset(tq));
                    }
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1)
                        term += __shfl_xor_sync(0xFFFFFFFFu, term, off);
                    if (lane == 0) tile_bias_part[warp][tsub] = term;
                }
                __syncthreads();
                if (c < pass_tiles) {
                    float acc = 0.0f;
#pragma unroll
                    for (int w = 0; w < kSelThreads / 32; ++w) acc += tile_bias_part[w][c];
                    tile_bias[c] = acc;
                }
            }
            __syncthreads();
        }
        for (int s2 = 0; s2 < kThetaBufs - 1 && s2 < n_stages; ++s2) load(s2, s2);
        for (int s2 = 0; s2 < n_stages; ++s2) {
            // stage s2 has landed once at most (stages issued after it) groups are pending
            if (s2 + kThetaBufs - 1 < n_stages) {
                load(s2 + kThetaBufs - 1, (s2 + kThetaBufs - 1) % kThetaBufs);
                cp_async_wait<kThetaBufs - 1>();
            } else if (s2 + 1 < n_stages) {
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();
            const uint32_t(*rows)[kThetaCols] = stage[s2 % kThetaBufs];
            const int j1 = min(n_own, (s2 + 1) * kStageChannels);
            for (int j = s2 * kStageChannels; j < j1; ++j) {
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2) {
                    if (k2 < thread_tiles) {
                        const int tsub = sub + k2 * kThetaThreadTiles;
                        const uint32_t nib =
                            gather_nibbles<kThetaCols>(rows + kBits * (j - s2 * kStageChannels),
                                                       tsub * kTileCols + col, sh);
                        float2 v[4];
                        nibbles_to_floats(nib, neg, v);   // rows past the depth are zero
                        const float wj =
                            kBlocked ? tile_w[kBlocked ? tsub : 0][kBlocked ? j : 0] : own_w[j];
                        const float2 w2 = make_float2(wj, wj);
#pragma unroll
                        for (int i = 0; i < 4; ++i) acc[k2][i] = __ffma2_rn(v[i], w2, acc[k2][i]);
                    }
                }
            }
            __syncthreads();   // buffer s2 % kThetaBufs is reloaded kThetaBufs stages on
        }
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
            const int tsub = sub + k2 * kThetaThreadTiles;
            const int tile = t0 + tsub;
            if (k2 < thread_tiles && tile < S.m_tiles) {
                const int wcol = tile * S.sample_stride * kTileCols + col;
                const float tb = kBlocked ? tile_bias[tsub] : bias;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int j = wcol * 32 + r + 4 * m;
                    vals[tile * kTileKeys + col * 32 + r + 4 * m] =
                        (wcol < S.n_cols && j < S.n) ? order_key(score_of(acc[k2], m, tb)) : 0u;
                }
            }
        }
    }
    __syncthreads();
    const int m = S.m_keys;
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (int i = threadIdx.x; i < m; i += kSelThreads) {
        lo = min(lo, vals[i]);
        hi = max(hi, vals[i]);
    }
    sel_range(ss, lo, hi);
    const uint32_t base = ss.lo;
    const int top = 32 + bit_length(ss.hi - base);
    sel_run(ss, (unsigned)m, (unsigned)S.sample_rank, top, max(32, top - kThetaResolutionBits),
            [&](unsigned i) { return (unsigned long long)(vals[i] - base) << 32; });
    if (threadIdx.x == 0) {
        st[0] = base + (uint32_t)(ss.prefix >> 32);
        st[1] = 0;
        st[2] = 0;
    }
}

// ------------------------------------------------------------- exact path
// The exact top-k of query qq of session S by radix select over the
// composite (order key, ~index), recomputing the query's scores from its own
// plan on every pass: slow, rare (a query the sampled threshold did not suit,
// or a forced or k > kMaxFastK scan), and independent of the sample.  Run by
// the query's final CTA; threads past kScanThreads only take part in the
// barriers (the scan stages cover kScanThreads threads).  Uses the dynamic
// shared memory for its stages and the k selected.
template <int NS, bool kBlocked>
__device__ void exact_query(const Batch<NS> &b, const SessionDesc &S, int qq)
{
    __shared__ ScanMeta<1> sm;
    __shared__ SelectState ss;
    __shared__ float q_raw[kBlocked ? kMaxHeadDim : 1];   // unscaled weights (grouped scales)
    extern __shared__ __align__(16) uint32_t fb_dyn[];
    StageBuf stage = reinterpret_cast<StageBuf>(fb_dyn);
    unsigned long long *sel =
        reinterpret_cast<unsigned long long *>(fb_dyn + kMainStages * kStageRows * kTileCols);
    const int d = b.d, k = b.k;
    const int h = qq / b.G;
    const uint8_t *trow = S.t + (size_t)qq * d;
    setup_head<1>(sm, h, 1, d, trow, trow, S.q + (size_t)qq * d, kBlocked ? nullptr : S.mn + h * d,
                  kBlocked ? nullptr : S.scale + h * d);
    select_reset(ss, (unsigned)k);
    const int col = threadIdx.x >> 2, r = threadIdx.x & 3;
    float bias = sm.bias[0];
    int cur_blk = -1;
    if constexpr (kBlocked) {
        for (int u = threadIdx.x; u < sm.U; u += blockDim.x) q_raw[u] = sm.Wp[u][0];
        __syncthreads();
    }
    // grouped scales: before scanning tile c0, the weights and bias of its
    // block (the query reads every union channel at full depth here)
    auto use_block = [&](int c0) {
        if constexpr (kBlocked) {
            const int blk = c0 / S.block_words;
            if (blk != cur_blk) {
                __syncthreads();   // the previous tile's compute is done with sm
                const float *sc_row = S.scale + ((size_t)h * S.nb + blk) * d;
                for (int u = threadIdx.x; u < sm.U; u += blockDim.x) {
                    const int c = (int)(sm.row_g[u * kBits] / kBits) - h * d;
                    const float w = __fmul_rn(q_raw[u], sc_row[c]);
                    sm.W2[u][0] = make_float2(w, w);
                    sm.Wp[u][0] = w;
                }
                bias = S.bias_blk[((size_t)h * S.nb + blk) * b.G + (qq - h * b.G)];
                cur_blk = blk;
                __syncthreads();
            }
        }
    };
    float2 acc[1][4];
    for (int digit = 7; digit >= 0; --digit) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) ss.hist[i] = 0;
        __syncthreads();
        const unsigned long long pm = ss.pmask, pf = ss.prefix;
        for (int c0 = 0; c0 < S.n_cols; c0 += kTileCols) {
            const int c1 = min(S.n_cols, c0 + kTileCols);
            use_block(c0);
            scan_chunk<1, kMainStages>(sm, stage, S.planes, S.n_words, c0, c1, acc);
            const int key0 = (c0 + col) * 32 + r;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int j = key0 + 4 * m;
                if (c0 + col < c1 && j < S.n) {
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
    for (int c0 = 0; c0 < S.n_cols; c0 += kTileCols) {
        const int c1 = min(S.n_cols, c0 + kTileCols);
        use_block(c0);
        scan_chunk<1, kMainStages>(sm, stage, S.planes, S.n_words, c0, c1, acc);
        const int key0 = (c0 + col) * 32 + r;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int j = key0 + 4 * m;
            if (c0 + col < c1 && j < S.n) {
                const unsigned long long v = composite(order_key(score_of(acc[0], m, bias)), (uint32_t)j);
                if ((v >> shift) >= lim) {
                    const unsigned slot = atomicAdd(&ss.nsel, 1u);
                    if (slot < (unsigned)k) sel[slot] = v;
                }
            }
        }
    }
    __syncthreads();   // every selected composite has been written
    emit_sorted_by_index(sel, k, b.kpad, S.out_idx + (size_t)qq * k, S.out_score + (size_t)qq * k);
}

// ---------------------------------------------------------------- final
// One CTA per query: exact top-k of the candidates when k <= count <= cap,
// written in ascending key index.  Shared memory: the selected k (kMaxFastK
// composites), then the candidates, later reused to put the k in index order.
template <int NS, bool kBlocked>
__global__ void __launch_bounds__(kSelThreads) final_kernel(const __grid_constant__ Batch<NS> b)
{
    extern __shared__ unsigned long long dyn[];
    __shared__ SelShared ss;
    const int gq = blockIdx.x;
    const int si = find_session_by_query(b, gq);
    const SessionDesc &S = b.s[si];
    const int qq = gq - S.q_begin;
    const uint32_t *st = S.qstate + qq * kQueryStateWords;
    const unsigned cnt = st[1];
    const int k = b.k;
    if (st[2] || cnt < (unsigned)k || cnt > (unsigned)b.cap) {
        exact_query<NS, kBlocked>(b, S, qq);   // the exact path, in this CTA
        return;
    }
    unsigned long long *sel = dyn;                  // [kMaxFastK]
    unsigned long long *x = dyn + kMaxFastK;        // [cap] candidates, then the emit scratch
    const unsigned long long *cq = S.cand + (size_t)qq * b.cap;
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    // 16-byte loads, kLoadDepth in flight per thread before any is used
    constexpr int kLoadDepth = 4;
    for (unsigned i0 = 2 * threadIdx.x; i0 < cnt; i0 += 2 * kSelThreads * kLoadDepth) {
        ulonglong2 p[kLoadDepth];
#pragma unroll
        for (int u = 0; u < kLoadDepth; ++u) {
            const unsigned i = i0 + u * 2 * kSelThreads;
            p[u] = make_ulonglong2(0ull, 0ull);
            if (i + 1 < cnt) p[u] = *reinterpret_cast<const ulonglong2 *>(cq + i);
            else if (i < cnt) p[u].x = cq[i];
        }
#pragma unroll
        for (int u = 0; u < kLoadDepth; ++u) {
            const unsigned i = i0 + u * 2 * kSelThreads;
            if (i < cnt) {
                x[i] = p[u].x;
                lo = min(lo, (uint32_t)(p[u].x >> 32));
                hi = max(hi, (uint32_t)(p[u].x >> 32));
            }
            if (i + 1 < cnt) {
                x[i + 1] = p[u].y;
                lo = min(lo, (uint32_t)(p[u].y >> 32));
                hi = max(hi, (uint32_t)(p[u].y >> 32));
            }
        }
    }
    sel_range(ss, lo, hi);
    const unsigned long long base = (unsigned long long)ss.lo << 32;
    const int top = 32 + bit_length(ss.hi - ss.lo);
    sel_run(ss, cnt, (unsigned)k, top, 0, [&](unsigned i) { return x[i] - base; });
    // compact exactly the k selected in any order (the emit sorts them by
    // key index): one shared-memory reservation per warp and round
    const int cut = ss.cut;
    const unsigned long long lim = ss.prefix >> cut;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) ss.above = 0u;   // the selected count so far
    __syncthreads();
    for (unsigned r0 = 0; r0 < cnt; r0 += kSelThreads) {
        const unsigned i = r0 + threadIdx.x;
        const unsigned long long v = (i < cnt) ? x[i] : 0ull;
        const bool take = i < cnt && ((v - base) >> cut) >= lim;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, take);
        if (m) {
            const int leader = __ffs(m) - 1;
            unsigned at = 0;
            if (lane == leader) at = atomicAdd(&ss.above, (unsigned)__popc(m));
            at = __shfl_sync(0xFFFFFFFFu, at, leader);
            const unsigned pos = at + (unsigned)__popc(m & ((1u << lane) - 1u));
            if (take && pos < (unsigned)k) sel[pos] = v;
        }
    }
    __syncthreads();
    emit_by_buckets(sel, k, S.n, x, ss, S.out_idx + (size_t)qq * k, S.out_score + (size_t)qq * k);
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
// m ~ 128*n/(2k) clamped to [4096, 8192] and to a quarter of the tiles;
// theta is the r-th largest sampled key, r = ceil(f*k*m/n) with f = 2 (or 3
// when f = 2 would give r < 128), so about f*k keys pass the filter.  The
// count of passing keys has a relative spread of about 1/sqrt(r): at one
// million keys and k = 2048, m = 8192 gives r = 48 at f = 3, so falling
// below k (the exact path) is a 4.6-sigma event and passing the
// capacity of 6k a 7-sigma one, while the sampled pass reads a quarter of
// what 32768 keys cost (B200: 50 -> 17 us per plan on that layer).
Sizing size_session(int n, int n_words, int k, int block_keys)
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
    // Grouped scales shift every block's scores by its own unread-channel
    // constant, so a sample of few blocks misplaces theta and sends queries
    // to the exact path; at least kBlockedSampleTiles tiles (from as many
    // blocks) keep it on the fast path.
    if (block_keys) mt = std::max(mt, kBlockedSampleTiles);
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
    size_t qstate, cand, tables, bias_blk, total;
};

// Query heads per KV head rounded up to the kernels' template width.
inline int gp_for(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }
inline size_t head_table_bytes(int G)
{
    switch (gp_for(G)) {
    case 1: return sizeof(ScanMeta<1>);
    case 2: return sizeof(ScanMeta<2>);
    case 4: return sizeof(ScanMeta<4>);
    default: return sizeof(ScanMeta<8>);
    }
}

inline bool host_resident(const fathom_index &ix) { return ix.residency == FATHOM_RES_HOST_MAPPED; }

WsLayout layout_session(const fathom_index &ix, int k, size_t at)
{
    const int Q = ix.n_kv_heads * ix.group;
    const int cap = capacity_for(std::min(k, kMaxFastK));
    WsLayout L{};
    L.qstate = at;
    at += align256((size_t)Q * kQueryStateWords * sizeof(uint32_t));
    L.cand = at;
    at += align256((size_t)Q * cap * sizeof(unsigned long long));
    L.tables = at;
    at += align256((size_t)ix.n_kv_heads * head_table_bytes(ix.group));
    L.bias_blk = at;   // grouped scales: a bias per (KV head, block, query head)
    if (ix.block_keys)
        at += align256((size_t)ix.n_kv_heads * index_blocks(ix) * ix.group * sizeof(float));
    L.total = at;
    return L;
}

// Multiprocessors of the current device (cached per device).
inline int sm_count()
{
    static int cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Raise a kernel's dynamic shared-memory limit to its largest possible need,
// once per device.  `done` must belong to that kernel alone.
template <class Kernel>
cudaError_t ensure_smem(int (&done)[64], Kernel kernel, size_t max_bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!done[dev]) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)max_bytes);
        if (e != cudaSuccess) return e;
        done[dev] = 1;
    }
    return cudaSuccess;
}

// One set of "limit raised" flags per kernel instantiation.
template <int NS>
struct SmemFlags {
    static int final_[64];
};
template <int NS> int SmemFlags<NS>::final_[64];

constexpr size_t kStageBytes = (size_t)kStageRows * kTileCols * sizeof(uint32_t);

// Record a timing event; inside a stream capture it must be an external
// record to stay a timing record in the graph (the flag is invalid outside).
inline void record_timing_event(cudaEvent_t ev, cudaStream_t stream)
{
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, stream);
}

template <int NS, int GP, bool kBlocked>
cudaError_t run_batch(const Batch<NS> &bt, int total_chunks, int total_queries, int total_heads,
                      int total_blocks, int max_m_keys, uint32_t flags, cudaStream_t stream,
                      ScanProfileHook *hook)
{
    cudaError_t e;
    const bool force = (flags & FATHOM_SCAN_FORCE_EXACT) != 0;
    int launches = 0;
    {
        // per-head tables, sampled scores and theta per query (or the
        // exact-path flags)
        static int threshold_smem_set[64];
        auto kern = threshold_kernel<NS, GP, kBlocked>;
        const size_t dyn = kThetaBufs * kThetaStageBytes + (size_t)max_m_keys * sizeof(uint32_t);
        if ((e = ensure_smem(threshold_smem_set, kern,
                             kThetaBufs * kThetaStageBytes +
                                 (size_t)kSampleMaxKeys * sizeof(uint32_t))) !=
            cudaSuccess)
            return note_error(e, "threshold set-up");
        // one CTA per query, then (unless the exact path is forced) one per
        // KV head building its tables, then with grouped scales one per
        // (KV head, block) writing its biases (the scan and the exact path
        // read them)
        const int table_ctas = force ? 0 : total_heads;
        const int ctas = total_queries + table_ctas + (kBlocked ? total_blocks : 0);
        kern<<<ctas, kSelThreads, dyn, stream>>>(bt, force ? 1u : 0u, total_queries, table_ctas);
        if ((e = cudaGetLastError()) != cudaSuccess) return note_error(e, "threshold launch");
        ++launches;
    }
    if (!force && total_chunks > 0) {
        const bool timed = hook && hook->enabled;
        static int main_smem_set[64];
        auto kern = scan_kernel<NS, GP, kMainStages, kBlocked>;
        const size_t dyn = kMainStages * kStageBytes;
        if ((e = ensure_smem(main_smem_set, kern, dyn)) != cudaSuccess) return note_error(e, "scan set-up");
        if (timed) record_timing_event(hook->begin, stream);
        kern<<<total_chunks, kScanThreads, dyn, stream>>>(bt);
        if ((e = cudaGetLastError()) != cudaSuccess) return note_error(e, "scan launch");
        if (timed) {
            record_timing_event(hook->end, stream);
            hook->recorded = true;
        }
        ++launches;
    }
    // the fast path's selected k and candidates, or the exact path's stages
    // and its k selected, whichever is larger
    const size_t exact_smem = kMainStages * kStageBytes + (size_t)bt.kpad * sizeof(unsigned long long);
    const size_t final_smem =
        std::max((kMaxFastK + (size_t)bt.cap) * sizeof(unsigned long long), exact_smem);
    static int final_smem_set[64];
    if ((e = ensure_smem(final_smem_set, final_kernel<NS, kBlocked>,
                         std::max((kMaxFastK + (size_t)capacity_for(kMaxFastK)) *
                                      sizeof(unsigned long long),
                                  kMainStages * kStageBytes +
                                      (size_t)kMaxK * sizeof(unsigned long long)))) != cudaSuccess)
        return note_error(e, "final set-up");
    final_kernel<NS, kBlocked><<<total_queries, kSelThreads, final_smem, stream>>>(bt);
    launches += 1;
    note_launch(launches);
    if ((e = cudaGetLastError()) != cudaSuccess) return note_error(e, "final launch");
    return cudaSuccess;
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
    int groups = 0, queries = 0, heads = 0, blocks = 0, max_m = 0;
    size_t at = 0;
    char *base = static_cast<char *>(ws);
    for (int s = 0; s < n_sessions; ++s) {
        const fathom_index &ix = *ss[s].ix;
        const Sizing z = size_session(ix.n_keys, ix.n_words, k, ix.block_keys);
        const WsLayout L = layout_session(ix, k, at);
        at = L.total;
        SessionDesc &D = bt.s[s];
        D.planes = ix.planes;   // device rows (a host-resident index arrives as ring-slot views)
        D.mn = ix.mn;
        D.scale = ix.scale;
        D.q = ss[s].q;
        D.t = ss[s].t;
        D.tu = ss[s].t_union;
        D.out_idx = ss[s].out_idx;
        D.out_score = ss[s].out_score;
        D.qstate = reinterpret_cast<uint32_t *>(base + L.qstate);
        D.cand = reinterpret_cast<unsigned long long *>(base + L.cand);
        D.tables = reinterpret_cast<unsigned char *>(base + L.tables);
        D.bias_blk = reinterpret_cast<float *>(base + L.bias_blk);
        D.block_words = ix.block_keys / 32;
        D.nb = index_blocks(ix);
        D.n_filled = ix.block_keys ? ceil_div(ix.n_keys, ix.block_keys) : 1;
        D.blk_begin = blocks;
        if (ix.block_keys) blocks += ix.n_kv_heads * D.n_filled;
        D.H = ix.n_kv_heads;
        D.n = ix.n_keys;
        D.n_words = ix.n_words;
        D.n_cols = z.n_cols;
        D.col_groups = z.n_cols / 4;
        D.m_tiles = z.m_tiles;
        D.sample_stride = z.stride;
        D.m_keys = z.m_keys;
        D.sample_rank = z.rank;
        D.exact_only = z.exact_only;
        D.chunks = (D.col_groups + kTileGroups - 1) / kTileGroups;   // chunks of <= 64 words
        if (ix.block_keys)   // the same number of chunks in every scale block
            D.chunks = D.n_filled * ceil_div(D.block_words / 4, kTileGroups);
        D.q_begin = queries;
        D.head_begin = heads;
        heads += ix.n_kv_heads;
        groups += D.H * D.chunks;
        queries += D.H * bt.G;
        max_m = std::max(max_m, z.m_keys);
    }
    // Below one wave of CTA slots, cut the heads into more, equal chunks (at
    // least kMinChunkGroups groups each) so the grid fills the slots evenly;
    // a chunk never spans two heads.
    const int slots = sm_count() * ((bt.G > 4) ? 2 : 4);
    if (groups < slots) {
        const double grow = (double)slots / (double)groups;
        groups = 0;
        for (int s = 0; s < n_sessions; ++s) {
            SessionDesc &D = bt.s[s];
            if (D.block_words) {
                const int per = D.chunks / D.n_filled;
                const int most = std::max(1, (D.block_words / 4) / kMinChunkGroups);
                D.chunks = D.n_filled * std::max(per, std::min(most, (int)(per * grow)));
            } else {
                const int most = std::max(1, D.col_groups / kMinChunkGroups);
                D.chunks = std::max(D.chunks, std::min(most, (int)(D.chunks * grow)));
            }
            groups += D.H * D.chunks;
        }
    }
    groups = 0;
    for (int s = 0; s < n_sessions; ++s) {
        SessionDesc &D = bt.s[s];
        D.chunk_begin = groups;
        D.chunk_q = D.col_groups / D.chunks;
        D.chunk_rem = D.col_groups - D.chunk_q * D.chunks;
        groups += D.H * D.chunks;
    }
    const int G = bt.G;
    if (blocks > 0) {   // every session has grouped scales (the C ABI checks)
        if (G <= 1) return run_batch<NS, 1, true>(bt, groups, queries, heads, blocks, max_m, flags, stream, hook);
        if (G <= 2) return run_batch<NS, 2, true>(bt, groups, queries, heads, blocks, max_m, flags, stream, hook);
        if (G <= 4) return run_batch<NS, 4, true>(bt, groups, queries, heads, blocks, max_m, flags, stream, hook);
        return run_batch<NS, 8, true>(bt, groups, queries, heads, blocks, max_m, flags, stream, hook);
    }
    if (G <= 1) return run_batch<NS, 1, false>(bt, groups, queries, heads, 0, max_m, flags, stream, hook);
    if (G <= 2) return run_batch<NS, 2, false>(bt, groups, queries, heads, 0, max_m, flags, stream, hook);
    if (G <= 4) return run_batch<NS, 4, false>(bt, groups, queries, heads, 0, max_m, flags, stream, hook);
    return run_batch<NS, 8, false>(bt, groups, queries, heads, 0, max_m, flags,
                                   stream, hook);
}


// ------------------------------------------------- host-resident indices
// A scan over host-resident planes is pipelined over units of KV heads (one
// head per unit for a single session, one session per unit for a batch): the
// union planes of unit u + 1 cross the host link into one slot of a two-slot
// device ring while unit u is scored from the other slot, so only the last
// unit's scoring adds to the link time, and the device holds two units'
// planes instead of the whole index.  The fetches run on a side stream that
// forks from the caller's stream and joins it again before the call returns
// (event waits only, so the sequence can be captured in a CUDA graph).
struct HostUnit {
    int s, h0, nh;   // session, first KV head, KV heads
};

inline bool any_host(const fathom_index *sessions, int n)
{
    for (int s = 0; s < n; ++s)
        if (host_resident(sessions[s])) return true;
    return false;
}

std::vector<HostUnit> host_units(const fathom_index *sessions, int n)
{
    std::vector<HostUnit> u;
    for (int s = 0; s < n; ++s) {
        if (n == 1)
            for (int h = 0; h < sessions[s].n_kv_heads; ++h) u.push_back(HostUnit{s, h, 1});
        else
            u.push_back(HostUnit{s, 0, sessions[s].n_kv_heads});
    }
    return u;
}

// Heads h0 .. h0+nh-1 of an index as a device-resident index of nh heads
// whose planes start at `planes` (a ring slot, or the index's own rows).
fathom_index unit_view(const fathom_index &ix, int h0, int nh, uint32_t *planes)
{
    fathom_index v = ix;
    const size_t stat = (size_t)h0 * index_blocks(ix) * ix.head_dim;
    v.n_kv_heads = nh;
    v.residency = FATHOM_RES_DEVICE;
    v.planes = planes;
    v.mn = ix.mn + stat;
    v.scale = ix.scale + stat;
    v.sigma2 = ix.sigma2 ? ix.sigma2 + (size_t)h0 * ix.head_dim : nullptr;
    v.sum_code = ix.sum_code ? ix.sum_code + stat : nullptr;
    v.sum_code2 = ix.sum_code2 ? ix.sum_code2 + stat : nullptr;
    return v;
}

inline size_t head_plane_bytes(const fathom_index &ix)
{
    return (size_t)ix.head_dim * kBits * (size_t)ix.n_words * sizeof(uint32_t);
}

struct HostLayout {
    size_t unit_ws;      // scratch of one unit's scan (reused by every unit)
    size_t slot_bytes;   // one ring slot
    size_t total;
};

HostLayout host_layout(const fathom_index *sessions, int n, int k)
{
    HostLayout L{};
    for (const HostUnit &u : host_units(sessions, n)) {
        const fathom_index &ix = sessions[u.s];
        const fathom_index v = unit_view(ix, u.h0, u.nh, nullptr);
        L.unit_ws = std::max(L.unit_ws, layout_session(v, k, 0).total);
        if (host_resident(ix)) L.slot_bytes = std::max(L.slot_bytes, u.nh * head_plane_bytes(ix));
    }
    L.unit_ws = align256(L.unit_ws);
    L.slot_bytes = align256(L.slot_bytes);
    L.total = L.unit_ws + 2 * L.slot_bytes;
    return L;
}

// The side stream and events of the pipelined path, one set per (device,
// caller stream), created on first use and kept for the process.
struct SideContext {
    cudaStream_t side;
    cudaEvent_t fork, join, fetched[2], done[2];
};

cudaError_t side_context(cudaStream_t stream, SideContext **out)
{
    static std::mutex mu;
    static std::map<std::pair<int, cudaStream_t>, SideContext> contexts;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = contexts.find({dev, stream});
    if (it == contexts.end()) {
        SideContext c{};
        if ((e = cudaStreamCreateWithFlags(&c.side, cudaStreamNonBlocking)) != cudaSuccess) return e;
        cudaEvent_t *evs[] = {&c.fork, &c.join, &c.fetched[0], &c.fetched[1], &c.done[0], &c.done[1]};
        for (int i = 0; i < 6; ++i) {
            if ((e = cudaEventCreateWithFlags(evs[i], cudaEventDisableTiming)) != cudaSuccess) {
                for (int j = 0; j < i; ++j) cudaEventDestroy(*evs[j]);   // nothing half-made stays
                cudaStreamDestroy(c.side);
                return e;
            }
        }
        it = contexts.emplace(std::make_pair(dev, stream), c).first;
    }
    *out = &it->second;
    return cudaSuccess;
}

// The units of a pipelined scan, enqueued after the fork; the first error
// stops the enqueueing (the caller joins the side stream either way).
cudaError_t enqueue_units(const ScanSessionArgs *ss, const std::vector<fathom_index> &ix,
                          const std::vector<HostUnit> &units, const HostLayout &L, int k,
                          void *ws, uint32_t flags, cudaStream_t stream, SideContext *c,
                          ScanProfileHook *hook)
{
    char *base = static_cast<char *>(ws);
    cudaError_t e;
    const bool timed = hook && hook->enabled;
    if (timed) record_timing_event(hook->begin, c->side);
    for (size_t u = 0; u < units.size(); ++u) {
        const HostUnit &U = units[u];
        const ScanSessionArgs &a = ss[U.s];
        const fathom_index &x = ix[U.s];
        const int d = x.head_dim, G = x.group;
        const size_t row0 = (size_t)U.h0 * d * kBits * (size_t)x.n_words;
        uint32_t *planes = x.planes + row0;
        if (host_resident(x)) {
            uint32_t *slot = reinterpret_cast<uint32_t *>(base + L.unit_ws + (u % 2) * L.slot_bytes);
            if (u >= 2 && (e = cudaStreamWaitEvent(c->side, c->done[u % 2], 0)) != cudaSuccess)
                return note_error(e, "ring wait");
            const FetchJob job{planes, slot, a.t_union + (size_t)U.h0 * d, U.nh * d, x.n_words};
            if ((e = launch_fetch(&job, 1, c->side, kFetchCtasPerSmShared)) != cudaSuccess)
                return note_error(e, "fetch launch");
            if ((e = cudaEventRecord(c->fetched[u % 2], c->side)) != cudaSuccess)
                return note_error(e, "fetch event");
            if ((e = cudaStreamWaitEvent(stream, c->fetched[u % 2], 0)) != cudaSuccess)
                return note_error(e, "fetch wait");
            planes = slot;
        }
        const fathom_index v = unit_view(x, U.h0, U.nh, planes);
        const size_t qo = (size_t)U.h0 * G;
        const ScanSessionArgs ua{&v, a.q + qo * d, a.t + qo * d, a.t_union + (size_t)U.h0 * d,
                                 a.out_idx + qo * k, a.out_score + qo * k};
        if ((e = build_and_run<1>(&ua, 1, k, ws, flags & ~FATHOM_SCAN_PROFILE, stream, nullptr)) !=
            cudaSuccess)
            return e;
        if ((e = cudaEventRecord(c->done[u % 2], stream)) != cudaSuccess)
            return note_error(e, "done event");
    }
    if (timed) {
        record_timing_event(hook->end, c->side);
        hook->recorded = true;
    }
    return cudaSuccess;
}

cudaError_t run_host_pipelined(const ScanSessionArgs *ss, int n_sessions, int k, void *ws,
                               uint32_t flags, cudaStream_t stream, ScanProfileHook *hook)
{
    std::vector<fathom_index> ix(n_sessions);
    for (int s = 0; s < n_sessions; ++s) ix[s] = *ss[s].ix;
    const HostLayout L = host_layout(ix.data(), n_sessions, k);
    const std::vector<HostUnit> units = host_units(ix.data(), n_sessions);
    SideContext *c = nullptr;
    cudaError_t e = side_context(stream, &c);
    if (e != cudaSuccess) return note_error(e, "side stream set-up");
    if ((e = cudaEventRecord(c->fork, stream)) != cudaSuccess) return note_error(e, "fork");
    if ((e = cudaStreamWaitEvent(c->side, c->fork, 0)) != cudaSuccess) return note_error(e, "fork");
    e = enqueue_units(ss, ix, units, L, k, ws, flags, stream, c, hook);
    // join whatever was enqueued on the side stream, also after an error, so
    // the caller's stream (and a capture in progress) waits for all of it
    cudaError_t j = cudaEventRecord(c->join, c->side);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(stream, c->join, 0);
    if (j != cudaSuccess) note_error(j, "join");
    return e != cudaSuccess ? e : j;
}

}  // namespace

size_t scan_workspace_bytes(const fathom_index *sessions, int n_sessions, int k)
{
    if (any_host(sessions, n_sessions)) return host_layout(sessions, n_sessions, k).total;
    size_t at = 0;
    for (int s = 0; s < n_sessions; ++s) at = layout_session(sessions[s], k, at).total;
    return at;
}

cudaError_t launch_scan(const ScanSessionArgs *sessions, int n_sessions, int k, void *ws,
                        size_t ws_bytes, uint32_t flags, cudaStream_t stream,
                        ScanProfileHook *hook)
{
    (void)ws_bytes;
    std::vector<fathom_index> ix(n_sessions);
    for (int s = 0; s < n_sessions; ++s) ix[s] = *sessions[s].ix;
    if (any_host(ix.data(), n_sessions))
        return run_host_pipelined(sessions, n_sessions, k, ws, flags, stream, hook);
    if (n_sessions == 1) return build_and_run<1>(sessions, 1, k, ws, flags, stream, hook);
    return build_and_run<kMaxSessions>(sessions, n_sessions, k, ws, flags, stream, hook);
}

}  // namespace fathom
