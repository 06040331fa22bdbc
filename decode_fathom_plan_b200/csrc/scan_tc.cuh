// Filtering pass of the Fathom scan with the union-channel sum on the
// 5th-generation tensor cores (tcgen05.mma kind::i8, accumulators in TMEM).
// Included by scan.cu inside its anonymous namespace, after the session and
// batch descriptors and the CUDA-core scan kernel.
//
// Source: Fathom explainer (papers.ananclaw.com), 核心方法: query head g
// reads the t_gc most significant planes of channel c and scores the key
// rebuilt from that t_gc-bit quantiser, s_gj = bias_g + sum_c W_gc v_gcj with
// v_gcj = code_cj with its low 4 - t_gc bits cleared (the decomposition at the
// top of scan.cu).
//
// Matrix form.  A KV head reads the union plan T_c = max_g t_gc once; a_cj is
// the code rebuilt from those T_c planes (bits below them zero).  A query
// reading 0 < t < T_c planes needs a_cj - (a_cj & low(t)), low(t) = 2^(4-t)-1,
// so with one A column per union channel (a_c) and one per (channel, partial
// depth present) (a_c & low(t)):
//   sum_c W_gc v_gcj = sum_cols A_j,col * B_col,g,
// B = W_gc on the channel's column for every query reading it, -W_gc on the
// column of the query's own partial depth.  That is an [n x C] x [C x G]
// product with C = union channels + partial columns (about 60-90 on the
// Qwen3-8B-shaped plans): M = keys, N = query heads, K = columns.
//
// Exact integer arithmetic.  A is a 4-bit code, exact in int8.  Each query's
// weights are scaled by a power of two 2^(29-e_g), 2^e_g > max_c |W_gc|, and
// rounded to integers X (|X| <= 2^29, error <= 2^-30 of 2^e_g per weight),
// written as four signed base-256 digits D0..D3 (D0 in [-32, 32], the rest in
// [-128, 127]); the MMA sums A*D exactly in s32 (|sum| < 2^21), one N column
// per (query, digit), N = 16 for up to 4 query heads.  The score is
// bias_g + 2^(e_g-29) * (((S0*256 + S1)*256 + S2)*256 + S3) in fp32.
//
// Data path per CTA (256 threads, a chunk of up to 32 plane words = 1024 keys
// of one KV head, 8 M-tiles of 128 keys):
//   * stages of 8 union channels x their live plane rows x the chunk's words
//     arrive by 16-byte cp.async, 3 buffers deep (rows past a channel's depth
//     are never copied or read: the channel's warp knows its depth);
//   * warp w builds the columns of the stage's channel w: lane l owns plane
//     word l (32 keys); 4 shared loads, a 4x4 bit transpose per nibble column
//     by delta swaps (20 logic ops) gives each key's 4-bit code, two masks split
//     the codes of the 32 keys into 32 bytes, stored as two 16-byte rows of
//     the A tile (keys contiguous: MN-major, no swizzle);
//   * one thread issues, for every K-block of 32 columns complete, 8 MMAs
//     (128 keys x 16 x 32 each) into 8 TMEM accumulators and commits them to
//     the K-block buffer's mbarrier; A is double-buffered per K-block, and a
//     stage waits (bounded) for the MMAs that read a buffer before rewriting it;
//   * after the last K-block each warp reads 4 accumulator tiles of its TMEM
//     lane quarter (tcgen05.ld), forms the scores of 4 keys x G query heads,
//     and appends the keys scoring >= theta as the CUDA-core kernel does.
// Every wait has a limit; a CTA whose wait runs out flags its queries for the
// exact path (the final kernel then redoes them from the planes), waits with
// a limit for its MMAs in flight and frees its TMEM before it returns.
#pragma once

constexpr int kTcWords = 32;                        // plane words per CTA
constexpr int kTcTiles = kTcWords / 4;              // M-tiles of 128 keys
constexpr int kTcMaxGroup = 4;                      // query heads per KV head
constexpr int kTcN = 4 * kTcMaxGroup;               // (query head, digit) columns
constexpr int kTcCols = kBits * kMaxHeadDim;        // A columns per head, at most
constexpr int kTcMaxKBlocks = kTcCols / 32;
constexpr int kTcKBlockB = kTcN * 32;               // bytes of B per K-block
// A tile (128 keys x 32 columns, int8, keys contiguous): 16-key rows
// kTcRowStride apart, 8-column groups kTcGroupStride apart, tiles
// kTcTileStride apart; all three are 16 bytes past a multiple of 128, so the
// 8 lanes of a quarter-warp storing 16 bytes each reach 8 different bank groups.
constexpr int kTcRowStride = 144;
constexpr int kTcGroupStride = 1152;
constexpr int kTcTileStride = 4624;
constexpr int kTcABytes = kTcTiles * kTcTileStride;          // one K-block buffer
constexpr int kTcStageBytes = kStageRows * kTcWords * 4;     // 4 KB
constexpr int kTcTmemCols = kTcTiles * kTcN;                 // 128
constexpr int kTcMinGroups = 4;                               // smallest chunk: 16 words
constexpr unsigned long long kTcWaitNs = 500000000ull;        // limit of every wait
// Instruction descriptor: s32 accumulate, A and B s8, A MN-major, B K-major,
// N = 16, M = 128.
constexpr uint32_t kTcIdesc = (2u << 4) | (1u << 7) | (1u << 10) | (1u << 15) |
                              ((uint32_t)(kTcN >> 3) << 17) | ((128u >> 4) << 24);

struct alignas(16) TcChan {
    uint32_t row;        // plane row of slot 0: (h*d + c)*4
    uint16_t col;        // first A column of the channel
    uint8_t T;           // planes read (union depth)
    uint8_t ncols;       // 1 + partial columns
    uint8_t low[3];      // low(t) of each partial column
    uint8_t pad[5];
};
struct alignas(16) TcHead {
    float bias[kTcMaxGroup];
    float unit[kTcMaxGroup];   // 2^(e_g - 29)
    int U, n_stages, C, n_kblocks;
};
// Per-head tables of the tensor-core scan, built once per (session, KV head)
// by the threshold launch; a scanning CTA copies the header, the first U
// channel records and the first n_kblocks K-blocks of B.
struct alignas(16) TcMeta {
    TcHead hd;
    TcChan ch[kMaxHeadDim];
    int8_t B[kTcMaxKBlocks][kTcKBlockB];   // per K-block: K-major, no swizzle
};

// Byte of B for (column k of a K-block, N column n): 8 N rows x 16 K bytes per
// core matrix, the two K halves 128 bytes apart, the two N halves 256 apart.
__device__ __forceinline__ int tc_b_offset(int n, int k)
{
    return (n & 7) * 16 + (n >> 3) * 256 + (k & 15) + (k >> 4) * 128;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for the phase of the given parity to complete; false after kTcWaitNs.
__device__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity)
{
    if (mbar_test(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_test(bar, parity))
        if (global_ns() - t0 > kTcWaitNs) return false;
    return true;
}
// Shared-memory matrix descriptor, no swizzle: start, leading byte offset
// (stride of core matrices along K), stride byte offset (along M or N),
// descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kTcIdesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void proxy_fence_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(addr));
}
// Exact int -> float for |x| < 2^22: x under the mantissa of 1.5 * 2^23.
__device__ __forceinline__ float small_int_to_float(uint32_t x)
{
    return __uint_as_float(x + 0x4B400000u) - 12582912.0f;
}

// ------------------------------------------------------------ head tables
// Tensor-core tables of KV head h from its CUDA-core tables `sm` (built by
// setup_head in shared memory): channel records with their A columns, B in
// digits, and per query the bias and the unit 2^(e_g-29).  All kSelThreads
// threads of the threshold launch's table CTA call it.
template <int GP>
__device__ void build_tc_table(const ScanMeta<GP> &sm, int G, TcMeta *out, SelShared &ss)
{
    static_assert(GP <= kTcMaxGroup, "tensor-core tables hold up to 4 query heads");
    __shared__ unsigned wmax[kTcMaxGroup];
    __shared__ unsigned s_total;
    const int U = sm.U;
    const int u = threadIdx.x;
    if (u < kTcMaxGroup) wmax[u] = 0u;
    int T = 0, ncols = 0;
    uint8_t low[3] = {0, 0, 0}, ldep[3] = {0, 0, 0};
    if (u < U) {
#pragma unroll
        for (int s = 0; s < kBits; ++s) T += sm.row_g[u * kBits + s] != 0xFFFFFFFFu;
        unsigned depths = 0u;
#pragma unroll
        for (int g = 0; g < GP; ++g) {
            const int t = (g < G) ? (int)sm.tq[u][g] : 0;
            if (t > 0 && t < T) depths |= 1u << t;
        }
        ncols = 1;
#pragma unroll
        for (int t = 1; t < kBits; ++t)
            if (depths & (1u << t)) {
                low[ncols - 1] = (uint8_t)((1u << (kBits - t)) - 1u);
                ldep[ncols - 1] = (uint8_t)t;
                ++ncols;
            }
    }
    __syncthreads();   // wmax cleared
    if (u < U) {
#pragma unroll
        for (int g = 0; g < GP; ++g)
            if (g < G && sm.tq[u][g] > 0) atomicMax(&wmax[g], __float_as_uint(fabsf(sm.Wp[u][g])));
    }
    unsigned total = 0;
    const unsigned col0 = block_exclusive_scan((unsigned)ncols, ss.wsum, &total);
    if (threadIdx.x == 0) s_total = total;
    __syncthreads();   // wmax complete, s_total set
    const int C = (int)s_total;
    const int nkb = (C + 31) / 32;
    int e[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
        const float m = __uint_as_float(wmax[g]);
        int ex = 0;
        if (m > 0.0f && isfinite(m)) frexpf(m, &ex);   // m < 2^ex
        e[g] = ex;
    }
    // B: zero every K-block in use, then each channel writes its columns
    uint4 *bz = reinterpret_cast<uint4 *>(&out->B[0][0]);
    for (int i = threadIdx.x; i < nkb * (kTcKBlockB / 16); i += blockDim.x)
        bz[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    if (u < U) {
        int X[GP];
#pragma unroll
        for (int g = 0; g < GP; ++g) {
            const bool reads = g < G && sm.tq[u][g] > 0;
            X[g] = reads ? __float2int_rn(ldexpf(sm.Wp[u][g], 29 - e[g])) : 0;
        }
        for (int j = 0; j < ncols; ++j) {
            const int col = (int)col0 + j;
            int8_t *Bk = out->B[col >> 5];
            const int k = col & 31;
#pragma unroll
            for (int g = 0; g < GP; ++g) {
                int x = 0;
                if (j == 0) x = X[g];
                else if (g < G && (int)sm.tq[u][g] == (int)ldep[j - 1]) x = -X[g];
                // four signed base-256 digits, most significant first
                int dg[4];
#pragma unroll
                for (int i = 3; i > 0; --i) {
                    dg[i] = ((x + 128) & 255) - 128;
                    x = (x - dg[i]) >> 8;
                }
                dg[0] = x;
#pragma unroll
                for (int i = 0; i < 4; ++i) Bk[tc_b_offset(4 * g + i, k)] = (int8_t)dg[i];
            }
        }
        TcChan rec;
        rec.row = sm.row_g[u * kBits];
        rec.col = (uint16_t)col0;
        rec.T = (uint8_t)T;
        rec.ncols = (uint8_t)ncols;
#pragma unroll
        for (int i = 0; i < 3; ++i) rec.low[i] = low[i];
#pragma unroll
        for (int i = 0; i < 5; ++i) rec.pad[i] = 0;
        out->ch[u] = rec;
    }
    if (threadIdx.x == 0) {
        TcHead hd;
#pragma unroll
        for (int g = 0; g < kTcMaxGroup; ++g) {
            hd.bias[g] = (g < GP && g < G) ? sm.bias[g] : 0.0f;
            hd.unit[g] = (g < GP && g < G) ? ldexpf(1.0f, e[g < GP ? g : 0] - 29) : 0.0f;
        }
        hd.U = U;
        hd.n_stages = (U + kStageChannels - 1) / kStageChannels;
        hd.C = C;
        hd.n_kblocks = nkb;
        out->hd = hd;
    }
}

// ------------------------------------------------------------ scan kernel
// Dynamic shared memory of scan_tc_kernel for head dimension d: two A
// buffers, the stage buffers, B and the channel records.
inline size_t tc_smem_bytes(int d)
{
    const int kb = (kBits * d + 31) / 32;
    return 2 * (size_t)kTcABytes + kStages * (size_t)kTcStageBytes + (size_t)kb * kTcKBlockB +
           (size_t)d * sizeof(TcChan);
}

// Copy stage st (8 channels x live plane rows x the chunk's words) into
// buffer buf: thread (row = tid/8, piece = tid%8) copies 16 bytes.
__device__ __forceinline__ void tc_load_stage(uint32_t *stage, const TcChan *ch, int U, int st,
                                              int buf, const uint32_t *planes, int n_words,
                                              int col_lo, int col_hi)
{
    const int row = threadIdx.x >> 3, piece = threadIdx.x & 7;
    const int u = st * kStageChannels + (row >> 2), p = row & 3;
    const int col = col_lo + piece * 4;
    if (u < U && col < col_hi) {
        const TcChan cc = ch[u];
        if (p < cc.T)
            cp_async16_full(stage + (size_t)buf * (kStageRows * kTcWords) + row * kTcWords + piece * 4,
                            planes + (size_t)(cc.row + p) * (size_t)n_words + col);
    }
}

// The A columns of one union channel for the lane's plane word (32 keys).
// rows: the channel's 4 stage rows (32 words each); A: the K-block buffers.
__device__ __forceinline__ void tc_columns(const TcChan &cc, const uint32_t *rows, int lane,
                                           unsigned char *A)
{
    const int T = cc.T;
    const uint32_t x0 = rows[lane];
    const uint32_t x1 = (T > 1) ? rows[kTcWords + lane] : 0u;
    const uint32_t x2 = (T > 2) ? rows[2 * kTcWords + lane] : 0u;
    const uint32_t x3 = (T > 3) ? rows[3 * kTcWords + lane] : 0u;
    // slot s holds code bit 3-s: y_r = plane of code bit r
    uint32_t y0 = x3, y1 = x2, y2 = x1, y3 = x0, t;
    // transpose each 4x4 block (words x nibble bits) by delta swaps:
    // afterwards nibble i of y_r is the code of key 4i + r
    t = ((y0 >> 1) ^ y1) & 0x55555555u; y1 ^= t; y0 ^= t << 1;
    t = ((y2 >> 1) ^ y3) & 0x55555555u; y3 ^= t; y2 ^= t << 1;
    t = ((y0 >> 2) ^ y2) & 0x33333333u; y2 ^= t; y0 ^= t << 2;
    t = ((y1 >> 2) ^ y3) & 0x33333333u; y3 ^= t; y1 ^= t << 2;
    // byte b of lo_r: key 8b + r; of hi_r: key 8b + 4 + r
    const uint4 lo = make_uint4(y0 & 0x0F0F0F0Fu, y1 & 0x0F0F0F0Fu, y2 & 0x0F0F0F0Fu, y3 & 0x0F0F0F0Fu);
    const uint4 hi = make_uint4((y0 >> 4) & 0x0F0F0F0Fu, (y1 >> 4) & 0x0F0F0F0Fu,
                                (y2 >> 4) & 0x0F0F0F0Fu, (y3 >> 4) & 0x0F0F0F0Fu);
    const int at = (lane >> 2) * kTcTileStride + 2 * (lane & 3) * kTcRowStride;
    for (int j = 0; j < (int)cc.ncols; ++j) {
        const int col = (int)cc.col + j;
        const int kb = col >> 5, k = col & 31;
        unsigned char *p = A + (kb & 1) * kTcABytes + at + (k >> 3) * kTcGroupStride + (k & 7) * 16;
        uint4 a = lo, b2 = hi;
        if (j > 0) {
            const uint32_t m = (uint32_t)cc.low[j - 1] * 0x01010101u;
            a = make_uint4(lo.x & m, lo.y & m, lo.z & m, lo.w & m);
            b2 = make_uint4(hi.x & m, hi.y & m, hi.z & m, hi.w & m);
        }
        *reinterpret_cast<uint4 *>(p) = a;
        *reinterpret_cast<uint4 *>(p + kTcRowStride) = b2;
    }
}

// MMAs of K-blocks [from, to) into the 8 tile accumulators, each K-block
// committed to its A buffer's mbarrier.  One thread.
__device__ __forceinline__ void tc_issue(int from, int to, uint32_t tmem, const unsigned char *A,
                                         const int8_t *Bs, const unsigned long long *bar)
{
    for (int kb = from; kb < to; ++kb) {
        const uint32_t a0 = smem_addr(A + (kb & 1) * kTcABytes);
        const uint64_t bdesc = umma_desc(smem_addr(Bs + kb * kTcKBlockB), 128, 256);
#pragma unroll
        for (int t = 0; t < kTcTiles; ++t)
            umma_i8(tmem + (uint32_t)(t * kTcN),
                    umma_desc(a0 + (uint32_t)(t * kTcTileStride), kTcGroupStride, kTcRowStride), bdesc,
                    kb > 0 ? 1u : 0u);
        umma_commit(smem_addr(&bar[kb & 1]));
    }
}

// Key (within the word) held by TMEM lane i of a warp's quarter: lanes 0..15
// are the lo bytes, 16..31 the hi bytes of the word's lane (see tc_columns).
__device__ __forceinline__ int tc_key_in_word(int i)
{
    const int p = i & 15;
    return 8 * (p & 3) + (p >> 2) + ((i >> 4) << 2);
}

template <int NS>
__global__ void __launch_bounds__(kScanThreads, 2) scan_tc_kernel(const __grid_constant__ Batch<NS> b)
{
    extern __shared__ __align__(1024) unsigned char tc_dyn[];
    __shared__ TcHead hd;
    __shared__ float s_theta_f[kTcMaxGroup];
    __shared__ __align__(8) unsigned long long bar[3];
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail, s_issued;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = b.d;
    unsigned char *A = tc_dyn;
    uint32_t *stage = reinterpret_cast<uint32_t *>(tc_dyn + 2 * kTcABytes);
    int8_t *Bs = reinterpret_cast<int8_t *>(tc_dyn + 2 * kTcABytes + kStages * kTcStageBytes);
    TcChan *ch = reinterpret_cast<TcChan *>(Bs + ((kBits * d + 31) / 32) * kTcKBlockB);

    // this CTA's chunk: chunk c of the KV head's S.chunks equal parts
    const int si = find_session_by_chunk(b, (int)blockIdx.x);
    const SessionDesc &S = b.s[si];
    const int local = (int)blockIdx.x - S.chunk_begin;
    const int h = local / S.chunks;
    const int c = local - h * S.chunks;
    const int g0 = c * S.chunk_q + min(c, S.chunk_rem);
    const int g1 = g0 + S.chunk_q + (c < S.chunk_rem ? 1 : 0);
    const int col_lo = g0 * 4;
    const int width = (g1 - g0) * 4;   // at most kTcWords
    const int col_hi = min(S.n_cols, col_lo + width);
    const int G = b.G;
    const int q0 = h * G;
    const TcMeta *tm = reinterpret_cast<const TcMeta *>(S.tables) + h;
    if (tid < kTcMaxGroup) {
        const uint32_t theta =
            (tid < G) ? S.qstate[(q0 + tid) * kQueryStateWords + 0] : 0xFFFFFFFFu;
        s_theta_f[tid] = theta == 0u ? -INFINITY : order_key_to_float(theta);
    }
    if (tid < (int)(sizeof(TcHead) / 4))
        reinterpret_cast<uint32_t *>(&hd)[tid] = reinterpret_cast<const uint32_t *>(&tm->hd)[tid];
    if (tid == 0) {
        mbar_init(smem_addr(&bar[0]));
        mbar_init(smem_addr(&bar[1]));
        mbar_init(smem_addr(&bar[2]));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_fail = 0;
        s_issued = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&s_tmem)),
                     "r"(kTcTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const int U = hd.U, n_stages = hd.n_stages, C = hd.C, nkb = hd.n_kblocks;
    // B and the channel records, then the first two stages
    {
        const uint4 *srcB = reinterpret_cast<const uint4 *>(&tm->B[0][0]);
        for (int i = tid; i < nkb * (kTcKBlockB / 16); i += kScanThreads)
            cp_async16_full(Bs + 16 * i, srcB + i);
        for (int i = tid; i < U; i += kScanThreads) cp_async16_full(ch + i, tm->ch + i);
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
    }
    const uint32_t *planes = S.planes;
    const int n_words = S.n_words;
#pragma unroll
    for (int st = 0; st < kStages - 1; ++st) {
        if (st < n_stages) tc_load_stage(stage, ch, U, st, st, planes, n_words, col_lo, col_hi);
        cp_async_commit();
    }
    int issued = 0;   // K-blocks issued (thread 0)
    int ready = 1;    // K-blocks whose A buffer is free to write (0 and 1 from the start)
    for (int st = 0; st < n_stages; ++st) {
        cp_async_wait<kStages - 2>();
        proxy_fence_smem();   // this thread's A stores of the last stage, for the MMAs
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (s_fail) break;
        const int u0 = st * kStageChannels;
        const int done = ch[u0].col;   // columns of the stages before this one
        if (tid == 0 && issued < done / 32) {
            tc_issue(issued, done / 32, tmem, A, Bs, bar);
            issued = done / 32;
        }
        const int nx = st + kStages - 1;
        if (nx < n_stages) tc_load_stage(stage, ch, U, nx, nx % kStages, planes, n_words, col_lo, col_hi);
        cp_async_commit();
        // the stage's columns may reach one K-block past the free ones: wait
        // for the MMAs that read that buffer two K-blocks ago
        const int end = (u0 + kStageChannels < U) ? (int)ch[u0 + kStageChannels].col : C;
        const int need = (end - 1) >> 5;
        bool ok = true;
        while (ready < need && ok) {
            ++ready;
            ok = mbar_wait_bounded(smem_addr(&bar[ready & 1]), (uint32_t)(((ready - 2) >> 1) & 1));
        }
        if (!ok) s_fail = 1;
        const int u = u0 + warp;
        if (ok && u < U)
            tc_columns(ch[u], stage + (size_t)(st % kStages) * (kStageRows * kTcWords) +
                                  warp * kBits * kTcWords,
                       lane, A);
    }
    cp_async_wait<0>();
    proxy_fence_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        if (!s_fail && issued < nkb) {
            tc_issue(issued, nkb, tmem, A, Bs, bar);
            issued = nkb;
        }
        if (issued > 0) umma_commit(smem_addr(&bar[2]));
        s_issued = issued;
    }
    __syncthreads();
    bool ok = !s_fail;
    if (s_issued > 0 && !mbar_wait_bounded(smem_addr(&bar[2]), 0u)) ok = false;
    tc_fence_after();
    // accumulators of the warp's 4 tiles: TMEM lanes 32*qd .. +31
    const int qd = warp & 3;
    uint32_t r[4][16];
    if (ok && nkb > 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            tmem_ld16(tmem + ((uint32_t)(32 * qd) << 16) + (uint32_t)(((warp >> 2) + 2 * j) * kTcN), r[j]);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int i = 0; i < 16; ++i) r[j][i] = 0u;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTcTmemCols)
                     : "memory");
    }
    if (!__syncthreads_and(ok ? 1 : 0)) {
        // a wait ran out: this head's queries take the exact path
        if (tid < G) atomicExch(&S.qstate[(q0 + tid) * kQueryStateWords + 2], 1u);
        return;
    }

    // scores of the thread's 4 keys (one per tile) and the append of those
    // scoring >= theta, with one reservation per warp and query
    int key[4];
    bool live[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int w = 4 * ((warp >> 2) + 2 * j) + qd;   // plane word within the chunk
        key[j] = (col_lo + w) * 32 + tc_key_in_word(lane);
        live[j] = w < width && col_lo + w < col_hi && key[j] < S.n;
    }
#pragma unroll
    for (int g = 0; g < kTcMaxGroup; ++g) {
        if (g >= G) break;
        const float bias = hd.bias[g], unit = hd.unit[g], th = s_theta_f[g];
        float sc[4];
        unsigned pass = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float f = small_int_to_float(r[j][4 * g]);
            f = fmaf(f, 256.0f, small_int_to_float(r[j][4 * g + 1]));
            f = fmaf(f, 256.0f, small_int_to_float(r[j][4 * g + 2]));
            f = fmaf(f, 256.0f, small_int_to_float(r[j][4 * g + 3]));
            sc[j] = fmaf(unit, f, bias);
            if (live[j] && sc[j] >= th) pass |= 1u << j;
        }
        if (!__any_sync(0xFFFFFFFFu, pass != 0u)) continue;
        const int cnt = __popc(pass);
        int inc = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, inc, off);
            if (lane >= off) inc += y;
        }
        unsigned at = 0;
        if (lane == 31 && inc) at = atomicAdd(&S.qstate[(q0 + g) * kQueryStateWords + 1], (unsigned)inc);
        at = __shfl_sync(0xFFFFFFFFu, at, 31);
        unsigned pos = at + (unsigned)(inc - cnt);
        unsigned long long *cq = S.cand + (size_t)(q0 + g) * b.cap;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (pass & (1u << j)) {
                if (pos < (unsigned)b.cap) cq[pos] = composite(order_key(sc[j]), (uint32_t)key[j]);
                ++pos;
            }
        }
    }
}
