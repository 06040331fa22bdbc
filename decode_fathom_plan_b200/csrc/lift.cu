// The 8-plane index as nibble channels for the scan.
//
// Source: Fathom explainer (papers.ananclaw.com, arXiv 2609.17652),
// 部署前必读 item 3 (an 8-bit upstream K cache needs the bit-plane index
// adapted to 8 planes) and 核心方法 / 读侧 (a channel read at t planes is
// rebuilt at the middle of its coarse t-bit bin).
//
// Channel c of an 8-plane index stores slots 0-7 = bits 7..0 of its code,
// which in the layout [H][d][8][n_words] are exactly two 4-slot channels
// 2c (bits 7..4, the high nibble hi) and 2c+1 (bits 3..0, the low nibble
// lo) of a 4-plane layout [H][2d][4][n_words].  With code = 16*hi + lo,
//   mn + scale*code = (mn + 16*scale*hi) + (0 + scale*lo),
// and reading t planes of the 8-bit code reads min(t,4) planes of hi and
// max(t-4,0) of lo.  The 8-bit bin middle is the sum of the two nibble bin
// middles: for t <= 4, 16*(2^(4-t)*u + (2^(4-t)-1)/2) + 7.5
// = 2^(8-t)*u + (2^(8-t)-1)/2, and for t > 4 the high nibble is exact.  So
// the 4-plane scan over 2d nibble channels with
//   mn'  = (mn_c, 0),  scale' = (16*scale_c, scale_c),
//   q'   = (q_c, q_c), t' = (min(t,4), max(t-4,0))   [likewise the union]
// scores every key exactly as the 8-plane definition does (16*scale is a
// power-of-two multiple, so W' = q*scale' is the same product scaled).
// This kernel writes those primed arrays; the planes are not touched.  With
// grouped per-token-block scales, mn and scale have a row per (head, block)
// and are lifted row by row the same way.
#include "common.cuh"
#include "internal.h"

namespace fathom {
namespace {

__global__ void __launch_bounds__(256)
lift_kernel(LiftArgs a)
{
    const int total = max(max(a.Q, a.H), a.stat_rows) * a.d;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
        if (i < a.Q * a.d) {   // query row i / d, channel i % d -> nibble channels 2i, 2i+1
            const uint16_t qv = a.q[i];
            const int t = min((int)a.t[i], 8);
            a.q2[2 * i] = qv;
            a.q2[2 * i + 1] = qv;
            a.t2[2 * i] = (uint8_t)min(t, 4);
            a.t2[2 * i + 1] = (uint8_t)max(t - 4, 0);
        }
        if (i < a.stat_rows * a.d) {
            const float sc = a.scale[i];
            a.mn2[2 * i] = a.mn[i];
            a.mn2[2 * i + 1] = 0.0f;
            a.scale2[2 * i] = __fmul_rn(16.0f, sc);
            a.scale2[2 * i + 1] = sc;
        }
        if (i < a.H * a.d) {
            const int tu = min((int)a.tu[i], 8);
            a.tu2[2 * i] = (uint8_t)min(tu, 4);
            a.tu2[2 * i + 1] = (uint8_t)max(tu - 4, 0);
        }
    }
}

}  // namespace

size_t lift_bytes(int H, int Q, int d, int stat_rows)
{
    auto a16 = [](size_t b) { return (b + 15) & ~(size_t)15; };
    const size_t d2 = 2 * (size_t)d;
    return 2 * a16((size_t)stat_rows * d2 * sizeof(float)) +
           a16((size_t)Q * d2 * sizeof(uint16_t)) + a16((size_t)Q * d2) + a16((size_t)H * d2);
}

void lift_carve(void *ws, int H, int Q, int d, int stat_rows, LiftArgs *a)
{
    auto a16 = [](size_t b) { return (b + 15) & ~(size_t)15; };
    const size_t d2 = 2 * (size_t)d;
    unsigned char *p = static_cast<unsigned char *>(ws);
    a->mn2 = reinterpret_cast<float *>(p);
    p += a16((size_t)stat_rows * d2 * sizeof(float));
    a->scale2 = reinterpret_cast<float *>(p);
    p += a16((size_t)stat_rows * d2 * sizeof(float));
    a->q2 = reinterpret_cast<uint16_t *>(p);
    p += a16((size_t)Q * d2 * sizeof(uint16_t));
    a->t2 = p;
    p += a16((size_t)Q * d2);
    a->tu2 = p;
    a->H = H;
    a->Q = Q;
    a->d = d;
    a->stat_rows = stat_rows;
}

cudaError_t launch_lift(const LiftArgs &a, cudaStream_t stream)
{
    const int rows = a.Q > a.H ? a.Q : a.H;
    const int total = (rows > a.stat_rows ? rows : a.stat_rows) * a.d;
    const int block = 256;
    const int grid = (total + block - 1) / block;
    lift_kernel<<<grid, block, 0, stream>>>(a);
    note_launch(1);
    return cudaGetLastError();
}

}  // namespace fathom
