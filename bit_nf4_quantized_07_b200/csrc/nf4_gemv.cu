// Fused NF4 doubleDequant + forward for decode-sized token counts (n <= 32).
// HBM-bound: the 4-bit weight is streamed once and W' lives only in registers.
//
// Method: "LoRA 与 QLoRA" section QLoRA 1 (4-bit weight -> dequant -> BF16 ->
// GEMM) and section LoRA (y = W0 x + s B(A x)); jjjymmm.cn "QLoRA"
// (doubleDequant: restore the block constant, then the weight).
//
//   Y[t][o] = sum_k X[t][k] W'[o][k] + sum_j sU[t][j] B[o][j],   t < n <= 32
//
// A CTA owns 32 weight rows (two 16-row MMA tiles) over all K; its 8 warps
// split K into 8 ranges and fold their partial tiles through shared memory.
// Codes are decoded straight into the register layout of the m16n8k16 A
// operand: within each 64-wide block, lane (g, c) owns code bytes 8c..8c+7 of
// rows g and g+8, and MMA step s uses bytes 8c+2s (k pair "2c", "2c+1") and
// 8c+2s+1 (pair "2c+8", "2c+9").  The activations are read with the same
// permutation of k, so every product still pairs equal k.  Per code byte a
// shared 256-entry table gives (c[hi], c[lo]); the products with the restored
// block constant are fp32 multiplies rounded once to BF16, exactly
// w' = bf16_RN(fp32(ahat * c[q])).
#include "qln_common.cuh"
#include "qln_internal.h"

namespace qln {

constexpr int kGvRows = 32;     // weight rows per CTA
constexpr int kGvWarps = 8;     // K splits per CTA

template <int NT>  // token tiles of 8: n <= 8 * NT
__global__ void __launch_bounds__(kGvWarps * 32) nf4_gemv_kernel(const uint8_t *__restrict__ codes,
                                                                  const float *__restrict__ absmax,
                                                                  const int8_t *__restrict__ qabs,
                                                                  const float *__restrict__ dq_scale,
                                                                  const float *__restrict__ dq_mean, int64_t rows,
                                                                  int64_t cols, const uint16_t *__restrict__ X,
                                                                  int n, const uint16_t *__restrict__ sU,
                                                                  const uint16_t *__restrict__ B, int r,
                                                                  uint16_t *__restrict__ Y) {
    __shared__ float2 pair_tab[256];
    __shared__ float red[kGvWarps][kGvRows][8 * NT];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    for (int i = tid; i < 256; i += blockDim.x) pair_tab[i] = make_float2(nf4_value(i >> 4), nf4_value(i & 15));
    __syncthreads();

    const int64_t m0 = (int64_t)blockIdx.x * kGvRows;
    const int64_t bpr = cols / 64;          // blocks per row
    const int64_t kb0 = (bpr * warp) / kGvWarps, kb1 = (bpr * (warp + 1)) / kGvWarps;
    const float mu = qabs ? __ldg(dq_mean) : 0.f;
    // the 4 weight rows of this lane: tile mt, half h -> row m0 + 16 mt + g + 8 h
    int64_t rowoff[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) rowoff[i] = m0 + 16 * (i >> 1) + g + 8 * (i & 1);

    float acc[2][NT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;

    // One block of operands, fetched one block ahead of its use.
    struct Blk {
        uint2 cw[4];
        float v[4];     // DQ scale (or plain absmax) of the 4 rows
        int32_t q[4];   // DQ codes of the 4 rows
        uint4 xa[NT], xb[NT];
    };
    auto fetch = [&](int64_t kb, Blk &o) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o.cw[i] = __ldcs(reinterpret_cast<const uint2 *>(codes + rowoff[i] * (cols / 2) + kb * 32 + 8 * c));
            const int64_t jb = rowoff[i] * bpr + kb;
            if (qabs) {
                o.q[i] = __ldg(qabs + jb);
                o.v[i] = __ldg(dq_scale + (jb >> 8));
            } else {
                o.q[i] = 0;
                o.v[i] = __ldg(absmax + jb);
            }
        }
        // activations: token 8 nt + g, k = 64 kb + 16 c .. 16 c + 15
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int t = 8 * nt + g;
            if (t < n) {
                const uint4 *xp = reinterpret_cast<const uint4 *>(X + (int64_t)t * cols + kb * 64 + 16 * c);
                o.xa[nt] = __ldg(xp);
                o.xb[nt] = __ldg(xp + 1);
            } else {
                o.xa[nt] = make_uint4(0u, 0u, 0u, 0u);
                o.xb[nt] = o.xa[nt];
            }
        }
    };
    Blk cur, nxt;
    if (kb0 < kb1) fetch(kb0, cur);
    for (int64_t kb = kb0; kb < kb1; ++kb) {
        if (kb + 1 < kb1) fetch(kb + 1, nxt);
        float ah[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) ah[i] = qabs ? dq_restore((int8_t)cur.q[i], cur.v[i], mu) : cur.v[i];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            // A fragments of both row tiles: bytes 8c + 2s and 8c + 2s + 1
            uint32_t a[2][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t w32 = (s < 2) ? cur.cw[i].x : cur.cw[i].y;
                const int sh = 16 * (s & 1);
                const float2 p0 = pair_tab[(w32 >> sh) & 0xffu];
                const float2 p1 = pair_tab[(w32 >> (sh + 8)) & 0xffu];
                const uint32_t v0 = pack_bf16x2(__fmul_rn(ah[i], p0.x), __fmul_rn(ah[i], p0.y));
                const uint32_t v1 = pack_bf16x2(__fmul_rn(ah[i], p1.x), __fmul_rn(ah[i], p1.y));
                const int mt = i >> 1, h = i & 1;
                a[mt][h] = v0;      // (row g or g+8, k pair "2c")
                a[mt][2 + h] = v1;  // (row g or g+8, k pair "2c+8")
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                // k = 16 c + 4 s .. 16 c + 4 s + 3 of this block, matching bytes 8c+2s, 8c+2s+1
                const uint4 xv = (s < 2) ? cur.xa[nt] : cur.xb[nt];
                const uint32_t b[2] = {(s & 1) ? xv.z : xv.x, (s & 1) ? xv.w : xv.y};
                mma_bf16_16816(acc[0][nt], a[0], b);
                mma_bf16_16816(acc[1][nt], a[1], b);
            }
        }
        cur = nxt;
    }

    // Fold the 8 K-range partials.
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) red[warp][16 * mt + g + 8 * (e >> 1)][8 * nt + 2 * c + (e & 1)] = acc[mt][nt][e];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int row = 16 * mt + g + 8 * (e >> 1), col = 8 * nt + 2 * c + (e & 1);
                    float v = 0.f;
#pragma unroll
                    for (int w = 0; w < kGvWarps; ++w) v = __fadd_rn(v, red[w][row][col]);
                    acc[mt][nt][e] = v;
                }
        // Adapter term: rows of B (K = j contiguous) times s*U (K = j contiguous).
        for (int j0 = 0; j0 < r; j0 += 16) {
            uint32_t a[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int64_t row = m0 + 16 * mt + g + 8 * (q & 1);
                    const int j = j0 + 2 * c + 8 * (q >> 1);
                    a[mt][q] = (j < r) ? *reinterpret_cast<const uint32_t *>(B + row * r + j) : 0u;
                }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int t = 8 * nt + g;
                uint32_t b[2];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int j = j0 + 2 * c + 8 * q;
                    b[q] = (t < n && j < r) ? *reinterpret_cast<const uint32_t *>(sU + (int64_t)t * r + j) : 0u;
                }
                mma_bf16_16816(acc[0][nt], a[0], b);
                mma_bf16_16816(acc[1][nt], a[1], b);
            }
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = 8 * nt + 2 * c + (e & 1);
                    const int64_t row = m0 + 16 * mt + g + 8 * (e >> 1);
                    if (t < n) Y[(int64_t)t * rows + row] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[mt][nt][e]));
                }
    }
}

bool nf4_gemv_supported(const qln_nf4_weight *w, int64_t n, int r) {
    return n >= 1 && n <= 32 && (w->rows % kGvRows) == 0 && (w->cols % 64) == 0 && (r % 8) == 0;
}

cudaError_t launch_nf4_gemv(const qln_nf4_weight *w, const uint16_t *X, int64_t n, const uint16_t *sU,
                            const uint16_t *B, int r, uint16_t *Y, cudaStream_t st) {
    const dim3 grid((unsigned)(w->rows / kGvRows));
    const int nt = (int)((n + 7) / 8);
#define QLN_GEMV(NTV)                                                                                              \
    nf4_gemv_kernel<NTV><<<grid, kGvWarps * 32, 0, st>>>(w->codes, w->absmax, w->qabs, w->dq_scale, w->dq_mean, \
                                                         w->rows, w->cols, X, (int)n, sU, B, r, Y)
    switch (nt) {
        case 1: QLN_GEMV(1); break;
        case 2: QLN_GEMV(2); break;
        case 3: QLN_GEMV(3); break;
        default: QLN_GEMV(4); break;
    }
#undef QLN_GEMV
    note_launch();
    return cudaGetLastError();
}

}  // namespace qln
