// Fused QLoRA forward for decode-sized token counts (n <= 32), one launch.
// HBM-bound: the 4-bit weight is streamed once and W' lives only in registers.
//
// Method: "LoRA 与 QLoRA" section QLoRA 1 (4-bit weight -> dequant -> BF16 ->
// GEMM) and section LoRA (y = W0 x + s B(A x), A x formed first);
// jjjymmm.cn "QLoRA" (doubleDequant: restore the block constant, then the
// weight).
//
//   U = X A^T                                   (n x r, fp32 accumulate)
//   Y[t][o] = sum_k X[t][k] W'[o][k] + sum_j bf16(s U)[t][j] B[o][j]
//
// A cooperative grid of CTAs, each owning 32 weight rows over all K:
//   1. CTAs 0..7 also form U over one eighth of K each and publish the fp32
//      partial with a release increment of a counter in the workspace.
//   2. Every CTA streams its rows: all code bytes of a warp's K range are
//      requested up front (cp.async into shared memory), the block constants
//      and activations one block ahead in registers.  Codes are decoded
//      straight into the register layout of the m16n8k16 A operand: in each
//      64-wide block, lane (g, c) owns code bytes 8c..8c+7 of rows g and g+8,
//      and MMA step s uses bytes 8c+2s (k pair "2c", "2c+1") and 8c+2s+1
//      (pair "2c+8", "2c+9"); the activations are read with the same
//      permutation of k, so every product still pairs equal k.  A shared
//      256-entry table gives (c[hi], c[lo]) per code byte; the products with
//      the restored constant are fp32 multiplies rounded once to BF16, i.e.
//      w' = bf16_RN(fp32(ahat * c[q])).
//   3. The 8 K-range partials are folded through shared memory; after a
//      bounded wait for the 8 U partials (co-residency is guaranteed by the
//      cooperative launch) the adapter term is one more MMA pass.
// A wait that gives up writes QLN_ERR_TIMEOUT to the status word.
#include "qln_common.cuh"
#include "qln_internal.h"

namespace qln {

constexpr int kGvRows = 32;      // weight rows per CTA
constexpr int kGvWarps = 8;      // K ranges per CTA
constexpr int kGvUParts = 8;     // CTAs that form U
constexpr int kGvMaxBlk = 8;     // 64-wide blocks per warp (cols <= 4096 per 8 warps x 8)
constexpr uint64_t kGvWaitNs = 1000000000ull;

struct GvParams {
    const uint8_t *codes;
    const float *absmax;
    const int8_t *qabs;
    const float *dq_scale;
    const float *dq_mean;
    int64_t rows, cols;
    const uint16_t *X;
    int n;
    const uint16_t *A;   // [r][cols]
    const uint16_t *B;   // [rows][r]
    int r;
    float s;
    uint16_t *Y;         // [n][rows]
    uint16_t *U_out;     // [n][r] or null
    float *upart;        // [kGvUParts][n][r]
    int *counter;        // zeroed before the launch
    int *status;
};

__device__ __forceinline__ uint64_t gv_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

template <int NT>  // token tiles of 8: n <= 8 * NT
__global__ void __launch_bounds__(kGvWarps * 32) nf4_decode_fwd_kernel(const GvParams p) {
    extern __shared__ __align__(16) uint8_t gsm[];
    constexpr int kRedCols = 8 * NT > 16 ? 8 * NT : 16;
    float2 *pair_tab = reinterpret_cast<float2 *>(gsm);                        // 256 entries
    float *red = reinterpret_cast<float *>(gsm + 256 * sizeof(float2));       // [8][32][kRedCols]
    uint16_t *su = reinterpret_cast<uint16_t *>(red + kGvWarps * kGvRows * kRedCols);  // [8*NT][r] bf16(s U)
    volatile int *uflag = reinterpret_cast<volatile int *>(su + 8 * NT * 128);  // 16-byte slot
    uint8_t *cst = reinterpret_cast<uint8_t *>(su + 8 * NT * 128) + 16;          // codes, per warp 8 KB
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int n = p.n, r = p.r;
    const int64_t cols = p.cols;
    const int64_t bpr = cols / 64;
    const int64_t kb0 = (bpr * warp) / kGvWarps, kb1 = (bpr * (warp + 1)) / kGvWarps;
    const int nblk = (int)(kb1 - kb0);

    uint8_t *wst = cst + warp * (kGvMaxBlk * 1024);
    // per block: 32 rows x 32 bytes = 64 chunks of 16 bytes, 2 per lane
    auto request_codes = [&](int64_t m0) {
        for (int b = 0; b < nblk; ++b) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int idx = lane + 32 * h, row = idx >> 1, half = idx & 1;
                cp_async16(wst + b * 1024 + row * 32 + half * 16,
                           p.codes + (m0 + row) * (cols / 2) + (kb0 + b) * 32 + half * 16);
            }
        }
        cp_async_commit();
    };
    const int64_t ngroups = p.rows / kGvRows;
    // ---- 1. request every code byte of this warp's K range of the first group -
    if ((int64_t)blockIdx.x < ngroups) request_codes((int64_t)blockIdx.x * kGvRows);
    for (int i = tid; i < 256; i += blockDim.x) pair_tab[i] = make_float2(nf4_value(i >> 4), nf4_value(i & 15));

    // ---- 2. U partial (CTAs 0..7): U_b = X[:, K_b] A[:, K_b]^T ----------------
    if (blockIdx.x < kGvUParts) {
        const int64_t k0 = (cols * blockIdx.x) / kGvUParts, k1 = (cols * (blockIdx.x + 1)) / kGvUParts;
        const int64_t ks0 = k0 + ((k1 - k0) / 16 * warp) / kGvWarps * 16;
        const int64_t ks1 = k0 + ((k1 - k0) / 16 * (warp + 1)) / kGvWarps * 16;
        // M = tokens (2 tiles of 16), N = 64 adapter columns at a time (8 tiles of 8), K steps of 16
        for (int jc = 0; jc < r; jc += 64) {
            float ua[2][8][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int jt = 0; jt < 8; ++jt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) ua[mt][jt][e] = 0.f;
            for (int64_t k = ks0; k < ks1; k += 16) {
                uint32_t a[2][4];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int t = 16 * mt + g + 8 * (q & 1);
                        const int64_t kk = k + 2 * c + 8 * (q >> 1);
                        a[mt][q] = (t < n) ? __ldg(reinterpret_cast<const uint32_t *>(p.X + (int64_t)t * cols + kk)) : 0u;
                    }
#pragma unroll
                for (int jt = 0; jt < 8; ++jt) {
                    if (jc + 8 * jt < r) {
                        const int j = jc + 8 * jt + g;
                        uint32_t b[2];
#pragma unroll
                        for (int q = 0; q < 2; ++q)
                            b[q] = __ldg(reinterpret_cast<const uint32_t *>(p.A + (int64_t)j * cols + k + 2 * c + 8 * q));
                        mma_bf16_16816(ua[0][jt], a[0], b);
                        if (n > 16) mma_bf16_16816(ua[1][jt], a[1], b);
                    }
                }
            }
            // fold the 8 warps, 16 adapter columns per pass
#pragma unroll
            for (int jp = 0; jp < 4; ++jp) {
                const int j0 = jc + 16 * jp;
                if (j0 >= r) break;
                __syncthreads();
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            red[(warp * 32 + 16 * mt + g + 8 * (e >> 1)) * kRedCols + 8 * jj + 2 * c + (e & 1)] =
                                ua[mt][2 * jp + jj][e];
                __syncthreads();
                for (int idx = tid; idx < 32 * 16; idx += blockDim.x) {
                    const int t = idx >> 4, j = j0 + (idx & 15);
                    if (t < n && j < r) {
                        float v = 0.f;
#pragma unroll
                        for (int w = 0; w < kGvWarps; ++w) v = __fadd_rn(v, red[(w * 32 + t) * kRedCols + (idx & 15)]);
                        p.upart[((int64_t)blockIdx.x * n + t) * r + j] = v;
                    }
                }
            }
        }
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            atomicAdd(p.counter, 1);
        }
    }
    __syncthreads();

    // ---- 3./4. per row group: weight stream, fold, adapter term, store --------
    const float mu = p.qabs ? __ldg(p.dq_mean) : 0.f;
    bool first = true;
    bool uok = false;
    for (int64_t rg = blockIdx.x; rg < ngroups; rg += gridDim.x) {
        const int64_t m0 = rg * kGvRows;
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

        struct Side {        // constants and activations of one block
            float v[4];      // DQ scale (or plain absmax) of the 4 rows
            int32_t q[4];    // DQ codes of the 4 rows
            uint4 xa[NT], xb[NT];
        };
        auto fetch = [&](int64_t kb, Side &o) {
    #pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int64_t jb = rowoff[i] * bpr + kb;
                if (p.qabs) {
                    o.q[i] = __ldg(p.qabs + jb);
                    o.v[i] = __ldg(p.dq_scale + (jb >> 8));
                } else {
                    o.q[i] = 0;
                    o.v[i] = __ldg(p.absmax + jb);
                }
            }
    #pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int t = 8 * nt + g;
                if (t < n) {
                    const uint4 *xp = reinterpret_cast<const uint4 *>(p.X + (int64_t)t * cols + kb * 64 + 16 * c);
                    o.xa[nt] = __ldg(xp);
                    o.xb[nt] = __ldg(xp + 1);
                } else {
                    o.xa[nt] = make_uint4(0u, 0u, 0u, 0u);
                    o.xb[nt] = o.xa[nt];
                }
            }
        };
        Side cur, nxt;
        if (nblk > 0) fetch(kb0, cur);
        cp_async_wait<0>();
        __syncwarp();
        for (int b = 0; b < nblk; ++b) {
            if (b + 1 < nblk) fetch(kb0 + b + 1, nxt);
            float ah[4];
            uint2 cw[4];
    #pragma unroll
            for (int i = 0; i < 4; ++i) {
                ah[i] = p.qabs ? dq_restore((int8_t)cur.q[i], cur.v[i], mu) : cur.v[i];
                const int row = 16 * (i >> 1) + g + 8 * (i & 1);
                cw[i] = *reinterpret_cast<const uint2 *>(wst + b * 1024 + row * 32 + 8 * c);
            }
    #pragma unroll
            for (int s = 0; s < 4; ++s) {
                uint32_t a[2][4];
    #pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t w32 = (s < 2) ? cw[i].x : cw[i].y;
                    const int sh = 16 * (s & 1);
                    const float2 p0 = pair_tab[(w32 >> sh) & 0xffu];
                    const float2 p1 = pair_tab[(w32 >> (sh + 8)) & 0xffu];
                    const int mt = i >> 1, h = i & 1;
                    a[mt][h] = pack_bf16x2(__fmul_rn(ah[i], p0.x), __fmul_rn(ah[i], p0.y));      // k pair "2c"
                    a[mt][2 + h] = pack_bf16x2(__fmul_rn(ah[i], p1.x), __fmul_rn(ah[i], p1.y));  // k pair "2c+8"
                }
    #pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint4 xv = (s < 2) ? cur.xa[nt] : cur.xb[nt];
                    const uint32_t bb[2] = {(s & 1) ? xv.z : xv.x, (s & 1) ? xv.w : xv.y};
                    mma_bf16_16816(acc[0][nt], a[0], bb);
                    mma_bf16_16816(acc[1][nt], a[1], bb);
                }
            }
            cur = nxt;
        }

        // ---- 4. fold the K ranges, wait for U, adapter term, store ----------------
    #pragma unroll
        for (int mt = 0; mt < 2; ++mt)
    #pragma unroll
            for (int nt = 0; nt < NT; ++nt)
    #pragma unroll
                for (int e = 0; e < 4; ++e)
                    red[(warp * kGvRows + 16 * mt + g + 8 * (e >> 1)) * kRedCols + 8 * nt + 2 * c + (e & 1)] = acc[mt][nt][e];
        if (first && tid == 0) {
            bool ok = false;
            const uint64_t t0 = gv_timer_ns();
            for (uint32_t it = 0;; ++it) {
                int v;
                asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p.counter) : "memory");
                if (v >= kGvUParts) {
                    ok = true;
                    break;
                }
                if ((it & 63u) == 0u && gv_timer_ns() - t0 > kGvWaitNs) break;
            }
            if (!ok) atomicExch(p.status, (int)QLN_ERR_TIMEOUT);
            *uflag = ok ? 1 : 0;
        }
        __syncthreads();
        if (first) uok = *uflag != 0;
        // s*U for this CTA's tokens: fixed-order sum of the 8 partials (once)
        for (int idx = tid; first && idx < 8 * NT * r; idx += blockDim.x) {
            const int t = idx / r, j = idx % r;
            float v = 0.f;
            if (uok && t < n)
                for (int b = 0; b < kGvUParts; ++b) v = __fadd_rn(v, __ldcg(p.upart + ((int64_t)b * n + t) * r + j));
            su[t * r + j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(p.s, v)));
            if (blockIdx.x == 0 && p.U_out && t < n) p.U_out[t * r + j] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        }
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
                        for (int w = 0; w < kGvWarps; ++w) v = __fadd_rn(v, red[(w * kGvRows + row) * kRedCols + col]);
                        acc[mt][nt][e] = v;
                    }
            for (int j0 = 0; j0 < r; j0 += 16) {
                uint32_t a[2][4];
    #pragma unroll
                for (int mt = 0; mt < 2; ++mt)
    #pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int64_t row = m0 + 16 * mt + g + 8 * (q & 1);
                        const int j = j0 + 2 * c + 8 * (q >> 1);
                        a[mt][q] = (j < r) ? __ldg(reinterpret_cast<const uint32_t *>(p.B + row * r + j)) : 0u;
                    }
    #pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int t = 8 * nt + g;
                    uint32_t b[2];
    #pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int j = j0 + 2 * c + 8 * q;
                        b[q] = (j < r) ? *reinterpret_cast<const uint32_t *>(su + t * r + j) : 0u;
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
                        if (t < n) p.Y[(int64_t)t * p.rows + row] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[mt][nt][e]));
                    }
        }

        // next group: its code bytes go into the same per-warp buffer
        __syncthreads();
        if (rg + gridDim.x < ngroups) request_codes((rg + gridDim.x) * kGvRows);
        first = false;
    }
}

static size_t gv_smem_bytes(int nt) {
    const size_t red_cols = 8 * nt > 16 ? 8 * nt : 16;
    return 256 * sizeof(float2) + (size_t)kGvWarps * kGvRows * red_cols * sizeof(float) +
           (size_t)8 * nt * 128 * sizeof(uint16_t) + 16 + (size_t)kGvWarps * kGvMaxBlk * 1024;
}

bool nf4_gemv_supported(const qln_nf4_weight *w, int64_t n, int r) {
    const int64_t bpr = w->cols / 64;
    return n >= 1 && n <= 32 && (w->rows % kGvRows) == 0 && (w->cols % 64) == 0 && bpr >= kGvWarps &&
           bpr <= (int64_t)kGvWarps * kGvMaxBlk && (w->cols / kGvUParts) % 16 == 0 && (r % 8) == 0 && r <= 128 &&
           (w->rows / kGvRows) >= kGvUParts;
}

size_t nf4_gemv_upart_bytes(int64_t n, int r) { return (size_t)kGvUParts * (size_t)n * (size_t)r * sizeof(float); }

cudaError_t launch_nf4_gemv(const qln_nf4_weight *w, const uint16_t *X, int64_t n, const uint16_t *A,
                            const uint16_t *B, int r, float s, uint16_t *Y, uint16_t *U_out, float *upart,
                            int *counter, int *status, cudaStream_t st, int num_sms) {
    GvParams p;
    p.codes = w->codes;
    p.absmax = w->absmax;
    p.qabs = w->qabs;
    p.dq_scale = w->dq_scale;
    p.dq_mean = w->dq_mean;
    p.rows = w->rows;
    p.cols = w->cols;
    p.X = X;
    p.n = (int)n;
    p.A = A;
    p.B = B;
    p.r = r;
    p.s = s;
    p.Y = Y;
    p.U_out = U_out;
    p.upart = upart;
    p.counter = counter;
    p.status = status;
    const int nt = (int)((n + 7) / 8);
    const size_t smem = gv_smem_bytes(nt);
    void *args[] = {&p};
    // persistent: at most one CTA per SM, so the whole grid is co-resident
    const int64_t ngroups = w->rows / kGvRows;
    const dim3 grid((unsigned)(ngroups < num_sms ? ngroups : num_sms)), block(kGvWarps * 32);
    const void *fn;
    switch (nt) {
        case 1: fn = (const void *)nf4_decode_fwd_kernel<1>; break;
        case 2: fn = (const void *)nf4_decode_fwd_kernel<2>; break;
        case 3: fn = (const void *)nf4_decode_fwd_kernel<3>; break;
        default: fn = (const void *)nf4_decode_fwd_kernel<4>; break;
    }
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchCooperativeKernel(fn, grid, block, args, smem, st);
    note_launch();
    return e;
}

}  // namespace qln
