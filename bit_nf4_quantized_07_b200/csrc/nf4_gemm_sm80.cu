// Fused NF4 doubleDequant + GEMM on the register-level mma.sync tensor path.
// Serves the token counts between the decode-sized forward (n <= 32) and the
// tcgen05 GEMM (n >= 64), i.e. 32 < n < 64, and any shape the decode-sized
// kernel does not take; and the dX GEMM for n < 64.
//
// Method: "LoRA 与 QLoRA" section QLoRA 1 (4-bit weight -> dequant -> BF16
// -> GEMM); jjjymmm.cn "QLoRA" (doubleDequant: constants first, then the
// weights; BF16 activations); "LoRA 与 QLoRA" section LoRA (y = W0 x +
// s B(A x)); deck "3 QLoRA Finetuning" card 1 (gradients flow through the
// dequantized weight).
//
//   forward (TRANS = false): out[t][m] = sum_k act[t][k] W'[m][k] + sum_j lact[t][j] lw[m][j]
//                            (act = X, lact = s*U, lw = B, out = Y)
//   dX      (TRANS = true) : out[t][m] = sum_k act[t][k] W'[k][m] + sum_j lact[t][j] lw[j][m]
//                            (act = dY, lact = s*G, lw = A, out = dX)
// A 64x64 tile of W' is decoded per k-step into shared memory (W' never
// reaches HBM); ldmatrix (.trans for dX) feeds the MMA.
#include "qln_common.cuh"
#include "qln_internal.h"

namespace qln {

constexpr int kSmBM = 64, kSmBN = 64, kSmBK = 64, kSmPad = 72;

struct SmemSm80 {
    uint8_t codes[2][64][32];
    uint16_t act[2][kSmBN][kSmPad];
    uint16_t w[64][kSmPad];
    float cb[16];
};

template <bool TRANS>
__global__ void __launch_bounds__(128) nf4_mma_gemm_kernel(const uint8_t *__restrict__ codes,
                                                           const float *__restrict__ absmax,
                                                           const int8_t *__restrict__ qabs,
                                                           const float *__restrict__ dq_scale,
                                                           const float *__restrict__ dq_mean, int64_t rows,
                                                           int64_t cols, const uint16_t *__restrict__ act, int64_t n,
                                                           const uint16_t *__restrict__ lact,
                                                           const uint16_t *__restrict__ lw, int r,
                                                           uint16_t *__restrict__ out, bool e4m3) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    pdl_wait();  // every input may come from the previous kernel on the stream
    pdl_trigger();
    SmemSm80 &S = *reinterpret_cast<SmemSm80 *>(smem_raw);
    const int rpad = (r + 15) & ~15;
    // adapter tiles after the main structure
    uint16_t *Ls = reinterpret_cast<uint16_t *>(smem_raw + sizeof(SmemSm80));
    const int ls_ld = TRANS ? kSmPad : rpad + 8;                 // fwd: [64][rpad+8], dX: [rpad][72]
    const int ls_rows = TRANS ? rpad : 64;
    uint16_t *Ms = Ls + ls_rows * ls_ld;                          // [64][rpad+8]
    const int ms_ld = rpad + 8;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int wm = warp & 1, wn = warp >> 1;
    const int64_t t0 = (int64_t)blockIdx.x * kSmBN;
    const int64_t m0 = (int64_t)blockIdx.y * kSmBM;
    const int64_t K = TRANS ? rows : cols;
    const int64_t M = TRANS ? cols : rows;
    const int KT = (int)(K / kSmBK);
    const int64_t bpr = cols / 64;  // blocks per W row
    if (tid < 16) S.cb[tid] = nf4_value(tid);
    const float mu = qabs ? __ldg(dq_mean) : 0.f;

    // W tile origin for k-step kt: fwd (m0, k0), dX (k0, m0)
    auto wtile_row0 = [&](int kt) -> int64_t { return TRANS ? (int64_t)kt * kSmBK : m0; };
    auto wtile_col0 = [&](int kt) -> int64_t { return TRANS ? m0 : (int64_t)kt * kSmBK; };

    auto load_stage = [&](int buf, int kt) {
        const int64_t wr0 = wtile_row0(kt), wc0 = wtile_col0(kt);
        {   // codes: 64 rows x 32 bytes = 128 chunks of 16 bytes
            const int row = tid >> 1, ck = tid & 1;
            cp_async16(&S.codes[buf][row][16 * ck], codes + (wr0 + row) * (cols / 2) + wc0 / 2 + 16 * ck);
        }
        const int64_t k0 = (int64_t)kt * kSmBK;
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // activations: 64 tokens x 64 k = 512 chunks
            const int idx = tid + 128 * i, row = idx >> 3, ck = idx & 7;
            const int64_t t = t0 + row;
            const bool ok = t < n;
            cp_async16_zfill(&S.act[buf][row][8 * ck], ok ? act + t * K + k0 + 8 * ck : act, ok ? 16 : 0);
        }
        cp_async_commit();
    };
    auto block_const = [&](int kt) -> float {
        const int row = tid >> 1;
        const int64_t jb = (wtile_row0(kt) + row) * bpr + wtile_col0(kt) / 64;
        if (qabs) return dq_restore((uint32_t)__ldg(qabs + jb), __ldg(dq_scale + (jb >> 8)), mu, e4m3);
        return __ldg(absmax + jb);
    };

    float acc[2][4][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

    auto mma_tile = [&](const uint16_t *Abase, int a_ld, bool a_trans, const uint16_t *Bbase, int b_ld, int kk) {
        uint32_t a[2][4], b[4][2];
        const int mat = lane >> 3;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            if (!a_trans) {
                const int mrow = wm * 32 + mt * 16 + (mat & 1) * 8 + (lane & 7);
                const int kcol = kk + (mat >> 1) * 8;
                ldmatrix_x4(a[mt][0], a[mt][1], a[mt][2], a[mt][3], Abase + mrow * a_ld + kcol);
            } else {
                const int krow = kk + (mat >> 1) * 8 + (lane & 7);
                const int mcol = wm * 32 + mt * 16 + (mat & 1) * 8;
                ldmatrix_x4_trans(a[mt][0], a[mt][1], a[mt][2], a[mt][3], Abase + krow * a_ld + mcol);
            }
        }
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            const int trow = wn * 32 + np * 16 + (mat >> 1) * 8 + (lane & 7);
            const int kcol = kk + (mat & 1) * 8;
            uint32_t r0, r1, r2, r3;
            ldmatrix_x4(r0, r1, r2, r3, Bbase + trow * b_ld + kcol);
            b[2 * np][0] = r0;
            b[2 * np][1] = r1;
            b[2 * np + 1][0] = r2;
            b[2 * np + 1][1] = r3;
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) mma_bf16_16816(acc[mt][nt], a[mt], b[nt]);
    };

    load_stage(0, 0);
    float ah = block_const(0);
    for (int kt = 0; kt < KT; ++kt) {
        const int buf = kt & 1;
        float ah_next = 0.f;
        if (kt + 1 < KT) {
            load_stage(buf ^ 1, kt + 1);
            ah_next = block_const(kt + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        {   // decode: thread -> row tid/2, 32 elements (16 code bytes)
            const int row = tid >> 1, half = tid & 1;
            const uint4 cw = *reinterpret_cast<const uint4 *>(&S.codes[buf][row][16 * half]);
            const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
            uint32_t o[16];
#pragma unroll
            for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                for (int bi = 0; bi < 4; ++bi) {
                    const uint32_t byte = (words[wi] >> (8 * bi)) & 0xffu;
                    o[4 * wi + bi] = pack_bf16x2(__fmul_rn(ah, S.cb[byte >> 4]), __fmul_rn(ah, S.cb[byte & 15u]));
                }
            uint4 *dst = reinterpret_cast<uint4 *>(&S.w[row][32 * half]);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kSmBK; kk += 16) mma_tile(&S.w[0][0], kSmPad, TRANS, &S.act[buf][0][0], kSmPad, kk);
        __syncthreads();
        ah = ah_next;
    }

    // Adapter term as extra K steps over j (zero-padded to a multiple of 16).
    {
        const int cpr = rpad / 8;  // 16-byte chunks per adapter row (padded)
        const int rc = r / 8;      // real chunks (r % 8 == 0)
        // Ls: fwd rows m (lw = B [rows][r]); dX rows j (lw = A [r][cols])
        const int ls_chunks = TRANS ? rpad * 8 : 64 * cpr;
        for (int idx = tid; idx < ls_chunks; idx += 128) {
            int row, ck;
            const uint16_t *src;
            bool ok;
            if (!TRANS) {
                row = idx / cpr;
                ck = idx % cpr;
                ok = ck < rc;
                src = lw + (m0 + row) * r + 8 * ck;
            } else {
                row = idx >> 3;
                ck = idx & 7;
                ok = row < r;
                src = lw + (int64_t)row * cols + m0 + 8 * ck;
            }
            cp_async16_zfill(Ls + row * ls_ld + 8 * ck, ok ? src : lw, ok ? 16 : 0);
        }
        for (int idx = tid; idx < 64 * cpr; idx += 128) {
            const int row = idx / cpr, ck = idx % cpr;
            const int64_t t = t0 + row;
            const bool ok = (t < n) && (ck < rc);
            cp_async16_zfill(Ms + row * ms_ld + 8 * ck, ok ? lact + t * r + 8 * ck : lact, ok ? 16 : 0);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        for (int kk = 0; kk < rpad; kk += 16) mma_tile(Ls, ls_ld, TRANS, Ms, ms_ld, kk);
        __syncthreads();
    }

    // Epilogue: fp32 -> bf16, transpose through shared memory, 16-byte stores.
    uint16_t *Os = &S.act[0][0][0];  // [64 tokens][72]
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = wm * 32 + mt * 16 + g + 8 * (e >> 1);
                const int t = wn * 32 + nt * 8 + 2 * c + (e & 1);
                Os[t * kSmPad + m] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[mt][nt][e]));
            }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int idx = tid + 128 * i, row = idx >> 3, ck = idx & 7;
        const int64_t t = t0 + row;
        if (t < n)
            *reinterpret_cast<uint4 *>(out + t * M + m0 + 8 * ck) =
                *reinterpret_cast<const uint4 *>(&Os[row * kSmPad + 8 * ck]);
    }
}

cudaError_t launch_nf4_mma_gemm(const qln_nf4_weight *w, bool trans, const uint16_t *act, int64_t n,
                                const uint16_t *lact, const uint16_t *lw, int r, uint16_t *out, int *status,
                                cudaStream_t st, int num_sms) {
    (void)status;
    (void)num_sms;
    const int rpad = (r + 15) & ~15;
    const int ls_ld = trans ? kSmPad : rpad + 8;
    const int ls_rows = trans ? rpad : 64;
    const size_t smem = sizeof(SmemSm80) + (size_t)ls_rows * ls_ld * 2 + (size_t)64 * (rpad + 8) * 2;
    const int64_t M = trans ? w->cols : w->rows;
    dim3 grid((unsigned)((n + kSmBN - 1) / kSmBN), (unsigned)(M / kSmBM));
    const bool e4m3 = w->dq_format == QLN_DQ_E4M3;
    auto kern = trans ? nf4_mma_gemm_kernel<true> : nf4_mma_gemm_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, grid, dim3(128), smem, st, w->codes, w->absmax, w->qabs, w->dq_scale, w->dq_mean, w->rows,
                      w->cols, act, n, lact, lw, r, out, e4m3);
}

}  // namespace qln
