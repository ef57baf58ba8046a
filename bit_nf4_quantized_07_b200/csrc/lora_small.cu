// Skinny products around the rank-r adapters.  All are HBM-bound (they read
// one activation tensor once and touch an r-wide side), so they use the
// register-level mma.sync tensor path with fp32 accumulation.
//
// Method: "LoRA 与 QLoRA" section LoRA: y = W0 x + s B(A x), A x is formed
// first (r x dseq) and BA never is; only A and B are trained.  Deck
// "3 QLoRA Finetuning" card 1: gradients flow through the dequantized weight.
//   lora_down : U = X A^T  (forward)  and  G = dY B  (backward)
//   tn_skinny : dA = s G^T X  and  dB = s dY^T U    (reductions over tokens)
#include "qln_common.cuh"
#include "qln_internal.h"

namespace qln {

// sum_{z < splits} p[z * pitch] in the order z = 0, 1, ...; the loads go out
// eight at a time ahead of their adds.
__device__ __forceinline__ float fold_splits(const float *__restrict__ p, int64_t pitch, int splits) {
    float v = 0.f;
    for (int z0 = 0; z0 < splits; z0 += 8) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = (z0 + u < splits) ? __ldcg(p + (int64_t)(z0 + u) * pitch) : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (z0 + u < splits) v = __fadd_rn(v, x[u]);
    }
    return v;
}

// ===========================================================================
// lora_down: out[t][j] = sum_k in[t][k] * wt[j][k], in [n][K], wt [r][K]
// (WKM = false) or wt stored K-major as [K][r] (WKM = true, i.e. wt^T row-major:
// G = dY B reads B [dout][r] as it is stored, no transpose).
// Split-K tiles: a CTA owns 64 tokens x all r outputs over `cps` chunks of 64
// k, streamed through a 4-stage cp.async ring (both operands K-contiguous, so
// plain ldmatrix feeds the MMA); 4 warps x 16 tokens each.  Each split writes
// an fp32 partial tile; lora_fold adds the splits in a fixed order
// (deterministic) and writes out = bf16(sum) and out_scaled = bf16(scale*sum).
// ===========================================================================
constexpr int kDnStages = 4;
constexpr int kDnLd = 72;  // padded row (bf16) of the staged tiles

template <int NT, bool WKM>
__global__ void __launch_bounds__(128) lora_down_kernel(const uint16_t *__restrict__ in, int64_t n, int64_t K,
                                                        const uint16_t *__restrict__ wt, int r, int cps,
                                                        float *__restrict__ partial, int *status_reset) {
    extern __shared__ __align__(16) uint16_t dsm[];
    pdl_wait();  // every input may come from the previous kernel on the stream
    pdl_trigger();
    if (status_reset && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *status_reset = QLN_OK;
    constexpr int WR = NT * 8;                              // adapter rows staged (r rounded up to 8)
    constexpr int WKLD = WR + 8;                            // padded row of a K-major wt stage
    constexpr int STAGE = 64 * kDnLd + (WKM ? 64 * WKLD : WR * kDnLd);  // elements per stage
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int64_t t0 = (int64_t)blockIdx.x * 64;
    const int split = blockIdx.y;
    const int64_t nch = K / 64;
    const int64_t ch0 = (int64_t)split * cps;
    const int64_t ch1 = ch0 + cps < nch ? ch0 + cps : nch;

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;

    auto load = [&](int stage, int64_t ch) {
        uint16_t *Xs = dsm + stage * STAGE;
        uint16_t *Ws = Xs + 64 * kDnLd;
        const int64_t k0 = ch * 64;
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // 64 rows x 8 chunks
            const int idx = tid + 128 * i, row = idx >> 3, ck = idx & 7;
            const int64_t t = t0 + row;
            const bool ok = t < n;
            cp_async16_zfill(Xs + row * kDnLd + 8 * ck, ok ? in + t * K + k0 + 8 * ck : in, ok ? 16 : 0);
        }
        if (WKM) {  // 64 k rows x WR/8 chunks of the [K][r] layout
            for (int idx = tid; idx < 64 * (WR / 8); idx += 128) {
                const int row = idx / (WR / 8), ck = idx % (WR / 8);
                const bool ok = 8 * ck < r;
                cp_async16_zfill(Ws + row * WKLD + 8 * ck, ok ? wt + (k0 + row) * (int64_t)r + 8 * ck : wt, ok ? 16 : 0);
            }
        } else {
            for (int idx = tid; idx < WR * 8; idx += 128) {
                const int row = idx >> 3, ck = idx & 7;
                const bool ok = row < r;
                cp_async16_zfill(Ws + row * kDnLd + 8 * ck, ok ? wt + (int64_t)row * K + k0 + 8 * ck : wt, ok ? 16 : 0);
            }
        }
    };

    // prologue: fill kDnStages-1 stages (empty commit groups keep the count uniform)
#pragma unroll
    for (int i = 0; i < kDnStages - 1; ++i) {
        if (ch0 + i < ch1) load(i, ch0 + i);
        cp_async_commit();
    }
    for (int64_t ch = ch0; ch < ch1; ++ch) {
        const int it = (int)(ch - ch0);
        {
            const int64_t nx = ch + kDnStages - 1;
            if (nx < ch1) load((it + kDnStages - 1) % kDnStages, nx);
            cp_async_commit();
        }
        cp_async_wait<kDnStages - 1>();
        __syncthreads();
        const uint16_t *Xs = dsm + (it % kDnStages) * STAGE;
        const uint16_t *Ws = Xs + 64 * kDnLd;
#pragma unroll
        for (int kk = 0; kk < 64; kk += 16) {
            uint32_t a[4];
            {
                const int row = 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int col = kk + (lane >> 4) * 8;
                ldmatrix_x4(a[0], a[1], a[2], a[3], Xs + row * kDnLd + col);
            }
            if (WKM) {  // Ws [k][j]: the transposing load gives the k x n fragment
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    const int krow = kk + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int ncol = np * 16 + (lane >> 4) * 8;
                    uint32_t r0, r1, r2, r3;
                    ldmatrix_x4_trans(r0, r1, r2, r3, Ws + krow * WKLD + ncol);
                    const uint32_t b0[2] = {r0, r1}, b1[2] = {r2, r3};
                    mma_bf16_16816(acc[2 * np], a, b0);
                    mma_bf16_16816(acc[2 * np + 1], a, b1);
                }
                if (NT & 1) {
                    const int krow = kk + (lane & 7) + ((lane >> 3) & 1) * 8;
                    uint32_t r0, r1;
                    ldmatrix_x2_trans(r0, r1, Ws + krow * WKLD + (NT - 1) * 8);
                    const uint32_t b0[2] = {r0, r1};
                    mma_bf16_16816(acc[NT - 1], a, b0);
                }
            } else {
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    const int row = np * 16 + (lane & 7) + (lane >> 4) * 8;
                    const int col = kk + ((lane >> 3) & 1) * 8;
                    uint32_t r0, r1, r2, r3;
                    ldmatrix_x4(r0, r1, r2, r3, Ws + row * kDnLd + col);
                    const uint32_t b0[2] = {r0, r1}, b1[2] = {r2, r3};
                    mma_bf16_16816(acc[2 * np], a, b0);
                    mma_bf16_16816(acc[2 * np + 1], a, b1);
                }
                if (NT & 1) {
                    const int row = (NT - 1) * 8 + (lane & 7);
                    const int col = kk + ((lane >> 3) & 1) * 8;
                    uint32_t r0, r1;
                    ldmatrix_x2(r0, r1, Ws + row * kDnLd + col);
                    const uint32_t b0[2] = {r0, r1};
                    mma_bf16_16816(acc[NT - 1], a, b0);
                }
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

    float *dst = partial + (int64_t)split * n * r;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t t = t0 + 16 * warp + g + 8 * (e >> 1);
            const int j = 8 * nt + 2 * c + (e & 1);
            if (t < n && j < r) dst[t * r + j] = acc[nt][e];
        }
}

__global__ void lora_fold_kernel(const float *__restrict__ partial, int splits, int64_t total, float scale,
                                 uint16_t *__restrict__ out, uint16_t *__restrict__ out_scaled) {
    pdl_wait();
    pdl_trigger();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const float v = fold_splits(partial + i, total, splits);
        out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        if (out_scaled) out_scaled[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(scale, v)));
    }
}

// CTAs of `smem` bytes that fit on one SM (228 KB per SM, 1 KB reserved per
// CTA, at most 16 CTAs of 128 threads); registers are not the limit for these
// kernels at their launch bounds.
static int64_t ctas_per_sm(size_t smem) {
    const int64_t k = (int64_t)(228 * 1024) / (int64_t)(smem + 1024);
    return k < 1 ? 1 : (k > 16 ? 16 : k);
}

static size_t lora_down_smem(int r, bool wkm) {
    const int nt = (r + 7) / 8;
    return (size_t)kDnStages * (64 * kDnLd + (wkm ? 64 * (nt * 8 + 8) : nt * 8 * kDnLd)) * sizeof(uint16_t);
}

// Splits of the K range: one full wave of resident CTAs (rounded down, so the
// grid never spills into a second, mostly empty wave), at least 4 chunks of
// 64 per CTA.  The staged-tile size is the same for both operand layouts to
// within a few KB, so the plan uses the larger (k-major) one.
void lora_down_plan(int64_t n, int64_t K, int r, int num_sms, int *splits, int *cps) {
    const int64_t nch = K / 64;
    const int64_t ttiles = (n + 63) / 64;
    const size_t smem = lora_down_smem(r, true) > lora_down_smem(r, false) ? lora_down_smem(r, true)
                                                                            : lora_down_smem(r, false);
    int64_t sp = ctas_per_sm(smem) * (int64_t)num_sms / ttiles;
    const int64_t maxsp = nch / 4 > 0 ? nch / 4 : 1;
    if (sp > maxsp) sp = maxsp;
    if (sp < 1) sp = 1;
    const int64_t c = (nch + sp - 1) / sp;
    *cps = (int)c;
    *splits = (int)((nch + c - 1) / c);
}

size_t lora_down_partial_bytes(int64_t n, int64_t K, int r, int num_sms) {
    int sp, cps;
    lora_down_plan(n, K, r, num_sms, &sp, &cps);
    return (size_t)sp * (size_t)n * (size_t)r * sizeof(float);
}

template <int NT, bool WKM>
static cudaError_t launch_down_t(const uint16_t *in, int64_t n, int64_t K, const uint16_t *wt, int r, int splits,
                                 int cps, float *partial, int *status_reset, cudaStream_t st) {
    const size_t smem = lora_down_smem(NT * 8, WKM);
    auto kern = lora_down_kernel<NT, WKM>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)((n + 63) / 64), (unsigned)splits);
    return launch_pdl(kern, grid, dim3(128), smem, st, in, n, K, wt, r, cps, partial, status_reset);
}

template <bool WKM>
static cudaError_t launch_down_nt(const uint16_t *in, int64_t n, int64_t K, const uint16_t *wt, int r, int splits,
                                  int cps, float *partial, int *sr, cudaStream_t st) {
    const int nt = (r + 7) / 8;
    cudaError_t e;
    switch (nt) {
        case 1: e = launch_down_t<1, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 2: e = launch_down_t<2, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 3: e = launch_down_t<3, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 4: e = launch_down_t<4, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 5: e = launch_down_t<5, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 6: e = launch_down_t<6, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 7: e = launch_down_t<7, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 8: e = launch_down_t<8, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 9: e = launch_down_t<9, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 10: e = launch_down_t<10, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 11: e = launch_down_t<11, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 12: e = launch_down_t<12, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 13: e = launch_down_t<13, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 14: e = launch_down_t<14, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        case 15: e = launch_down_t<15, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
        default: e = launch_down_t<16, WKM>(in, n, K, wt, r, splits, cps, partial, sr, st); break;
    }
    return e;
}

cudaError_t launch_lora_down(const uint16_t *in, int64_t n, int64_t K, const uint16_t *wt, bool wt_kmajor, int r,
                             float scale, uint16_t *out, uint16_t *out_scaled, float *partial, cudaStream_t st,
                             int num_sms, int *status_reset) {
    int splits, cps;
    lora_down_plan(n, K, r, num_sms, &splits, &cps);
    cudaError_t e = wt_kmajor ? launch_down_nt<true>(in, n, K, wt, r, splits, cps, partial, status_reset, st)
                              : launch_down_nt<false>(in, n, K, wt, r, splits, cps, partial, status_reset, st);
    if (e != cudaSuccess) return e;
    const int64_t total = n * r;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    return launch_pdl(lora_fold_kernel, dim3((unsigned)blocks), dim3(256), 0, st, (const float *)partial, splits, total,
                      scale, out, out_scaled);
}

// ===========================================================================
// tn_skinny: C[m][j] = scale * sum_t P[t][m] Q[t][j] for a narrow side j < R
// (R = the adapter rank, <= 128): P [n][M], Q [n][R] row-major bf16, fp32 out,
// stored as C[m][j] or, with `transpose`, as C[j][m].  dB = s dY^T U is
// (P = dY, Q = U); dA = s G^T X is the transpose of (P = X, Q = G).  A CTA owns
// 128 m x all R over an interleaved share of the 32-token steps: 4 warps x 32
// m, both operands staged by cp.async and read with ldmatrix.trans (t is the row
// index of both).  Partials per token split are folded in a fixed order.
// ===========================================================================
constexpr int kSkBM = 128, kSkBK = 32, kSkPad = 136, kSkStages = 4;

// One 128-row tile of C over the token steps split, split + nsplit, ...:
// accumulate P^T Q for rows [m0, m0 + 128) and all R columns, then store the
// fp32 partial (partials != null) or scale * sum into C.  STG-stage cp.async
// ring; the caller's CTA has 128 threads and STG * kSkBK * (kSkPad + QLD)
// bf16 of shared memory.
template <int NTJ, int STG>
__device__ __forceinline__ void skinny_tile(const uint16_t *__restrict__ P, const uint16_t *__restrict__ Q, int64_t n,
                                            int64_t M, int R, float scale, bool transpose, float *__restrict__ C,
                                            float *__restrict__ partials, int64_t m0, int split, int nsplit,
                                            uint16_t *sk) {
    constexpr int QW = NTJ * 8, QLD = QW + 8;
    uint16_t *Ps = sk;                             // [stages][32][kSkPad]
    uint16_t *Qs = sk + STG * kSkBK * kSkPad;      // [stages][32][QLD]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int64_t nsteps = (n + kSkBK - 1) / kSkBK;

    float acc[2][NTJ][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < NTJ; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

    auto load = [&](int buf, int64_t step) {
        const int64_t tb = step * kSkBK;
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // P: 32 rows x 16 chunks
            const int idx = tid + 128 * i, row = idx >> 4, ck = idx & 15;
            const int64_t t = tb + row, col = m0 + 8 * ck;
            const bool ok = t < n && col < M;
            cp_async16_zfill(Ps + (buf * kSkBK + row) * kSkPad + 8 * ck, ok ? P + t * M + col : P, ok ? 16 : 0);
        }
        for (int idx = tid; idx < kSkBK * NTJ; idx += 128) {  // Q: 32 rows x NTJ chunks
            const int row = idx / NTJ, ck = idx % NTJ;
            const int64_t t = tb + row;
            const bool ok = t < n && 8 * ck < R;
            cp_async16_zfill(Qs + (buf * kSkBK + row) * QLD + 8 * ck, ok ? Q + t * R + 8 * ck : Q, ok ? 16 : 0);
        }
    };

    const int64_t mysteps = split < nsteps ? (nsteps - split + nsplit - 1) / nsplit : 0;
#pragma unroll
    for (int i = 0; i < STG - 1; ++i) {
        if (i < mysteps) load(i, split + (int64_t)i * nsplit);
        cp_async_commit();
    }
    for (int64_t it = 0; it < mysteps; ++it) {
        {
            const int64_t nx = it + STG - 1;
            if (nx < mysteps) load((int)(nx % STG), split + nx * nsplit);
            cp_async_commit();
        }
        cp_async_wait<STG - 1>();
        __syncthreads();
        const int buf = (int)(it % STG);
        const uint16_t *Pb = Ps + buf * kSkBK * kSkPad;
        const uint16_t *Qb = Qs + buf * kSkBK * QLD;
#pragma unroll
        for (int kk = 0; kk < kSkBK; kk += 16) {
            uint32_t a[2][4];
            const int mat = lane >> 3;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int krow = kk + (mat >> 1) * 8 + (lane & 7);
                const int mcol = warp * 32 + mt * 16 + (mat & 1) * 8;
                ldmatrix_x4_trans(a[mt][0], a[mt][1], a[mt][2], a[mt][3], Pb + krow * kSkPad + mcol);
            }
            const int krow = kk + (mat & 1) * 8 + (lane & 7);
#pragma unroll
            for (int np = 0; np < NTJ / 2; ++np) {
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4_trans(r0, r1, r2, r3, Qb + krow * QLD + np * 16 + (mat >> 1) * 8);
                const uint32_t b0[2] = {r0, r1}, b1[2] = {r2, r3};
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    mma_bf16_16816(acc[mt][2 * np], a[mt], b0);
                    mma_bf16_16816(acc[mt][2 * np + 1], a[mt], b1);
                }
            }
            if (NTJ & 1) {
                uint32_t r0, r1;
                ldmatrix_x2_trans(r0, r1, Qb + krow * QLD + (NTJ - 1) * 8);
                const uint32_t b0[2] = {r0, r1};
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) mma_bf16_16816(acc[mt][NTJ - 1], a[mt], b0);
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NTJ; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t m = m0 + warp * 32 + mt * 16 + g + 8 * (e >> 1);
                const int j = nt * 8 + 2 * c + (e & 1);
                if (m < M && j < R) {
                    if (partials)
                        partials[((int64_t)split * M + m) * R + j] = acc[mt][nt][e];
                    else
                        C[transpose ? (int64_t)j * M + m : m * R + j] = __fmul_rn(scale, acc[mt][nt][e]);
                }
            }
}

template <int NTJ>  // R <= 8 NTJ
__global__ void __launch_bounds__(128) tn_skinny_kernel(const uint16_t *__restrict__ P, const uint16_t *__restrict__ Q,
                                                        int64_t n, int64_t M, int R, float scale, bool transpose,
                                                        float *__restrict__ C, float *__restrict__ partials) {
    extern __shared__ __align__(16) uint16_t sk[];
    pdl_wait();  // P and Q may come from the previous kernel on the stream
    pdl_trigger();
    skinny_tile<NTJ, kSkStages>(P, Q, n, M, R, scale, transpose, C, partials, (int64_t)blockIdx.x * kSkBM, blockIdx.y,
                                gridDim.y, sk);
}

// dB = s dY^T U and dA = s (X^T G)^T as one persistent launch of few CTAs,
// for SMs the dX GEMM leaves idle: CTA b takes tiles b, b + gridDim.x, ... of
// the list [dB tiles | dA tiles], each over all tokens (no split, no partials,
// no fold: the order of every sum is fixed).  More stages than the split
// kernel, since each CTA has an SM to itself.
//
// It is launched on the caller's stream right after the dX GEMM, as its
// programmatic dependent, and runs beside it.  It reads dY, U, X and G before
// any dependency wait.  That is safe because a dependent can start only once
// every CTA of the GEMM has released it, and every kernel of this library
// releases its dependents only after its own dependency wait; so when this
// kernel starts, every kernel before the GEMM (those that wrote G, U, dY, X)
// has completed, and its writes are in L2, which is where the cp.async.cg
// copies read.  The GEMM writes none of these inputs and reads neither dA nor
// dB.  The kernel waits on the GEMM before it exits, so it never completes
// before the GEMM does, and a kernel that follows it on the stream sees dX.
constexpr int kSideStages = 8;

template <int NTJ>
__global__ void __launch_bounds__(128) tn_skinny_side_kernel(const uint16_t *__restrict__ dY,
                                                             const uint16_t *__restrict__ U, int64_t dout,
                                                             const uint16_t *__restrict__ X,
                                                             const uint16_t *__restrict__ G, int64_t din, int64_t n,
                                                             int R, float scale, float *__restrict__ dA,
                                                             float *__restrict__ dB) {
    extern __shared__ __align__(16) uint16_t sk[];
    const int64_t tB = (dout + kSkBM - 1) / kSkBM, tA = (din + kSkBM - 1) / kSkBM;
    for (int64_t v = blockIdx.x; v < tB + tA; v += gridDim.x) {
        __syncthreads();  // the previous tile's buffers are free
        if (v < tB)
            skinny_tile<NTJ, kSideStages>(dY, U, n, dout, R, scale, false, dB, nullptr, v * kSkBM, 0, 1, sk);
        else
            skinny_tile<NTJ, kSideStages>(X, G, n, din, R, scale, true, dA, nullptr, (v - tB) * kSkBM, 0, 1, sk);
    }
    pdl_wait();  // complete only after the dX GEMM
}

__global__ void tn_skinny_fold_kernel(const float *__restrict__ partials, int splits, int64_t M, int R, float scale,
                                      bool transpose, float *__restrict__ C) {
    pdl_wait();
    pdl_trigger();
    const int64_t MR = M * R;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < MR; i += stride) {
        const float v = fold_splits(partials + i, MR, splits);
        const int64_t m = i / R;
        const int j = (int)(i % R);
        C[transpose ? (int64_t)j * M + m : i] = __fmul_rn(scale, v);
    }
}

// About 6 CTAs per SM, each with at least 4 token steps (128 tokens).
// Token splits: one full wave of resident CTAs (rounded down), at least 4
// token steps per CTA, at most 64 splits.
int tn_skinny_splits(int64_t n, int64_t M, int R, int num_sms) {
    const int64_t tiles = (M + kSkBM - 1) / kSkBM;
    const int64_t steps = (n + kSkBK - 1) / kSkBK;
    const int ntj = (R + 7) / 8;
    const size_t smem = (size_t)kSkStages * kSkBK * (kSkPad + ntj * 8 + 8) * sizeof(uint16_t);
    int64_t splits = ctas_per_sm(smem) * (int64_t)num_sms / tiles;
    const int64_t maxsp = steps / 4 > 0 ? steps / 4 : 1;
    if (splits > maxsp) splits = maxsp;
    if (splits > 64) splits = 64;
    if (splits < 1) splits = 1;
    return (int)splits;
}

size_t tn_skinny_partials_bytes(int64_t M, int R, int splits) {
    return splits > 1 ? (size_t)splits * (size_t)M * (size_t)R * sizeof(float) : 0;
}

template <int NTJ>
static cudaError_t launch_skinny_t(const uint16_t *P, const uint16_t *Q, int64_t n, int64_t M, int R, float scale,
                                   bool transpose, float *C, float *partials, int splits, cudaStream_t st) {
    const size_t smem = (size_t)kSkStages * kSkBK * (kSkPad + NTJ * 8 + 8) * sizeof(uint16_t);
    auto kern = tn_skinny_kernel<NTJ>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)((M + kSkBM - 1) / kSkBM), (unsigned)splits);
    return launch_pdl(kern, grid, dim3(128), smem, st, P, Q, n, M, R, scale, transpose, C,
                      splits > 1 ? partials : nullptr);
}

cudaError_t launch_tn_skinny(const uint16_t *P, const uint16_t *Q, int64_t n, int64_t M, int R, float scale,
                             bool transpose, float *C, float *partials, int splits, cudaStream_t st) {
    cudaError_t e;
    switch ((R + 7) / 8) {
        case 1: e = launch_skinny_t<1>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 2: e = launch_skinny_t<2>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 3: e = launch_skinny_t<3>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 4: e = launch_skinny_t<4>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 5: e = launch_skinny_t<5>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 6: e = launch_skinny_t<6>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 7: e = launch_skinny_t<7>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 8: e = launch_skinny_t<8>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 9: e = launch_skinny_t<9>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 10: e = launch_skinny_t<10>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 11: e = launch_skinny_t<11>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 12: e = launch_skinny_t<12>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 13: e = launch_skinny_t<13>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 14: e = launch_skinny_t<14>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        case 15: e = launch_skinny_t<15>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
        default: e = launch_skinny_t<16>(P, Q, n, M, R, scale, transpose, C, partials, splits, st); break;
    }
    if (e != cudaSuccess || splits <= 1) return e;
    const int64_t MR = M * R;
    int64_t blocks = (MR + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    return launch_pdl(tn_skinny_fold_kernel, dim3((unsigned)blocks), dim3(256), 0, st, (const float *)partials, splits,
                      M, R, scale, transpose, C);
}

template <int NTJ>
static cudaError_t launch_side_t(const uint16_t *dY, const uint16_t *U, int64_t dout, const uint16_t *X,
                                 const uint16_t *G, int64_t din, int64_t n, int R, float scale, float *dA, float *dB,
                                 int nside, cudaStream_t st) {
    const size_t smem = (size_t)kSideStages * kSkBK * (kSkPad + NTJ * 8 + 8) * sizeof(uint16_t);
    auto kern = tn_skinny_side_kernel<NTJ>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3((unsigned)nside), dim3(128), smem, st, dY, U, dout, X, G, din, n, R, scale, dA, dB);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_tn_skinny_side(const uint16_t *dY, const uint16_t *U, int64_t dout, const uint16_t *X,
                                  const uint16_t *G, int64_t din, int64_t n, int R, float scale, float *dA, float *dB,
                                  int nside, cudaStream_t st) {
    switch ((R + 7) / 8) {
        case 1: return launch_side_t<1>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 2: return launch_side_t<2>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 3: return launch_side_t<3>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 4: return launch_side_t<4>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 5: return launch_side_t<5>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 6: return launch_side_t<6>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 7: return launch_side_t<7>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 8: return launch_side_t<8>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 9: return launch_side_t<9>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 10: return launch_side_t<10>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 11: return launch_side_t<11>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 12: return launch_side_t<12>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 13: return launch_side_t<13>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 14: return launch_side_t<14>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        case 15: return launch_side_t<15>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
        default: return launch_side_t<16>(dY, U, dout, X, G, din, n, R, scale, dA, dB, nside, st);
    }
}

}  // namespace qln
