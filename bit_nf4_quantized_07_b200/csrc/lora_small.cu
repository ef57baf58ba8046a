// Skinny products around the rank-r adapters.  All are HBM-bound (they read
// one activation tensor once and touch an r-wide side), so they use the
// register-level mma.sync tensor path with fp32 accumulation.
//
// Method: "LoRA 与 QLoRA" section LoRA: y = W0 x + s B(A x), A x is formed
// first (r x dseq) and BA never is; only A and B are trained.  Deck
// "3 QLoRA Finetuning" card 1: gradients flow through the dequantized weight.
//   lora_down : U = X A^T  (forward)  and  G = dY B  (backward)
//   tn_reduce : dA = s G^T X  and  dB = s dY^T U    (reductions over tokens)
#include "qln_common.cuh"
#include "qln_internal.h"

namespace qln {

// ===========================================================================
// lora_down: out[t][j] = sum_k in[t][k] * wt[j][k], in [n][K], wt [r][K].
// Split-K tiles: a CTA owns 64 tokens x all r outputs over `cps` chunks of 64
// k, streamed through a 4-stage cp.async ring (both operands K-contiguous, so
// plain ldmatrix feeds the MMA); 4 warps x 16 tokens each.  Each split writes
// an fp32 partial tile; lora_fold adds the splits in a fixed order
// (deterministic) and writes out = bf16(sum) and out_scaled = bf16(scale*sum).
// ===========================================================================
constexpr int kDnStages = 4;
constexpr int kDnLd = 72;  // padded row (bf16) of the staged tiles

template <int NT>
__global__ void __launch_bounds__(128) lora_down_kernel(const uint16_t *__restrict__ in, int64_t n, int64_t K,
                                                        const uint16_t *__restrict__ wt, int r, int cps,
                                                        float *__restrict__ partial) {
    extern __shared__ __align__(16) uint16_t dsm[];
    constexpr int WR = NT * 8;                              // adapter rows staged (r rounded up to 8)
    constexpr int STAGE = (64 + WR) * kDnLd;                // elements per stage
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
        for (int idx = tid; idx < WR * 8; idx += 128) {
            const int row = idx >> 3, ck = idx & 7;
            const bool ok = row < r;
            cp_async16_zfill(Ws + row * kDnLd + 8 * ck, ok ? wt + (int64_t)row * K + k0 + 8 * ck : wt, ok ? 16 : 0);
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
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        float v = 0.f;
        for (int z = 0; z < splits; ++z) v = __fadd_rn(v, partial[(int64_t)z * total + i]);
        out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        if (out_scaled) out_scaled[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(scale, v)));
    }
}

// Splits of the K range: about 6 CTAs per SM, at least 4 chunks of 64 per CTA.
void lora_down_plan(int64_t n, int64_t K, int num_sms, int *splits, int *cps) {
    const int64_t nch = K / 64;
    const int64_t ttiles = (n + 63) / 64;
    int64_t sp = (6 * (int64_t)num_sms + ttiles - 1) / ttiles;
    const int64_t maxsp = nch / 4 > 0 ? nch / 4 : 1;
    if (sp > maxsp) sp = maxsp;
    if (sp < 1) sp = 1;
    const int64_t c = (nch + sp - 1) / sp;
    *cps = (int)c;
    *splits = (int)((nch + c - 1) / c);
}

size_t lora_down_partial_bytes(int64_t n, int64_t K, int r, int num_sms) {
    int sp, cps;
    lora_down_plan(n, K, num_sms, &sp, &cps);
    return (size_t)sp * (size_t)n * (size_t)r * sizeof(float);
}

template <int NT>
static cudaError_t launch_down_t(const uint16_t *in, int64_t n, int64_t K, const uint16_t *wt, int r, int splits,
                                 int cps, float *partial, cudaStream_t st) {
    const size_t smem = (size_t)kDnStages * (64 + NT * 8) * kDnLd * sizeof(uint16_t);
    auto kern = lora_down_kernel<NT>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)((n + 63) / 64), (unsigned)splits);
    kern<<<grid, 128, smem, st>>>(in, n, K, wt, r, cps, partial);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_lora_down(const uint16_t *in, int64_t n, int64_t K, const uint16_t *wt, int r, float scale,
                             uint16_t *out, uint16_t *out_scaled, float *partial, cudaStream_t st, int num_sms) {
    int splits, cps;
    lora_down_plan(n, K, num_sms, &splits, &cps);
    const int nt = (r + 7) / 8;
    cudaError_t e;
    switch (nt) {
        case 1: e = launch_down_t<1>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 2: e = launch_down_t<2>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 3: e = launch_down_t<3>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 4: e = launch_down_t<4>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 5: e = launch_down_t<5>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 6: e = launch_down_t<6>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 7: e = launch_down_t<7>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 8: e = launch_down_t<8>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 9: e = launch_down_t<9>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 10: e = launch_down_t<10>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 11: e = launch_down_t<11>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 12: e = launch_down_t<12>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 13: e = launch_down_t<13>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 14: e = launch_down_t<14>(in, n, K, wt, r, splits, cps, partial, st); break;
        case 15: e = launch_down_t<15>(in, n, K, wt, r, splits, cps, partial, st); break;
        default: e = launch_down_t<16>(in, n, K, wt, r, splits, cps, partial, st); break;
    }
    if (e != cudaSuccess) return e;
    const int64_t total = n * r;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    lora_fold_kernel<<<(unsigned)blocks, 256, 0, st>>>(partial, splits, total, scale, out, out_scaled);
    note_launch();
    return cudaGetLastError();
}

// ===========================================================================
// tn_reduce: C[m][c] = scale * sum_t P[t][m] Q[t][c], P [n][M], Q [n][N]
// (both row-major bf16), fp32 C.  64x64 output tiles, 32 tokens per step,
// both operands staged with cp.async and read with ldmatrix.trans (the
// reduction index t is the row index of both).  With splits > 1 each z-slice
// of the grid covers an interleaved share of the token steps and writes an
// fp32 partial tile; tn_fold adds the slices in a fixed order.
// ===========================================================================
constexpr int kTnBM = 64, kTnBN = 64, kTnBK = 32, kTnPad = 72, kTnStages = 4;

__global__ void __launch_bounds__(128) tn_reduce_kernel(const uint16_t *__restrict__ P, const uint16_t *__restrict__ Q,
                                                        int64_t n, int64_t M, int64_t N, float scale,
                                                        float *__restrict__ C, float *__restrict__ partials) {
    __shared__ __align__(16) uint16_t Ps[kTnStages][kTnBK][kTnPad];
    __shared__ __align__(16) uint16_t Qs[kTnStages][kTnBK][kTnPad];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int wm = warp & 1, wn = warp >> 1;  // 2x2 warps, 32x32 each
    const int64_t m0 = (int64_t)blockIdx.y * kTnBM, n0 = (int64_t)blockIdx.x * kTnBN;
    const int split = blockIdx.z, nsplit = gridDim.z;
    const int64_t nsteps = (n + kTnBK - 1) / kTnBK;

    float acc[2][4][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

    auto load = [&](int buf, int64_t step) {
        const int64_t tb = step * kTnBK;
        // 32 rows x 64 cols x 2 operands = 512 16-byte chunks; 4 per thread
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = tid + 128 * i;  // 0..511
            const int op = idx >> 8, rem = idx & 255, row = rem >> 3, ck = rem & 7;
            const int64_t t = tb + row;
            const uint16_t *base = op ? Q : P;
            const int64_t width = op ? N : M;
            const int64_t col = (op ? n0 : m0) + 8 * ck;
            const bool ok = (t < n) && (col < width);
            const uint16_t *src = ok ? base + t * width + col : base;
            uint16_t *dst = op ? &Qs[buf][row][8 * ck] : &Ps[buf][row][8 * ck];
            cp_async16_zfill(dst, src, ok ? 16 : 0);
        }
    };

    // this split's token steps: split, split + nsplit, ...
    const int64_t mysteps = split < nsteps ? (nsteps - split + nsplit - 1) / nsplit : 0;
#pragma unroll
    for (int i = 0; i < kTnStages - 1; ++i) {
        if (i < mysteps) load(i, split + (int64_t)i * nsplit);
        cp_async_commit();
    }
    for (int64_t it = 0; it < mysteps; ++it) {
        {
            const int64_t nx = it + kTnStages - 1;
            if (nx < mysteps) load((int)(nx % kTnStages), split + nx * nsplit);
            cp_async_commit();
        }
        cp_async_wait<kTnStages - 1>();
        __syncthreads();
        const int buf = (int)(it % kTnStages);
#pragma unroll
        for (int kk = 0; kk < kTnBK; kk += 16) {
            uint32_t a[2][4], b[4][2];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int mat = lane >> 3;
                const int krow = kk + (mat >> 1) * 8 + (lane & 7);
                const int mcol = wm * 32 + mt * 16 + (mat & 1) * 8;
                ldmatrix_x4_trans(a[mt][0], a[mt][1], a[mt][2], a[mt][3], &Ps[buf][krow][mcol]);
            }
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                const int mat = lane >> 3;
                const int krow = kk + (mat & 1) * 8 + (lane & 7);
                const int ncol = wn * 32 + np * 16 + (mat >> 1) * 8;
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4_trans(r0, r1, r2, r3, &Qs[buf][krow][ncol]);
                b[2 * np][0] = r0;
                b[2 * np][1] = r1;
                b[2 * np + 1][0] = r2;
                b[2 * np + 1][1] = r3;
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) mma_bf16_16816(acc[mt][nt], a[mt], b[nt]);
        }
        __syncthreads();
    }
    cp_async_wait<0>();

#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t m = m0 + wm * 32 + mt * 16 + g + 8 * (e >> 1);
                const int64_t cc = n0 + wn * 32 + nt * 8 + 2 * c + (e & 1);
                if (m < M && cc < N) {
                    if (partials) partials[((int64_t)split * M + m) * N + cc] = acc[mt][nt][e];
                    else C[m * N + cc] = __fmul_rn(scale, acc[mt][nt][e]);
                }
            }
}

__global__ void tn_fold_kernel(const float *__restrict__ partials, int splits, int64_t MN, float scale,
                               float *__restrict__ C) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < MN; i += stride) {
        float s = 0.f;
        for (int z = 0; z < splits; ++z) s = __fadd_rn(s, partials[(int64_t)z * MN + i]);
        C[i] = __fmul_rn(scale, s);
    }
}

// About 6 CTAs per SM, each with at least 8 token steps (256 tokens).
int tn_reduce_splits(int64_t n, int64_t M, int64_t N, int num_sms) {
    const int64_t tiles = ((M + kTnBM - 1) / kTnBM) * ((N + kTnBN - 1) / kTnBN);
    const int64_t steps = (n + kTnBK - 1) / kTnBK;
    int64_t splits = (6 * (int64_t)num_sms + tiles - 1) / tiles;
    const int64_t maxsp = steps / 8 > 0 ? steps / 8 : 1;
    if (splits > maxsp) splits = maxsp;
    if (splits > 64) splits = 64;
    if (splits < 1) splits = 1;
    return (int)splits;
}

size_t tn_reduce_partials_bytes(int64_t M, int64_t N, int splits) {
    return splits > 1 ? (size_t)splits * (size_t)M * (size_t)N * sizeof(float) : 0;
}

cudaError_t launch_tn_reduce(const uint16_t *P, const uint16_t *Q, int64_t n, int64_t M, int64_t N, float scale,
                             float *C, float *partials, int splits, cudaStream_t st) {
    dim3 grid((unsigned)((N + kTnBN - 1) / kTnBN), (unsigned)((M + kTnBM - 1) / kTnBM), (unsigned)splits);
    tn_reduce_kernel<<<grid, 128, 0, st>>>(P, Q, n, M, N, scale, C, splits > 1 ? partials : nullptr);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || splits <= 1) return e;
    const int64_t MN = M * N;
    int64_t blocks = (MN + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    tn_fold_kernel<<<(unsigned)blocks, 256, 0, st>>>(partials, splits, MN, scale, C);
    note_launch();
    return cudaGetLastError();
}

}  // namespace qln
