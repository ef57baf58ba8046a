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
// A CTA owns 16*MT tokens; its 8 warps split K (64-wide chunks round robin)
// and fold their partial tiles pairwise through shared memory (a fixed order:
// deterministic).  Fragments come straight from global memory: in mma step s
// of a chunk, lane (g, c) feeds k = 16s + 4c .. 16s + 4c + 3 (one 8-byte load
// per row), i.e. each 16-wide step uses k in the natural order.
// ===========================================================================
constexpr int kDownWarps = 8;

template <int MT, int NT>
__global__ void __launch_bounds__(kDownWarps * 32) lora_down_kernel(const uint16_t *__restrict__ in, int64_t n,
                                                                     int64_t K, const uint16_t *__restrict__ wt,
                                                                     int r, float scale, uint16_t *__restrict__ out,
                                                                     uint16_t *__restrict__ out_scaled) {
    extern __shared__ float red[];  // [kDownWarps/2][16*MT][8*NT]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int64_t t0 = (int64_t)blockIdx.x * 16 * MT;
    float acc[MT][NT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;

    const int64_t nchunks = K / 64;
    for (int64_t ch = warp; ch < nchunks; ch += kDownWarps) {
        const int64_t k0 = ch * 64;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int64_t kk = k0 + 16 * s + 4 * c;
            uint32_t a[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int64_t ta = t0 + 16 * mt + g, tb = ta + 8;
                uint2 va = make_uint2(0u, 0u), vb = va;
                if (ta < n) va = __ldg(reinterpret_cast<const uint2 *>(in + ta * K + kk));
                if (tb < n) vb = __ldg(reinterpret_cast<const uint2 *>(in + tb * K + kk));
                a[mt][0] = va.x;  // (row g,   k 4c, 4c+1)
                a[mt][1] = vb.x;  // (row g+8, k 4c, 4c+1)
                a[mt][2] = va.y;  // (row g,   k 4c+2, 4c+3)
                a[mt][3] = vb.y;  // (row g+8, k 4c+2, 4c+3)
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int j = 8 * nt + g;
                uint2 vw = make_uint2(0u, 0u);
                if (j < r) vw = __ldg(reinterpret_cast<const uint2 *>(wt + (int64_t)j * K + kk));
                const uint32_t b[2] = {vw.x, vw.y};
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) mma_bf16_16816(acc[mt][nt], a[mt], b);
            }
        }
    }
    // Pairwise fold of the 8 warp tiles: 8 -> 4 -> 2 -> 1.
    constexpr int TILE = 16 * MT * 8 * NT;
#pragma unroll
    for (int half = kDownWarps / 2; half >= 1; half >>= 1) {
        if (warp >= half && warp < 2 * half) {
            float *dst = red + (warp - half) * TILE;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int row = 16 * mt + g + 8 * (e >> 1), col = 8 * nt + 2 * c + (e & 1);
                        dst[row * 8 * NT + col] = acc[mt][nt][e];
                    }
        }
        __syncthreads();
        if (warp < half) {
            const float *src = red + warp * TILE;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int row = 16 * mt + g + 8 * (e >> 1), col = 8 * nt + 2 * c + (e & 1);
                        acc[mt][nt][e] = __fadd_rn(acc[mt][nt][e], src[row * 8 * NT + col]);
                    }
        }
        __syncthreads();
    }
    if (warp == 0) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int64_t t = t0 + 16 * mt + g + 8 * (e >> 1);
                    const int j = 8 * nt + 2 * c + (e & 1);
                    if (t < n && j < r) {
                        const float v = acc[mt][nt][e];
                        out[t * r + j] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                        if (out_scaled)
                            out_scaled[t * r + j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(scale, v)));
                    }
                }
    }
}

template <int MT, int NT>
static cudaError_t launch_down_t(const uint16_t *in, int64_t n, int64_t K, const uint16_t *wt, int r, float scale,
                                 uint16_t *out, uint16_t *out_scaled, cudaStream_t st) {
    const size_t smem = (size_t)(kDownWarps / 2) * 16 * MT * 8 * NT * sizeof(float);
    auto kern = lora_down_kernel<MT, NT>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t grid = (n + 16 * MT - 1) / (16 * MT);
    kern<<<(unsigned)grid, kDownWarps * 32, smem, st>>>(in, n, K, wt, r, scale, out, out_scaled);
    note_launch();
    return cudaGetLastError();
}

template <int MT>
static cudaError_t launch_down_mt(const uint16_t *in, int64_t n, int64_t K, const uint16_t *wt, int r, float scale,
                                  uint16_t *out, uint16_t *out_scaled, cudaStream_t st) {
    const int nt = (r + 7) / 8;
    if (nt <= 1) return launch_down_t<MT, 1>(in, n, K, wt, r, scale, out, out_scaled, st);
    if (nt <= 2) return launch_down_t<MT, 2>(in, n, K, wt, r, scale, out, out_scaled, st);
    if (nt <= 4) return launch_down_t<MT, 4>(in, n, K, wt, r, scale, out, out_scaled, st);
    if (nt <= 8) return launch_down_t<MT, 8>(in, n, K, wt, r, scale, out, out_scaled, st);
    return launch_down_t<MT, 16>(in, n, K, wt, r, scale, out, out_scaled, st);
}

cudaError_t launch_lora_down(const uint16_t *in, int64_t n, int64_t K, const uint16_t *wt, int64_t wt_sj,
                             int64_t wt_sk, int r, float scale, uint16_t *out, uint16_t *out_scaled,
                             cudaStream_t st, int num_sms) {
    (void)wt_sj;
    (void)wt_sk;  // wt is always [r][K] row-major here (the caller transposes B once)
    if (n / 32 >= num_sms) return launch_down_mt<2>(in, n, K, wt, r, scale, out, out_scaled, st);
    return launch_down_mt<1>(in, n, K, wt, r, scale, out, out_scaled, st);
}

// ===========================================================================
// tn_reduce: C[m][c] = scale * sum_t P[t][m] Q[t][c], P [n][M], Q [n][N]
// (both row-major bf16), fp32 C.  64x64 output tiles, 32 tokens per step,
// both operands staged with cp.async and read with ldmatrix.trans (the
// reduction index t is the row index of both).  With splits > 1 each z-slice
// of the grid covers an interleaved share of the token steps and writes an
// fp32 partial tile; tn_fold adds the slices in a fixed order.
// ===========================================================================
constexpr int kTnBM = 64, kTnBN = 64, kTnBK = 32, kTnPad = 72;

__global__ void __launch_bounds__(128) tn_reduce_kernel(const uint16_t *__restrict__ P, const uint16_t *__restrict__ Q,
                                                        int64_t n, int64_t M, int64_t N, float scale,
                                                        float *__restrict__ C, float *__restrict__ partials) {
    __shared__ __align__(16) uint16_t Ps[2][kTnBK][kTnPad];
    __shared__ __align__(16) uint16_t Qs[2][kTnBK][kTnPad];
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
        cp_async_commit();
    };

    int64_t step = split;
    if (step < nsteps) load(0, step);
    int buf = 0;
    for (; step < nsteps; step += nsplit) {
        const int64_t next = step + nsplit;
        if (next < nsteps) {
            load(buf ^ 1, next);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
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
        buf ^= 1;
    }

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

int tn_reduce_splits(int64_t n, int64_t M, int64_t N, int num_sms) {
    const int64_t tiles = ((M + kTnBM - 1) / kTnBM) * ((N + kTnBN - 1) / kTnBN);
    const int64_t steps = (n + kTnBK - 1) / kTnBK;
    int64_t splits = 1;
    while (tiles * splits < 2 * num_sms && splits * 2 <= steps && splits < 16) splits *= 2;
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
