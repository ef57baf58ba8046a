// Fused QLoRA forward for decode-sized token counts (n <= 32), one launch.
// HBM-bound: the 4-bit weight is streamed once and never materialised.
//
// Method: "LoRA 与 QLoRA" section QLoRA 1 (4-bit weight -> dequant -> BF16 ->
// GEMM) and section LoRA (y = W0 x + s B(A x), A x formed first);
// jjjymmm.cn "QLoRA" (doubleDequant: restore the block constant, then the
// weight).
//
//   U = X A^T                                    (n x r, fp32 accumulate)
//   Y[t][o] = sum_b ahat[o][b] * sum_{k in b} bf16(c[q[o][k]]) X[t][k]
//             + sum_j bf16(s U)[t][j] B[o][j]
//
// The block constant ahat is applied once per 64-wide block to the block's
// fp32 partial dot product instead of once per weight: the same value as
// X W'^T up to rounding (the codebook entries enter the tensor cores as BF16,
// relative error <= 2^-9, as W' = bf16(ahat c) does in the prefill path), at
// about half the instructions per weight, which is what lets the decode keep
// pace with HBM.
//
// Work split.  A thread-block cluster of S CTAs owns a range of 16-row tiles;
// CTA rank q owns the q-th of S K ranges, so X is read from L2 once per K range
// instead of once per SM.  Inside a CTA, 16 warps take "units" of (tile, K
// sub-range of <= 4 blocks); round k gives warp w the unit 16k + w, and a
// round covers 16 / nsub whole tiles.
//   1. At launch every warp requests the code bytes of its first two units
//      (one 2-D TMA copy each, 16 rows x 128 bytes, into its two-stage ring);
//      the CTA stages its K range of X and builds the decode table.
//   2. U = X A^T is formed once for the grid by UG = 8 extra CTAs that follow
//      the decode clusters and do nothing else: each takes one of 8 K ranges,
//      stores the fp32 part in the workspace and counts itself in; the last of
//      them folds the parts in order into bf16(s U) (and U_out) and raises the
//      ready flag.  The decode CTAs never wait for U before their fold.
//   3. Each round a warp decodes its unit into the register layout of the
//      m16n8k16 A operand (a byte of two codes -> a BF16 pair from the table),
//      multiplies with X per block, scales by ahat, stores the fp32 partial
//      into the shared memory of the CTA that folds the tile (tile i of an
//      epoch goes to rank i % S) and refills its stage.  After an epoch of
//      rounds and one cluster barrier every CTA folds its tiles from its own
//      shared memory in a fixed order (CTA rank, then sub-range), adds
//      bf16(s U) B^T (after a bounded wait on the ready flag) as one more MMA
//      pass and writes Y.  Each decode CTA counts itself out once it has read
//      bf16(s U); the last one resets the workspace counters for the next call,
//      so no memset precedes a launch.
// Decoding: in each 64-wide block, lane (g, c) owns code bytes 8c..8c+7 of rows
// g and g+8; MMA step st uses bytes 2st (k pair "2c") and 2st+1 (k pair
// "2c+8"), and X is read with the same permutation of k, so every product still
// pairs equal k.  The table holds one copy per lane, so any pattern of code
// bytes reads it without bank conflicts.
//
// Every sum is taken in an order fixed by the shape and the cluster size S (the
// host picks S per shape and device), so results do not depend on timing.
// Remote shared-memory accesses are stores only and all land before the
// epoch's cluster barrier.
#include <atomic>
#include <type_traits>

#include "qln_common.cuh"
#include "qln_internal.h"
#include "tc_ptx.cuh"

namespace qln {

constexpr int kDvWarps = 16;
constexpr int kDvThreads = kDvWarps * 32;
constexpr int kDvUnitKb = 4;                  // blocks per unit, at most
constexpr int kDvStageBytes = 16 * 128;       // TMA box: 16 rows x 128 code bytes, 128-byte swizzle
constexpr int kDvTabBytes = 256 * 256;        // per code byte a 256-B row: 32 lanes x BF16 pair, then 128 B of X
constexpr int kDvXMax = 256 * 128;            // X chunk: the second halves of the table rows
constexpr int kDvRingBytes = 2 * kDvWarps * kDvStageBytes;
constexpr int kDvRedBytes = 16384;            // U parts of the warps of a U CTA: (128 / r) x n x r fp32
constexpr int kDvSUBytes = 8192;              // bf16(s U) [8 NT][r]
constexpr int kDvBarBytes = 2 * kDvWarps * 8 + 16;
constexpr size_t kDvSmemMax = 232448;         // per-CTA dynamic shared memory limit of sm_100
constexpr int kDvUParts = 8;                  // CTAs that form U
constexpr uint64_t kDvWaitNs = 2000000000ull;  // bounded waits

struct DvParams {
    const float *absmax;
    const int8_t *qabs;
    bool e4m3;  // qabs holds E4M3 codes (QLN_DQ_E4M3), else int8
    const float *dq_scale;
    const float *dq_mean;
    int64_t rows, cols, KB, T;
    const uint16_t *X;   // [n][cols]
    int n;
    const uint16_t *A;   // [r][cols]
    const uint16_t *B;   // [rows][r]
    int r;
    float s;
    uint16_t *Y;         // [n][rows]
    uint16_t *U_out;     // [n][r] or null
    int *status;         // workspace header: status word, U counter and flag at their offsets
    float *upart;        // [UG][n][r]
    uint16_t *sUg;       // [8 NT][r], rows t >= n zero
    int S, Q, nsub, nkb_max, UG;
    int epoch;                                       // rounds per epoch
    int off_slots, off_su, off_bar;                  // shared-memory layout (bytes)
};

// ---- cluster and memory-model primitives -------------------------------------
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
__device__ __forceinline__ uint32_t dsmem_map(uint32_t saddr, uint32_t rank) {
    uint32_t d;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
    return d;
}
__device__ __forceinline__ void dsmem_st4(uint32_t a, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(int *p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint4 lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ uint4 ldg128(const uint16_t *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

// D = A * B with a zero accumulator in.
__device__ __forceinline__ void mma_bf16_16816_zero(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(0.f));
}

// Block constants of one unit for the lane's two rows (g and g + 8).
struct DvConsts {
    uint32_t raw[kDvUnitKb][2];  // int8 DQ code (sign-extended) or fp32 absmax bits
    float sc[2][2];              // DQ scale of the unit's first and last block, per row
    int lo[2];                   // first block's index within its DQ group, per row
};

template <int NT>  // token tiles of 8: n <= 8 * NT
__global__ void __launch_bounds__(kDvThreads, 1)
nf4_decode_fwd_kernel(const __grid_constant__ CUtensorMap tm_codes, const DvParams p) {
    extern __shared__ __align__(1024) uint8_t dsm[];
    uint8_t *tab = dsm;                                         // table rows; X lines in their second halves
    uint8_t *ring = dsm + kDvTabBytes;                          // [2][16 warps][16 rows][128 B], swizzled
    float *slots = reinterpret_cast<float *>(dsm + p.off_slots);  // pushed partials of one epoch
    uint16_t *sU = reinterpret_cast<uint16_t *>(dsm + p.off_su);  // [8 NT][r]
    const uint32_t bars = smem_u32(dsm + p.off_bar);            // [16 warps][2] mbarriers
    volatile int *flag = reinterpret_cast<volatile int *>(dsm + p.off_bar + 2 * kDvWarps * 8);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int n = p.n, r = p.r, S = p.S, nsub = p.nsub, nkbx = p.nkb_max;
    const int rank = (int)(blockIdx.x % S), cl = (int)(blockIdx.x / S);
    const int64_t cols = p.cols, KB = p.KB;
    const int64_t kb0 = KB * rank / S;
    const int nkb = (int)(KB * (rank + 1) / S - kb0);
    const int64_t t0 = p.T * cl / p.Q, t1 = p.T * (cl + 1) / p.Q;
    const int tpr = kDvWarps / nsub;  // tiles per round
    const int rounds = (int)((t1 - t0 + tpr - 1) / tpr);
    const int sub = warp % nsub;
    const int sb0 = nkb * sub / nsub, snb = nkb * (sub + 1) / nsub - sb0;  // <= 4 blocks
    const bool dq = p.qabs != nullptr;
    int *ucount = reinterpret_cast<int *>(reinterpret_cast<char *>(p.status) + kWsUCountOffset);
    int *uflag = reinterpret_cast<int *>(reinterpret_cast<char *>(p.status) + kWsUFlagOffset);
    int *udone = reinterpret_cast<int *>(reinterpret_cast<char *>(p.status) + kWsDoneOffset);
    const bool ucta = (int)blockIdx.x >= p.Q * S;
    const uint32_t wbar = bars + (uint32_t)warp * 16u;  // stage st's barrier at + 8 st
    if (!ucta) {
        // Before the dependency wait only shared memory and the launch's own
        // parameters are touched, nothing an earlier kernel on the stream can
        // change: the barriers and the decode table are ready while that
        // kernel finishes.
        if (lane == 0) {
            tc::mbar_init(wbar, 1);
            tc::mbar_init(wbar + 8, 1);
            tc::mbar_fence_init();
            tc::tma_prefetch_map(&tm_codes);
        }
        {   // table: warp w writes the rows e = 16 k + w, so c[e >> 4] = c[k] is a constant
            float clo = 0.f;
#pragma unroll
            for (int q = 0; q < 16; ++q)
                if (q == warp) clo = nf4_value(q);
#pragma unroll
            for (int k = 0; k < 16; ++k)
                *reinterpret_cast<uint32_t *>(tab + (16 * k + warp) * 256 + lane * 4) =
                    pack_bf16x2(nf4_value(k), clo);
        }
        __syncwarp();
    }
    pdl_wait();  // X, the weight and the workspace may all be touched by the previous kernel on the stream
    pdl_trigger();

    // ---- U CTAs: U = X A^T, once for the grid ------------------------------------
    if (ucta) {
        const int u = (int)blockIdx.x - p.Q * S;  // 0 .. UG-1; U clusters hold U CTAs only
        const int64_t ub0 = KB * u / p.UG, ub1 = KB * (u + 1) / p.UG;  // this CTA's K range of U
        const int njt = r / 8, nsubu = kDvWarps / njt;
        const int jt = warp % njt, subu = warp / njt;
        const int mtu = (n + 15) / 16;
        float *red = reinterpret_cast<float *>(dsm);  // [nsubu][n][r]
        if (subu < nsubu) {
            const int64_t b0 = ub0 + (ub1 - ub0) * subu / nsubu, b1 = ub0 + (ub1 - ub0) * (subu + 1) / nsubu;
            float acc_u[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc_u[mt][e] = 0.f;
            const uint16_t *arow = p.A + (int64_t)(8 * jt + g) * cols + 16 * c;
            for (int64_t b = b0; b < b1; ++b) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int64_t k0 = b * 64 + 8 * hh;  // + 16 c inside arow / the X rows
                    const uint4 av = ldg128(arow + k0);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        if (mt < mtu) {
                            const int ta = 16 * mt + g, tb = ta + 8;
                            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                            const uint4 xa = ta < n ? ldg128(p.X + (int64_t)ta * cols + k0 + 16 * c) : z;
                            const uint4 xb = tb < n ? ldg128(p.X + (int64_t)tb * cols + k0 + 16 * c) : z;
                            const uint32_t a0[4] = {xa.x, xb.x, xa.y, xb.y}, q0[2] = {av.x, av.y};
                            mma_bf16_16816(acc_u[mt], a0, q0);
                            const uint32_t a1[4] = {xa.z, xb.z, xa.w, xb.w}, q1[2] = {av.z, av.w};
                            mma_bf16_16816(acc_u[mt], a1, q1);
                        }
                    }
                }
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = 16 * mt + g + 8 * (e >> 1), j = 8 * jt + 2 * c + (e & 1);
                    if (mt < mtu && t < n) red[(subu * n + t) * r + j] = acc_u[mt][e];
                }
        }
        __syncthreads();
        float *up = p.upart + (int64_t)u * n * r;
        for (int i = tid; i < n * r; i += kDvThreads) {
            float v = 0.f;
            for (int q = 0; q < nsubu; ++q) v = __fadd_rn(v, red[q * n * r + i]);
            __stcg(up + i, v);
        }
        __threadfence();
        __syncthreads();
        volatile int *last = reinterpret_cast<volatile int *>(dsm + kDvRedBytes);
        if (tid == 0) *last = atomicAdd(ucount, 1) == p.UG - 1;
        __syncthreads();
        if (*last) {  // every part is published: fold them in order
            __threadfence();
            for (int i = tid; i < 8 * NT * r; i += kDvThreads) {
                const int t = i / r;
                float v = 0.f;
                if (t < n)
                    for (int q = 0; q < p.UG; ++q) v = __fadd_rn(v, __ldcg(p.upart + (int64_t)q * n * r + i));
                p.sUg[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(p.s, v)));
                if (p.U_out && t < n) p.U_out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            }
            __threadfence();
            __syncthreads();
            if (tid == 0) st_release_gpu(uflag, 1);
        }
        return;
    }

    if (blockIdx.x == 0 && tid == 0) *p.status = QLN_OK;
    cluster_arrive_relaxed();  // "started": no peer writes here before every CTA of the cluster runs

    // ---- 1. requests: two units of codes per warp, X chunk, constants --------------
    const uint32_t ring_s = smem_u32(ring) + (uint32_t)(warp * kDvStageBytes);  // stage st at + st * 16 stages
    auto issue_codes = [&](int k, int st) {  // round k's unit of this warp -> stage st
        const int64_t tl = t0 + (int64_t)(kDvWarps * k + warp) / nsub;
        if (k < rounds && tl < t1 && lane == 0) {
            tc::fence_proxy_async_smem();  // the stage's earlier reads come before the copy
            tc::mbar_arrive_expect_tx(wbar + 8u * st, (uint32_t)kDvStageBytes);
            tc::tma_load_2d(ring_s + (uint32_t)(st * kDvWarps * kDvStageBytes), &tm_codes,
                            (int32_t)((kb0 + sb0) * 32), (int32_t)(tl * 16), wbar + 8u * st);
        }
    };
    auto load_consts = [&](int k, DvConsts &o) {
        const int64_t tl = t0 + (int64_t)(kDvWarps * k + warp) / nsub;
        if (k < rounds && tl < t1) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t jb0 = (tl * 16 + g + 8 * h) * KB + kb0 + sb0;
                if (dq) {
#pragma unroll
                    for (int b = 0; b < kDvUnitKb; ++b)
                        if (b < snb) o.raw[b][h] = (uint32_t)(int)__ldg(p.qabs + jb0 + b);
                    o.sc[h][0] = __ldg(p.dq_scale + (jb0 >> 8));
                    o.sc[h][1] = __ldg(p.dq_scale + ((jb0 + snb - 1) >> 8));
                    o.lo[h] = (int)(jb0 & 255);
                } else {
#pragma unroll
                    for (int b = 0; b < kDvUnitKb; ++b)
                        if (b < snb) o.raw[b][h] = __float_as_uint(__ldg(p.absmax + jb0 + b));
                }
            }
        }
    };
    issue_codes(0, 0);
    issue_codes(1, 1);
    // X chunk: line (token t, block bl) at row t * nkbx + bl, second half; 16-B chunks swizzled by t & 1
    for (int t = warp; t < 8 * NT; t += kDvWarps)
        for (int j = lane; j < nkbx * 8; j += 32) {
            uint8_t *dst = tab + (t * nkbx + (j >> 3)) * 256 + 128 + (((j & 7) ^ (t & 1)) << 4);
            if (t < n && j < nkb * 8)
                cp_async16(dst, p.X + (int64_t)t * cols + kb0 * 64 + j * 8);
            else
                *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
    cp_async_commit();
    DvConsts kc;
    load_consts(0, kc);
    const float mu = dq ? __ldg(p.dq_mean) : 0.f;
    {   // the adapter rows this cluster folds with, into L2 (split over the ranks)
        const char *bb = reinterpret_cast<const char *>(p.B + t0 * 16 * r);
        const int64_t lines = ((t1 - t0) * 16 * r * 2 + 127) / 128;
        for (int64_t l = rank * kDvThreads + tid; l < lines; l += (int64_t)S * kDvThreads)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(bb + l * 128));
    }
    cp_async_wait<0>();  // X
    __syncthreads();
    cluster_wait();      // every CTA of the cluster has started

    // ---- 3. rounds ------------------------------------------------------------------
    const uint32_t lane4 = (uint32_t)lane * 4u;
    const uint32_t slots_s = smem_u32(slots);
    uint32_t xoff[NT];  // this lane's X fragment, block 0 of the unit, hh = 0
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int t = 8 * nt + g;
        xoff[nt] = (uint32_t)((t * nkbx + sb0) * 256 + 128 + (((2 * c) ^ (t & 1)) << 4));
    }
    // n <= 8: the warp's X fragments for its whole K sub-range stay in registers
    // (the sub-range is the same in every round)
    uint4 xr[kDvUnitKb][2];
    if constexpr (NT == 1) {
#pragma unroll
        for (int b = 0; b < kDvUnitKb; ++b)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                xr[b][hh] = b < snb ? lds128(tab + ((xoff[0] + b * 256) ^ (uint32_t)(hh << 4))) : make_uint4(0u, 0u, 0u, 0u);
    }
    int e0 = 0;  // first round of the current epoch
    for (int k = 0; k < rounds; ++k) {
        const int64_t tile = t0 + (int64_t)(kDvWarps * k + warp) / nsub;
        DvConsts kn;
        load_consts(k + 1, kn);
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
        if (tile < t1) {
            if (!tc::mbar_wait_bounded(wbar + 8u * (k & 1), (uint32_t)((k >> 1) & 1), nullptr, kDvWaitNs))
                atomicExch(p.status, (int)QLN_ERR_TIMEOUT);
            const uint8_t *cs = ring + (k & 1) * (kDvWarps * kDvStageBytes) + warp * kDvStageBytes + g * 128 + (c & 1) * 8;
            auto unit = [&](auto full_tag) {
                constexpr bool kFull = decltype(full_tag)::value;
#pragma unroll
                for (int b = 0; b < kDvUnitKb; ++b) {
                    if (kFull || b < snb) {
                        const int ch = ((2 * b + (c >> 1)) ^ g) << 4;  // 16-B chunk of block b, swizzled by row & 7
                        uint2 cw[2];
                        cw[0] = *reinterpret_cast<const uint2 *>(cs + ch);
                        cw[1] = *reinterpret_cast<const uint2 *>(cs + 8 * 128 + ch);
                        float ah[2];
    #pragma unroll
                        for (int h = 0; h < 2; ++h)
                            ah[h] = dq ? dq_restore(kc.raw[b][h], (kc.lo[h] + b >= 256) ? kc.sc[h][1] : kc.sc[h][0], mu, p.e4m3)
                                       : __uint_as_float(kc.raw[b][h]);
                        float tmp[NT][4];
    #pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            uint4 xv[NT];
    #pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                if constexpr (NT == 1)
                                    xv[nt] = xr[b][hh];
                                else
                                    xv[nt] = lds128(tab + ((xoff[nt] + b * 256) ^ (uint32_t)(hh << 4)));
                            }
    #pragma unroll
                            for (int sp = 0; sp < 2; ++sp) {
                                const int st = 2 * hh + sp;
                                uint32_t a[4];
    #pragma unroll
                                for (int q = 0; q < 4; ++q) {  // (row g, 2c) (row g+8, 2c) (row g, 2c+8) (row g+8, 2c+8)
                                    const int h = q & 1, bi = 2 * st + (q >> 1);  // byte of the lane's share
                                    const uint32_t word = (bi < 4) ? cw[h].x : cw[h].y;
                                    // table row of the code byte, this lane's column: byte * 256 + lane * 4
                                    const uint32_t off = prmt(word, lane4, 0x5504u | ((uint32_t)(bi & 3) << 4));
                                    a[q] = *reinterpret_cast<const uint32_t *>(tab + off);
                                }
    #pragma unroll
                                for (int nt = 0; nt < NT; ++nt) {
                                    const uint32_t bb[2] = {sp ? xv[nt].z : xv[nt].x, sp ? xv[nt].w : xv[nt].y};
                                    if (st == 0)
                                        mma_bf16_16816_zero(tmp[nt], a, bb);
                                    else
                                        mma_bf16_16816(tmp[nt], a, bb);
                                }
                            }
                        }
    #pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            acc[nt][0] = __fmaf_rn(ah[0], tmp[nt][0], acc[nt][0]);
                            acc[nt][1] = __fmaf_rn(ah[0], tmp[nt][1], acc[nt][1]);
                            acc[nt][2] = __fmaf_rn(ah[1], tmp[nt][2], acc[nt][2]);
                            acc[nt][3] = __fmaf_rn(ah[1], tmp[nt][3], acc[nt][3]);
                        }
                    }
                }
    
            };
            if (snb == kDvUnitKb)
                unit(std::true_type{});
            else
                unit(std::false_type{});
        }
        __syncwarp();  // every lane is done with this stage
        issue_codes(k + 2, k & 1);
        kc = kn;

        if (k == e0 && k > 0) cluster_wait();  // the last epoch's slots are folded everywhere
        if (tile < t1) {  // push the partial to the CTA that folds this tile
            const int i = (int)(tile - (t0 + (int64_t)kDvWarps * e0 / nsub));  // tile within the epoch
            const int owner = i % S, li = i / S;
            // owner's slot layout: [tile li][rank][sub][NT][32 lanes] float4
            const uint32_t a0 = slots_s + (uint32_t)(((((li * S + rank) * nsub + sub) * NT) * 32 + lane) * 16);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                dsmem_st4(dsmem_map(a0 + nt * 512, (uint32_t)owner),
                          make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]));
        }
        if (k - e0 + 1 < p.epoch && k + 1 < rounds) continue;

        // ---- end of an epoch: every partial has been pushed; fold the tiles owned here --
        const int64_t et0 = t0 + (int64_t)kDvWarps * e0 / nsub;
        const int64_t et1e = t0 + (int64_t)kDvWarps * (k + 1) / nsub;
        const int m = (int)((et1e < t1 ? et1e : t1) - et0);
        if (e0 == 0) {   // bf16(s U), once the U CTAs have folded it (long done by now, as a rule)
            if (tid == 0) {
                bool ok = ld_acquire_gpu(uflag) != 0;
                if (!ok) {
                    const uint64_t tw = tc::global_timer_ns();
                    for (uint32_t it = 0; !ok; ++it) {
                        ok = ld_acquire_gpu(uflag) != 0;
                        if (!ok && (it & 63u) == 63u && tc::global_timer_ns() - tw > kDvWaitNs) break;
                    }
                }
                if (!ok) atomicExch(p.status, (int)QLN_ERR_TIMEOUT);
                *flag = ok;
            }
            __syncthreads();
            const bool ok = *flag != 0;
            for (int i = tid; i < 8 * NT * r / 2; i += kDvThreads)
                reinterpret_cast<uint32_t *>(sU)[i] = ok ? __ldcg(reinterpret_cast<const unsigned int *>(p.sUg) + i) : 0u;
            if (tid == 0 && atomicAdd(udone, 1) == p.Q * S - 1) {
                // every decode CTA has read bf16(s U): leave the counters at zero for the next call
                *ucount = 0;
                *uflag = 0;
                *udone = 0;
            }
        }
        // B fragments of this warp's first tile of the epoch, requested before the barrier
        const int i0 = warp * S + rank;
        uint32_t ba[2][4];
#pragma unroll
        for (int js = 0; js < 2; ++js)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int64_t row = (et0 + (i0 < m ? i0 : 0)) * 16 + g + 8 * (q & 1);
                const int j = 16 * js + 2 * c + 8 * (q >> 1);
                ba[js][q] = (i0 < m && j < r) ? __ldg(reinterpret_cast<const uint32_t *>(p.B + row * r + j)) : 0u;
            }
        cluster_arrive();
        cluster_wait();  // every partial of the epoch has landed here (and sU is in place)
        for (int i = warp * S + rank; i < m; i += kDvWarps * S) {
            const int64_t row0 = (et0 + i) * 16;
            const int li = i / S;
            float f[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) f[nt][e] = 0.f;
            // partials in the order (CTA rank, sub-range)
            const float4 *sl = reinterpret_cast<const float4 *>(slots) + ((li * S * nsub) * NT) * 32 + lane;
            for (int q = 0; q < S * nsub; ++q) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float4 v = sl[(q * NT + nt) * 32];
                    f[nt][0] = __fadd_rn(f[nt][0], v.x);
                    f[nt][1] = __fadd_rn(f[nt][1], v.y);
                    f[nt][2] = __fadd_rn(f[nt][2], v.z);
                    f[nt][3] = __fadd_rn(f[nt][3], v.w);
                }
            }
            for (int j0 = 0; j0 < r; j0 += 16) {
                uint32_t a[4];
                if (i == i0 && j0 < 32) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) a[q] = j0 == 0 ? ba[0][q] : ba[1][q];
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int64_t row = row0 + g + 8 * (q & 1);
                        const int j = j0 + 2 * c + 8 * (q >> 1);
                        a[q] = (j < r) ? __ldg(reinterpret_cast<const uint32_t *>(p.B + row * r + j)) : 0u;
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int t = 8 * nt + g;
                    uint32_t bb[2];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int j = j0 + 2 * c + 8 * q;
                        bb[q] = (j < r) ? *reinterpret_cast<const uint32_t *>(sU + t * r + j) : 0u;
                    }
                    mma_bf16_16816(f[nt], a, bb);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = 8 * nt + 2 * c + (e & 1);
                    const int64_t row = row0 + g + 8 * (e >> 1);
                    if (t < n) p.Y[(int64_t)t * p.rows + row] = __bfloat16_as_ushort(__float2bfloat16_rn(f[nt][e]));
                }
        }
        e0 = k + 1;
        if (e0 < rounds) cluster_arrive();  // this CTA's slots may be refilled
    }
}

// Shared-memory layout and split of one launch.
struct DvLayout {
    int S, nsub, NT, nkb_max, epoch;
    int off_slots, off_su, off_bar;
    size_t smem;
    bool ok;
};

static int dv_a128(int64_t x) { return (int)((x + 127) & ~int64_t(127)); }

static DvLayout dv_layout(int64_t KB, int64_t n, int r, int S) {
    DvLayout L;
    L.S = S;
    L.NT = (int)((n + 7) / 8);
    L.nkb_max = (int)((KB + S - 1) / S);
    L.nsub = 1;
    while (L.nsub * kDvUnitKb < L.nkb_max) L.nsub *= 2;
    const int64_t xbytes = (int64_t)8 * L.NT * L.nkb_max * 128;
    L.ok = false;
    L.epoch = 0;
    L.off_slots = L.off_su = L.off_bar = 0;
    L.smem = 0;
    if (S > KB || xbytes > kDvXMax || L.nsub > kDvWarps) return L;  // (a round must hold whole tiles)
    // an owner parks, per tile it folds, S x nsub partials; with tile i of an epoch
    // going to rank i % S the busiest owner folds ceil(m / S) tiles, so the slots
    // hold (epoch * tiles per round + S - 1) tiles' worth of partials
    const int64_t per_tile = (int64_t)L.nsub * L.NT * 512;
    const int64_t tpr = kDvWarps / L.nsub;
    const int64_t fixed = (int64_t)kDvTabBytes + kDvRingBytes + kDvSUBytes + kDvBarBytes;
    const int64_t room = (int64_t)kDvSmemMax - fixed - (S - 1) * per_tile;
    int64_t ep = room > 0 ? room / (tpr * per_tile) : 0;
    if (ep > 16) ep = 16;
    L.epoch = (int)ep;
    L.off_slots = kDvTabBytes + kDvRingBytes;
    L.off_su = L.off_slots + dv_a128((ep * tpr + S - 1) * per_tile);
    L.off_bar = L.off_su + kDvSUBytes;
    L.smem = (size_t)L.off_bar + kDvBarBytes;
    L.ok = S <= KB && xbytes <= kDvXMax && L.nsub <= kDvWarps && ep >= 1 && L.smem <= kDvSmemMax &&
           (int64_t)(kDvWarps / (r / 8)) * n * r * 4 <= kDvRedBytes && (int64_t)8 * L.NT * r * 2 <= kDvSUBytes;
    return L;
}

bool nf4_gemv_supported(const qln_nf4_weight *w, int64_t n, int r) {
    if (n < 1 || n > 32 || (w->rows % 16) != 0 || (w->cols % 64) != 0 || (r % 8) != 0 || r < 8 || r > 128)
        return false;
    for (int S = 1; S <= 8; S *= 2)
        if (dv_layout(w->cols / 64, n, r, S).ok) return true;
    return false;
}

size_t nf4_gemv_ws_bytes(int64_t n, int r) {
    const int64_t NT = (n + 7) / 8;
    return (size_t)dv_a128((int64_t)kDvUParts * n * r * 4) + (size_t)dv_a128(8 * NT * r * 2);
}

template <int NT>
static cudaError_t dv_max_clusters(int S, int *out) {
    // per device and cluster size: co-resident clusters (0 = not asked yet);
    // host threads may launch at once, so the entries are atomics
    static std::atomic<int> cache[64][9];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) {
        const int c = cache[dev][S].load(std::memory_order_relaxed);
        if (c > 0) {
            *out = c;
            return cudaSuccess;
        }
    }
    e = cudaFuncSetAttribute(nf4_decode_fwd_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDvSmemMax);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t q = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    q.gridDim = dim3((unsigned)S);
    q.blockDim = dim3(kDvThreads);
    q.dynamicSmemBytes = kDvSmemMax;
    q.attrs = attr;
    q.numAttrs = 1;
    int nclus = 0;
    e = cudaOccupancyMaxActiveClusters(&nclus, (const void *)nf4_decode_fwd_kernel<NT>, &q);
    if (e != cudaSuccess) return e;
    if (nclus < 1) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 64) cache[dev][S].store(nclus, std::memory_order_relaxed);
    *out = nclus;
    return cudaSuccess;
}

template <int NT>
static cudaError_t launch_dv(DvParams p, const qln_nf4_weight *w, cudaStream_t st) {
    // cluster size: the one that keeps the most SMs busy (ties: the larger, for less X traffic)
    const int64_t KB = p.cols / 64, T = p.rows / 16;
    DvLayout best_L{};
    int64_t best = -1, bestQ = 0;
    for (int S = 8; S >= 1; S /= 2) {
        const DvLayout L = dv_layout(KB, p.n, p.r, S);
        if (!L.ok) continue;
        int nclus = 0;
        cudaError_t e = dv_max_clusters<NT>(S, &nclus);
        if (e != cudaSuccess) return e;
        // the decode clusters leave room for the 8 / S clusters of U CTAs
        int64_t Q = nclus - kDvUParts / S;
        if (Q > T) Q = T;
        if ((Q + kDvUParts / S) * S > kDvPlanSms) Q = kDvPlanSms / S - kDvUParts / S;
        if (Q < 1) continue;
        if (Q * S > best) {
            best = Q * S;
            best_L = L;
            bestQ = Q;
        }
    }
    if (best < 0) return cudaErrorInvalidConfiguration;
    const DvLayout &L = best_L;
    CUtensorMap tm;
    if (!make_tensor_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, (uint64_t)(p.cols / 2), (uint64_t)p.rows,
                            128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    p.KB = KB;
    p.T = T;
    p.S = L.S;
    p.Q = (int)bestQ;
    p.nsub = L.nsub;
    p.nkb_max = L.nkb_max;
    p.epoch = L.epoch;
    p.UG = kDvUParts;
    p.off_slots = L.off_slots;
    p.off_su = L.off_su;
    p.off_bar = L.off_bar;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)L.S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // the kernel waits before any global access
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)((bestQ + kDvUParts / L.S) * L.S));
    cfg.blockDim = dim3(kDvThreads);
    cfg.dynamicSmemBytes = L.smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, nf4_decode_fwd_kernel<NT>, tm, p);
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_nf4_gemv(const qln_nf4_weight *w, const uint16_t *X, int64_t n, const uint16_t *A,
                            const uint16_t *B, int r, float s, uint16_t *Y, uint16_t *U_out, void *ws,
                            cudaStream_t st) {
    DvParams p;
    p.absmax = w->absmax;
    p.qabs = w->qabs;
    p.e4m3 = w->dq_format == QLN_DQ_E4M3;
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
    char *wsb = reinterpret_cast<char *>(ws);
    p.status = reinterpret_cast<int *>(wsb);
    p.upart = reinterpret_cast<float *>(wsb + kWsHeaderBytes);
    p.sUg = reinterpret_cast<uint16_t *>(wsb + kWsHeaderBytes + dv_a128((int64_t)kDvUParts * n * r * 4));
    switch ((n + 7) / 8) {
        case 1: return launch_dv<1>(p, w, st);
        case 2: return launch_dv<2>(p, w, st);
        case 3: return launch_dv<3>(p, w, st);
        default: return launch_dv<4>(p, w, st);
    }
}

}  // namespace qln
