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
// The block constant ahat scales the block's fp32 partial dot product once
// instead of each weight: the same value as X W'^T up to rounding (the book
// entries enter the tensor cores as BF16, relative error <= 2^-9, as
// W' = bf16(ahat c) does in the prefill path) at about half the instructions
// per weight.
//
// Work split.  A cluster of S CTAs (one per SM) owns a range of m 16-row
// tiles; CTA rank q owns the q-th of S K ranges of every tile, so each CTA
// stages only its K range of X.  Inside a CTA the K range is cut into nsub
// sub-ranges and a warp owns the items (tile, sub-range) with item index
// congruent to its warp index mod 16: its sub-range is fixed and its tiles are
// every (16 / nsub)-th one.  After the weight tiles come ceil(r / 16) "A
// tiles": the same product with rows of A in place of decoded weights, which
// gives each cluster its own U = X A^T without any other cluster.
//   1. At launch every warp requests, by 2-D TMA (16 rows x 128 code bytes,
//      128-byte swizzle), the first RS boxes of its item list into a private
//      ring; a box that has been decoded is refilled with the box RS places
//      later.  For the decode layer (4096 x 4096) every box of the CTA is
//      requested before the first one is decoded.
//   2. Decode: a byte of two codes indexes a 64 KB shared table holding one
//      BF16 pair (c[hi], c[lo]) per lane, so any pattern of code bytes reads it
//      without bank conflicts; the pair is the A operand of an m16n8k16 MMA
//      whose B operand is X from shared memory.  One FFMA per output element
//      scales a block's partial by ahat.
//   3. Each finished item's fp32 partial (16 rows x 8 NT tokens) is stored
//      into the shared memory of the CTA that folds the tile (tile i goes to
//      rank i % S); A-tile partials go to every rank.  After one cluster
//      barrier each CTA folds U in a fixed order (rank, then sub-range),
//      keeps bf16(s U), folds the tiles it owns in the same order, adds
//      bf16(s U) B^T as one more MMA pass and writes Y.  A layer whose
//      partials do not fit in shared memory at once is done in epochs of E
//      tiles, with one more cluster barrier between epochs.
// Every sum is taken in an order fixed by the shape and the plan (S, nsub,
// E), so results do not depend on timing.  No CTA waits on another cluster;
// inside a cluster every CTA is co-scheduled by the hardware.
// Decoding layout: in each 64-wide block, lane (g, c) owns code bytes
// 8c..8c+7 of rows g and g+8; MMA step st uses bytes 2st (k pair "2c") and
// 2st+1 (k pair "2c+8"), and X and A are read with the same permutation of k,
// so every product still pairs equal k.
#include <atomic>

#include "qln_common.cuh"
#include "qln_internal.h"
#include "tc_ptx.cuh"

namespace qln {

constexpr int kDfWarps = 16;
constexpr int kDfThreads = kDfWarps * 32;
constexpr int kDfBoxBytes = 16 * 128;     // one TMA box: 16 rows x 128 code bytes (4 blocks)
constexpr int kDfTabBytes = 256 * 256;    // per code byte a 256-B row: 32 lanes x BF16 pair, then one X line
constexpr int kDfXLines = 256;            // X lines (token, block), in the second halves of the table rows
constexpr int kDfPartBytes = 512;         // one partial: 32 lanes x float4 (16 rows x 8 tokens)
constexpr size_t kDfSmemMax = 232448;     // per-CTA dynamic shared memory limit of sm_100
constexpr uint64_t kDfWaitNs = 2000000000ull;  // bounded waits

struct DfParams {
    const float *absmax;
    const int8_t *qabs;
    bool e4m3;  // qabs holds E4M3 codes (QLN_DQ_E4M3), else int8
    const float *dq_scale;
    const float *dq_mean;
    int64_t rows, cols;
    int KB, T;           // 64-blocks per row, 16-row tiles
    const uint16_t *X;   // [n][cols]
    int n;
    const uint16_t *A;   // [r][cols]
    const uint16_t *B;   // [rows][r]
    int r;
    float s;
    uint16_t *Y;         // [n][rows]
    uint16_t *U_out;     // [n][r] or null
    int *status;         // device status word
    int S, Q, nsub, nsubA, nkb_max, RS, E, JT;
    int off_ring, off_slots, off_uslots, off_sb, off_su, off_ah, off_bar;  // shared-memory layout (bytes)
};

// ---- cluster and memory-model primitives -------------------------------------
__device__ __forceinline__ void cl_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cl_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cl_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
__device__ __forceinline__ uint32_t cl_map(uint32_t saddr, uint32_t rank) {
    uint32_t d;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
    return d;
}
__device__ __forceinline__ void cl_st4(uint32_t a, const float (&v)[4]) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v[0]), "f"(v[1]), "f"(v[2]),
                 "f"(v[3])
                 : "memory");
}
__device__ __forceinline__ uint4 df_lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ uint4 df_ldg128(const uint16_t *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

// D = A * B with a zero accumulator in.
__device__ __forceinline__ void df_mma_zero(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(0.f));
}

template <int NT>  // token tiles of 8: n <= 8 * NT
__global__ void __launch_bounds__(kDfThreads, 1)
nf4_decode_fwd_kernel(const __grid_constant__ CUtensorMap tm_codes, const DfParams p) {
    extern __shared__ __align__(1024) uint8_t dsm[];
    uint8_t *tab = dsm;  // table rows; X lines in their second halves
    const uint16_t *sB = reinterpret_cast<const uint16_t *>(dsm + p.off_sb);  // [owned tile][16][r]
    uint16_t *sU = reinterpret_cast<uint16_t *>(dsm + p.off_su);              // [8 NT][r] bf16(s U)
    float *sAh = reinterpret_cast<float *>(dsm + p.off_ah);  // restored block constants [tile][16][nkb_max + 1]

    // All index arithmetic is 32-bit (the host checks that every block index
    // and tile row fits); 64-bit values appear only in global offsets.
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int n = p.n, r = p.r, S = p.S, nsub = p.nsub, nsubA = p.nsubA, nkbx = p.nkb_max, RS = p.RS, E = p.E;
    const int KB = p.KB, T = p.T, Q = p.Q;
    const int rank = (int)blockIdx.x % S, cl = (int)blockIdx.x / S;
    const int kb0 = KB * rank / S, nkb = KB * (rank + 1) / S - kb0;
    const int t0 = T * cl / Q, m = T * (cl + 1) / Q - t0;
    const int nep = (m + E - 1) / E;
    const int El = m - (nep - 1) * E;  // tiles of the last epoch
    const int L = kDfWarps / nsub, sub = warp % nsub, ts0 = warp / nsub;
    const int sb0 = nkb * sub / nsub, snb = nkb * (sub + 1) / nsub - sb0;
    const int nbox = (snb + 3) >> 2;
    // this warp's weight items: cntf per full epoch, cntl in the last one
    const int cntf = E > ts0 ? (E - ts0 + L - 1) / L : 0;
    const int cntl = El > ts0 ? (El - ts0 + L - 1) / L : 0;
    const int nboxes = ((nep - 1) * cntf + cntl) * nbox;
    const bool dq = p.qabs != nullptr;
    const uint32_t ring_w = smem_u32(dsm + p.off_ring) + (uint32_t)(warp * RS * kDfBoxBytes);
    const uint32_t bar_w = smem_u32(dsm + p.off_bar) + (uint32_t)(warp * RS * 8);
    const uint32_t slots_s = smem_u32(dsm + p.off_slots), uslots_s = smem_u32(dsm + p.off_uslots);
    const int ahs = nkbx + 1;

    // Before the dependency wait only shared memory and the launch's own
    // parameters are touched, nothing an earlier kernel on the stream can
    // change: barriers and the decode table are ready while that kernel ends.
    cl_arrive_relaxed();  // this CTA runs: peers may store into it once they have waited
    if (lane == 0) {
        for (int s = 0; s < RS; ++s) tc::mbar_init(bar_w + 8u * s, 1);
        tc::mbar_fence_init();
        tc::tma_prefetch_map(&tm_codes);
    }
    {   // table: warp w writes the rows e = 16 k + w, so c[e & 15] = c[w] is a constant
        const float clo = nf4_value(warp);
#pragma unroll
        for (int k = 0; k < 16; ++k)  // k is a compile-time index: c[k] is a literal
            *reinterpret_cast<uint32_t *>(tab + (16 * k + warp) * 256 + lane * 4) = pack_bf16x2(nf4_value(k), clo);
    }
    __syncwarp();

    // The boxes of this warp's list are requested in order: box k goes to ring
    // slot k % RS.  The cursor (epoch ie, item iu within it, box ig within the
    // item, slot is) follows the list without divisions.
    int ik = 0, ie = 0, iu = 0, ig = 0, is = 0;
    auto issue_next = [&]() {
        if (ik < nboxes && lane == 0) {
            const int tile = t0 + ie * E + ts0 + L * iu;
            tc::fence_proxy_async_smem();  // the slot's earlier reads come before the copy
            tc::mbar_arrive_expect_tx(bar_w + 8u * is, (uint32_t)kDfBoxBytes);
            tc::tma_load_2d(ring_w + (uint32_t)(is * kDfBoxBytes), &tm_codes, (kb0 + sb0 + 4 * ig) * 32, tile * 16,
                            bar_w + 8u * is);
        }
        ++ik;
        if (++is == RS) is = 0;
        if (++ig == nbox) {
            ig = 0;
            if (++iu == cntf) {
                iu = 0;
                ++ie;
            }
        }
    };

    // adapter rows B of the tiles this CTA folds in epoch e (tile ts = li * S + rank)
    auto stage_b = [&](int e) {
        const int Ee = e + 1 < nep ? E : El;
        const int nown = Ee > rank ? (Ee - rank + S - 1) / S : 0;
        const int rch = r / 8;  // 16-byte chunks per B row
#pragma unroll 1
        for (int i = tid; i < nown * 16 * rch; i += kDfThreads) {
            const int rowi = i / rch, ch = i - rowi * rch, li = rowi >> 4, row = rowi & 15;
            const int64_t grow = (int64_t)(t0 + e * E + li * S + rank) * 16 + row;
            cp_async16(dsm + p.off_sb + (rowi * r + ch * 8) * 2, p.B + grow * r + ch * 8);
        }
    };
    // restored block constants ahat of the epoch's tiles over this CTA's K
    // range (doubleDequant, first step): a thread takes 4 consecutive blocks of
    // one weight row, loads their codes and scales, then restores them
    float mu = 0.f;  // the mean of the constants: read after the dependency wait (below)
    const int nq = (nkb + 3) >> 2;
    auto stage_ah = [&](int e) {
        const int Ee = e + 1 < nep ? E : El;
#pragma unroll 1
        for (int i = tid; i < Ee * 16 * nq; i += kDfThreads) {
            const int tr = i / nq, b0 = (i - tr * nq) * 4;  // tr: tile of the epoch * 16 + row
            const int jb = ((t0 + e * E) * 16 + tr) * KB + kb0 + b0;
            uint32_t raw[4];
            float sc[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (b0 + u < nkb) {
                    if (dq) {
                        raw[u] = (uint32_t)(uint8_t)__ldg(p.qabs + jb + u);
                        sc[u] = __ldg(p.dq_scale + ((jb + u) >> 8));
                    } else {
                        raw[u] = __float_as_uint(__ldg(p.absmax + jb + u));
                    }
                }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (b0 + u < nkb)
                    sAh[tr * ahs + b0 + u] = dq ? dq_restore(raw[u], sc[u], mu, p.e4m3) : __uint_as_float(raw[u]);
        }
    };

    // ---- 1. requests: the code boxes first (the longest latency), then X and the
    //         B rows (asynchronous copies), then the block constants, whose loads
    //         this thread waits for -- so all of them are in flight together -------------
    pdl_wait();  // the weight, X, A, B and the workspace may be written by the previous kernel
    pdl_trigger();
    if (dq) mu = __ldg(p.dq_mean);
    if (blockIdx.x == 0 && tid == 0) *p.status = QLN_OK;
#pragma unroll 1
    for (int k = 0; k < RS; ++k) issue_next();
    // X chunk: line (token t, block bl) at row t * nkbx + bl, second half; 16-B chunks swizzled by t & 1
#pragma unroll 1
    for (int t = warp; t < 8 * NT; t += kDfWarps)
#pragma unroll 1
        for (int j = lane; j < nkbx * 8; j += 32) {
            uint8_t *dst = tab + (t * nkbx + (j >> 3)) * 256 + 128 + (((j & 7) ^ (t & 1)) << 4);
            if (t < n && j < nkb * 8)
                cp_async16(dst, p.X + (int64_t)t * p.cols + kb0 * 64 + j * 8);
            else
                *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
    stage_b(0);
    cp_async_commit();
    stage_ah(0);
    cp_async_wait<0>();
    __syncthreads();  // table, X, block constants and the B rows of epoch 0 in place

    // ---- 2. items ---------------------------------------------------------------------------
    const uint32_t lane4 = (uint32_t)lane * 4u;
    uint32_t xoff[NT];  // this lane's X line, block sb0 of its sub-range, 16-B chunk 2c
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int t = 8 * nt + g;
        xoff[nt] = (uint32_t)((t * nkbx + sb0) * 256 + 128 + (((2 * c) ^ (t & 1)) << 4));
    }
    // one 64-wide block: 4 MMA steps per token tile into tmp (A from the decode table
    // or, for A items, straight from registers)
    auto block_mma = [&](uint32_t xb, const uint32_t (&av)[4][4], float (&tmp)[NT][4], bool zero) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint4 xv[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)  // token rows past n are zero: no load
                xv[nt] = 8 * nt + g < n ? df_lds128(tab + ((xoff[nt] + xb) ^ (uint32_t)(hh << 4))) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int sp = 0; sp < 2; ++sp) {
                const int st = 2 * hh + sp;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint32_t bb[2] = {sp ? xv[nt].z : xv[nt].x, sp ? xv[nt].w : xv[nt].y};
                    if (zero && st == 0)
                        df_mma_zero(tmp[nt], av[st], bb);
                    else
                        mma_bf16_16816(tmp[nt], av[st], bb);
                }
            }
        }
    };
    int kbx = 0;  // boxes consumed by this warp
#pragma unroll 1
    for (int e = 0; e < nep; ++e) {
        const int Ee = e + 1 < nep ? E : El;
        // this warp's items: weight tiles ts0, ts0 + L, ...; then, in the first
        // epoch, A items w, w + 16, ... (A tile jt, block sub-range sa of nsubA)
        const int nwi = Ee > ts0 ? (Ee - ts0 + L - 1) / L : 0;
        const int nai = e == 0 && p.JT * nsubA > warp ? (p.JT * nsubA - warp + kDfWarps - 1) / kDfWarps : 0;
        bool waited = false;
#pragma unroll 1
        for (int it = 0; it < nwi + nai; ++it) {
            const bool wt = it < nwi;
            const int ts = ts0 + L * it;                   // weight tile of the epoch (wt)
            const int ja = warp + kDfWarps * (it - nwi);   // A item (!wt)
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[nt][q] = 0.f;
            if (wt) {
                // ---- a weight tile: decode and multiply, box by box, block by block ----
                const float *ahr = sAh + (ts * 16 + g) * ahs + sb0;  // row g; row g + 8 at + 8 * ahs
#pragma unroll 1
                for (int gb = 0; gb < nbox; ++gb) {
                    const int slot = kbx % RS;
                    const uint32_t bar = bar_w + 8u * slot, par = (uint32_t)((kbx / RS) & 1);
                    if (!tc::mbar_wait_bounded(bar, par, nullptr, kDfWaitNs)) {
                        atomicExch(p.status, (int)QLN_ERR_TIMEOUT);
                        // the copy may still land: wait once more (bounded) before the slot is reused
                        tc::mbar_wait_bounded(bar, par, nullptr, kDfWaitNs);
                    }
                    const uint8_t *cs = dsm + p.off_ring + (warp * RS + slot) * kDfBoxBytes + g * 128 + (c & 1) * 8;
                    const int nbv = min(4, snb - 4 * gb);
#pragma unroll 1
                    for (int b = 0; b < nbv; ++b) {
                        const int ch = ((2 * b + (c >> 1)) ^ g) << 4;  // 16-B chunk of block b, swizzled by row
                        const uint2 cw0 = *reinterpret_cast<const uint2 *>(cs + ch);
                        const uint2 cw1 = *reinterpret_cast<const uint2 *>(cs + 8 * 128 + ch);
                        uint32_t av[4][4];
#pragma unroll
                        for (int st = 0; st < 4; ++st)
#pragma unroll
                            for (int q = 0; q < 4; ++q) {  // (row g, 2c) (row g+8, 2c) (row g, 2c+8) (row g+8, 2c+8)
                                const int bi = 2 * st + (q >> 1);  // byte of the lane's share
                                const uint32_t word = (q & 1) ? (bi < 4 ? cw1.x : cw1.y) : (bi < 4 ? cw0.x : cw0.y);
                                // table row of the code byte, this lane's column: byte * 256 + lane * 4
                                const uint32_t off = prmt(word, lane4, 0x5504u | ((uint32_t)(bi & 3) << 4));
                                av[st][q] = *reinterpret_cast<const uint32_t *>(tab + off);
                            }
                        float tmp[NT][4];
                        block_mma((uint32_t)((4 * gb + b) * 256), av, tmp, true);
                        const float ah0 = ahr[4 * gb + b], ah1 = ahr[8 * ahs + 4 * gb + b];
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            acc[nt][0] = __fmaf_rn(ah0, tmp[nt][0], acc[nt][0]);
                            acc[nt][1] = __fmaf_rn(ah0, tmp[nt][1], acc[nt][1]);
                            acc[nt][2] = __fmaf_rn(ah1, tmp[nt][2], acc[nt][2]);
                            acc[nt][3] = __fmaf_rn(ah1, tmp[nt][3], acc[nt][3]);
                        }
                    }
                    __syncwarp();  // every lane is done with this slot
                    issue_next();  // box kbx + RS
                    ++kbx;
                }
            } else {
                // ---- an A item: rows 16 jt .. 16 jt + 15 of A (zero past r) over blocks
                //      [ab0, ab0 + anb) of this CTA's K range, the same MMA ----
                const int jt = ja / nsubA, sa = ja - jt * nsubA;
                const int ab0 = nkb * sa / nsubA, anb = nkb * (sa + 1) / nsubA - ab0;
                const int j0 = 16 * jt + g, j1 = j0 + 8;  // rows past r read as zero
                const uint16_t *ar0 = p.A + (int64_t)(j0 < r ? j0 : 0) * p.cols + (kb0 + ab0) * 64 + 16 * c;
                const uint16_t *ar1 = p.A + (int64_t)(j1 < r ? j1 : 0) * p.cols + (kb0 + ab0) * 64 + 16 * c;
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                const int xsh = (ab0 - sb0) * 256;  // X lines of block ab0 relative to this lane's xoff
#pragma unroll 1
                for (int b = 0; b < anb; ++b) {
                    const uint4 a00 = j0 < r ? df_ldg128(ar0 + b * 64) : z, a01 = j0 < r ? df_ldg128(ar0 + b * 64 + 8) : z;
                    const uint4 a10 = j1 < r ? df_ldg128(ar1 + b * 64) : z, a11 = j1 < r ? df_ldg128(ar1 + b * 64 + 8) : z;
                    // k pairs 16c + 4 st + {0, 1} and {2, 3}
                    const uint32_t av[4][4] = {{a00.x, a10.x, a00.y, a10.y}, {a00.z, a10.z, a00.w, a10.w},
                                               {a01.x, a11.x, a01.y, a11.y}, {a01.z, a11.z, a01.w, a11.w}};
                    block_mma((uint32_t)(xsh + b * 256), av, acc, false);
                }
            }
            if (!waited) {
                cl_wait();  // every CTA of the cluster runs / has folded the previous epoch
                waited = true;
            }
            if (wt) {  // to the CTA that folds this tile
                const int li = ts / S;
                const uint32_t a0 = slots_s + (uint32_t)(((((li * S + rank) * nsub + sub) * NT) * 32 + lane) * 16);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) cl_st4(cl_map(a0 + nt * kDfPartBytes, (uint32_t)(ts % S)), acc[nt]);
            } else {  // to every CTA of the cluster: slot [jt][rank][sa]
                const int jt = ja / nsubA, sa = ja - jt * nsubA;
                const uint32_t a0 = uslots_s + (uint32_t)(((((jt * S + rank) * nsubA + sa) * NT) * 32 + lane) * 16);
#pragma unroll 1
                for (int q = 0; q < S; ++q)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) cl_st4(cl_map(a0 + nt * kDfPartBytes, (uint32_t)q), acc[nt]);
            }
        }
        if (!waited) cl_wait();
        cp_async_wait<0>();  // this thread's B-row copies of the epoch have landed
        cl_arrive();
        cl_wait();  // every partial of the epoch has landed here
        // ---- 3. folds -----------------------------------------------------------------------
        if (e == 0) {  // U, in the order (rank, sub-range); every CTA keeps bf16(s U)
            const bool wu = p.U_out != nullptr && cl == 0 && rank == 0;
#pragma unroll 1
            for (int pc = warp; pc < p.JT * NT; pc += kDfWarps) {
                const int jt = pc / NT, nt = pc - jt * NT;
                float f[4] = {0.f, 0.f, 0.f, 0.f};
                const float4 *sl = reinterpret_cast<const float4 *>(dsm + p.off_uslots) + (jt * S * nsubA * NT + nt) * 32 + lane;
                const int np = S * nsubA;
#pragma unroll 1
                for (int q0 = 0; q0 < np; q0 += 4) {  // four partials in flight, added in order
                    float4 v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) v[u] = q0 + u < np ? sl[(q0 + u) * NT * 32] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (q0 + u < np) {
                            f[0] = __fadd_rn(f[0], v[u].x);
                            f[1] = __fadd_rn(f[1], v[u].y);
                            f[2] = __fadd_rn(f[2], v[u].z);
                            f[3] = __fadd_rn(f[3], v[u].w);
                        }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // U^T[j][t]: j = 16 jt + g (+8), t = 8 nt + 2c (+1)
                    const int j = 16 * jt + g + 8 * (q >> 1), t = 8 * nt + 2 * c + (q & 1);
                    if (j < r) {
                        sU[t * r + j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(p.s, f[q])));
                        if (wu && t < n) p.U_out[t * r + j] = __bfloat16_as_ushort(__float2bfloat16_rn(f[q]));
                    }
                }
            }
            __syncthreads();
        }
#pragma unroll 1
        for (int li = warp; li * S + rank < Ee; li += kDfWarps) {  // the tiles this CTA owns
            const int64_t row0 = (int64_t)(t0 + e * E + li * S + rank) * 16;
            float f[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) f[nt][q] = 0.f;
            const float4 *sl = reinterpret_cast<const float4 *>(dsm + p.off_slots) + (li * S * nsub * NT) * 32 + lane;
            const int np = S * nsub;
#pragma unroll 1
            for (int q0 = 0; q0 < np; q0 += 4) {  // four partials in flight, added in order
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float4 v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        v[u] = q0 + u < np ? sl[((q0 + u) * NT + nt) * 32] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (q0 + u < np) {
                            f[nt][0] = __fadd_rn(f[nt][0], v[u].x);
                            f[nt][1] = __fadd_rn(f[nt][1], v[u].y);
                            f[nt][2] = __fadd_rn(f[nt][2], v[u].z);
                            f[nt][3] = __fadd_rn(f[nt][3], v[u].w);
                        }
                }
            }
#pragma unroll 1
            for (int j0 = 0; j0 < r; j0 += 16) {
                uint32_t a[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int row = g + 8 * (q & 1), j = j0 + 2 * c + 8 * (q >> 1);
                    a[q] = j < r ? *reinterpret_cast<const uint32_t *>(sB + (li * 16 + row) * r + j) : 0u;
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int t = 8 * nt + g;
                    uint32_t bb[2];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int j = j0 + 2 * c + 8 * q;
                        bb[q] = j < r ? *reinterpret_cast<const uint32_t *>(sU + t * r + j) : 0u;
                    }
                    mma_bf16_16816(f[nt], a, bb);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int t = 8 * nt + 2 * c + (q & 1);
                    const int64_t row = row0 + g + 8 * (q >> 1);
                    if (t < n) p.Y[(int64_t)t * p.rows + row] = __bfloat16_as_ushort(__float2bfloat16_rn(f[nt][q]));
                }
        }
        if (e + 1 < nep) {
            __syncthreads();  // the slots, B rows and block constants of this epoch are read
            stage_b(e + 1);
            cp_async_commit();
            stage_ah(e + 1);
            cl_arrive();      // this CTA's slots may be refilled
            __syncthreads();  // the next epoch's block constants are in place
        }
    }
}

// ---- host: plan and launch --------------------------------------------------------------
struct DfLayout {
    int S, Q, nsub, nsubA, nkb_max, RS, E, JT;
    int off_ring, off_slots, off_uslots, off_sb, off_su, off_ah, off_bar;
    size_t smem;
};

static int df_a128(int64_t x) { return (int)((x + 127) & ~int64_t(127)); }

// Shared-memory layout for a plan; false if it does not fit.
static bool df_fit(DfLayout &L, int NT, int r) {
    const int64_t part = (int64_t)NT * kDfPartBytes;
    const int64_t own = (L.E + L.S - 1) / L.S;  // tiles a CTA folds per epoch, at most
    int64_t off = kDfTabBytes;
    L.off_ring = (int)off;
    off += (int64_t)kDfWarps * L.RS * kDfBoxBytes;
    L.off_slots = (int)off;
    off += df_a128(own * L.S * L.nsub * part);
    L.off_uslots = (int)off;
    off += df_a128((int64_t)L.JT * L.S * L.nsubA * part);
    L.off_sb = (int)off;
    off += df_a128(own * 16 * r * 2);
    L.off_su = (int)off;
    off += df_a128((int64_t)8 * NT * r * 2);
    L.off_ah = (int)off;
    off += df_a128((int64_t)L.E * 16 * (L.nkb_max + 1) * 4);
    L.off_bar = (int)off;
    off += (int64_t)kDfWarps * L.RS * 8;
    L.smem = (size_t)off;
    return off <= (int64_t)kDfSmemMax;
}

// Plan for one cluster size S given Q clusters: sub-ranges, A sub-ranges and
// epoch size.  Returns false if no layout fits.
static bool df_plan_s(int64_t T, int64_t KB, int r, int NT, int S, int64_t Q, DfLayout &L) {
    L.S = S;
    L.Q = (int)Q;
    L.nkb_max = (int)((KB + S - 1) / S);
    L.JT = (r + 15) / 16;
    if (S > KB || (int64_t)8 * NT * L.nkb_max > kDfXLines || Q < 1) return false;
    const int64_t m = (T + Q - 1) / Q;
    const int64_t nkb_min = KB / S;
    // A items (U): at most 32, ideally enough sub-ranges of one block or more for every warp to
    // take one; fewer when their partials do not fit
    int nsubA0 = (int)(nkb_min < kDfWarps ? nkb_min : kDfWarps);
    while (nsubA0 > 1 && L.JT * nsubA0 > 2 * kDfWarps) nsubA0 /= 2;
    // sub-ranges: fewest code boxes per warp (items of the first epoch spread
    // over 16 warps; a box carries 4 blocks whether or not all are used), ties
    // to fewer sub-ranges (fewer partials to fold), among the counts whose
    // layout fits; then the largest epoch, the largest A split, the deepest ring
    int64_t done = 0;  // costs already tried are below this
    for (;;) {
        int best_ns = 0;
        int64_t best_cost = -1;
        for (int ns = 1; ns <= kDfWarps && ns <= nkb_min; ns *= 2) {
            const int64_t cost = ((m * ns + kDfWarps - 1) / kDfWarps) * (((L.nkb_max + ns - 1) / ns + 3) / 4);
            if (cost >= done && (best_cost < 0 || cost < best_cost)) {
                best_cost = cost;
                best_ns = ns;
            }
        }
        if (best_ns == 0) return false;
        for (int ns = best_ns; ns <= kDfWarps && ns <= nkb_min; ns *= 2) {
            if (((m * ns + kDfWarps - 1) / kDfWarps) * (((L.nkb_max + ns - 1) / ns + 3) / 4) != best_cost) continue;
            L.nsub = ns;
            for (int64_t E = m; E >= 1; --E)
                for (int nsa = nsubA0; nsa >= 1; nsa /= 2)
                    for (int rs = 4; rs >= 2; --rs) {
                        L.nsubA = nsa;
                        L.E = (int)E;
                        L.RS = rs;
                        if (df_fit(L, NT, r)) return true;
                    }
        }
        done = best_cost + 1;
    }
}

bool nf4_decode_fwd_supported(const qln_nf4_weight *w, int64_t n, int r) {
    if (n < 1 || n > 32 || (w->rows % 16) != 0 || (w->cols % 64) != 0 || (r % 8) != 0 || r < 8 || r > 128)
        return false;
    // the kernel's index arithmetic is 32-bit: block indices and tile counts times the grid must fit
    if (w->rows * (w->cols / 64) >= ((int64_t)1 << 31) || (w->rows / 16) * 1024 >= ((int64_t)1 << 31)) return false;
    const int NT = (int)((n + 7) / 8);
    const int64_t T = w->rows / 16, KB = w->cols / 64;
    for (int S = 1; S <= 8; S *= 2) {
        DfLayout L;
        // one cluster per tile range is the smallest grid a device can take
        if (df_plan_s(T, KB, r, NT, S, T < 148 / S ? T : 148 / S, L)) return true;
    }
    return false;
}

template <int NT>
static cudaError_t df_max_clusters(int S, int *out) {
    // per device and cluster size: co-resident clusters of one CTA per SM (0 =
    // not asked yet); host threads may launch at once, so the entries are atomics
    static std::atomic<int> cache[64][9];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) {
        const int v = cache[dev][S].load(std::memory_order_relaxed);
        if (v > 0) {
            *out = v;
            return cudaSuccess;
        }
    }
    e = cudaFuncSetAttribute(nf4_decode_fwd_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDfSmemMax);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t q = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    q.gridDim = dim3((unsigned)S);
    q.blockDim = dim3(kDfThreads);
    q.dynamicSmemBytes = kDfSmemMax;
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
static cudaError_t launch_df(DfParams p, const qln_nf4_weight *w, cudaStream_t st) {
    const int64_t KB = p.cols / 64, T = p.rows / 16;
    // cluster size: fewest weight blocks per CTA (ties: the larger S, for less X per CTA)
    DfLayout best{};
    int64_t best_cost = -1;
    for (int S = 8; S >= 1; S /= 2) {
        if (S > KB) continue;
        int nclus = 0;
        cudaError_t e = df_max_clusters<NT>(S, &nclus);
        if (e != cudaSuccess) return e;
        const int64_t Q = nclus < T ? nclus : T;
        DfLayout L;
        if (!df_plan_s(T, KB, p.r, NT, S, Q, L)) continue;
        const int64_t cost = ((T + Q - 1) / Q) * L.nkb_max;
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = L;
        }
    }
    if (best_cost < 0) return cudaErrorInvalidConfiguration;
    CUtensorMap tm;
    if (!make_tensor_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, (uint64_t)(p.cols / 2), (uint64_t)p.rows,
                            128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    p.KB = (int)KB;
    p.T = (int)T;
    p.S = best.S;
    p.Q = best.Q;
    p.nsub = best.nsub;
    p.nsubA = best.nsubA;
    p.nkb_max = best.nkb_max;
    p.RS = best.RS;
    p.E = best.E;
    p.JT = best.JT;
    p.off_ring = best.off_ring;
    p.off_slots = best.off_slots;
    p.off_uslots = best.off_uslots;
    p.off_sb = best.off_sb;
    p.off_su = best.off_su;
    p.off_ah = best.off_ah;
    p.off_bar = best.off_bar;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)best.S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // the kernel waits before any global access
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)(best.Q * best.S));
    cfg.blockDim = dim3(kDfThreads);
    cfg.dynamicSmemBytes = best.smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, nf4_decode_fwd_kernel<NT>, tm, p);
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_nf4_decode_fwd(const qln_nf4_weight *w, const uint16_t *X, int64_t n, const uint16_t *A,
                                  const uint16_t *B, int r, float s, uint16_t *Y, uint16_t *U_out, int *status,
                                  cudaStream_t st) {
    DfParams p;
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
    p.status = status;
    switch ((n + 7) / 8) {
        case 1: return launch_df<1>(p, w, st);
        case 2: return launch_df<2>(p, w, st);
        case 3: return launch_df<3>(p, w, st);
        default: return launch_df<4>(p, w, st);
    }
}

}  // namespace qln
