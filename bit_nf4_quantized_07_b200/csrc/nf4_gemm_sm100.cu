// Fused NF4 doubleDequant + GEMM on the sm_100a tensor cores (tcgen05, TMEM
// accumulators, TMA operand loads).  W' is decoded tile by tile into shared
// memory and never reaches HBM.
//
// Method: "LoRA 与 QLoRA" section QLoRA 1 (4-bit weight -> dequant -> BF16 ->
// GEMM) and section LoRA (y = W0 x + s B(A x), A x formed first); jjjymmm.cn
// "QLoRA" (doubleDequant: restore the block constant, then the weight); deck
// "3 QLoRA Finetuning" card 1 (the matmul sees the dequantized BF16 weight and
// gradients flow through it).
//
//   forward (TRANS = false): out[t][m] = sum_k X[t][k] W'[m][k]  + sum_j sU[t][j] B[m][j]
//   dX      (TRANS = true) : out[t][m] = sum_k dY[t][k] W'[k][m] + sum_j sG[t][j] A[j][m]
//
// One CTA computes a (128*MT) (m) x (NT*BN) (tokens) tile as MT*NT <= 2
// accumulators of 128 TMEM lanes x BN columns, K in steps of 64.  MT = 2 lets
// two 128-row weight tiles share every activation tile (half the activation
// bytes per FLOP); NT = 2 lets every decoded weight tile serve two token
// tiles (half the decode work per FLOP, the integer-pipe bound of the
// decoders).  The shape is chosen per call.
//   A_op (weights): decoded by 128*MT threads (one 64-wide row block each)
//     into the canonical 128-byte-swizzled layout, K-major for the forward
//     (W' rows along K) and MN-major for dX (W' rows are the K index, their
//     consecutive columns the M index);
//   B_op (activations X / dY, K-major): TMA tiles with 128-byte swizzle;
//   the adapter term is extra K steps whose A_op (B or A, zero-padded to 64)
//     and B_op (s*U or s*G) both arrive by TMA.
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner + single-thread MMA
// issuer, warps 2.. decoders and then the epilogue (TMEM -> BF16 -> HBM).
// Every barrier wait is bounded; on give-up the CTA records QLN_ERR_TIMEOUT
// in the status word, drains its own copies and MMAs, frees TMEM and exits.
#include <cuda.h>

#include "qln_common.cuh"
#include "qln_internal.h"
#include "tc_ptx.cuh"

namespace qln {
namespace tc {

constexpr int kBM = 128;   // rows per accumulator (TMEM lanes)
constexpr int kBK = 64;
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s

template <int MT, int NT>
struct Cfg {
    static_assert(MT * NT <= 2, "two TMEM accumulators of up to 256 columns at most");
    static constexpr int kStages = MT * NT == 1 ? 4 : 3;
    static constexpr int kMaxBN = NT == 1 ? 256 : 208;     // tokens per accumulator
    static constexpr int kDecThreads = 128 * MT;
    static constexpr int kThreads = 64 + kDecThreads;
    static constexpr uint32_t kABytes = 16384u * MT;        // MT x (128 rows x 64 K) bf16
    static constexpr uint32_t kBBytes = NT * kMaxBN * kBK * 2;
    static constexpr uint32_t kCBytes = 4096u * MT;         // codes of the A tile
    static constexpr uint32_t kTmemCols = 256u * MT * NT;
    static constexpr uint32_t kOffA = 0;
    static constexpr uint32_t kOffB = kOffA + kStages * kABytes;
    static constexpr uint32_t kOffC = kOffB + kStages * kBBytes;
    static constexpr uint32_t kOffBar = kOffC + kStages * kCBytes;
    // barriers: tma_full[S], code_full[S], dec_full[S], empty[S], accum_full
    static constexpr uint32_t kNumBars = 4 * kStages + 1;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort flag, epilogue go
    static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
};

struct Params {
    const int8_t *qabs;
    bool e4m3;  // qabs holds E4M3 codes (QLN_DQ_E4M3), else int8
    const float *absmax;
    const float *dq_scale;
    const float *dq_mean;
    int64_t cols;      // W columns (din)
    int64_t n;         // tokens
    uint16_t *out;     // [n][out_ld]
    int64_t out_ld;
    int *status;
    int KT;            // weight k-steps
    int RT;            // adapter k-steps
    int BN;            // tokens per accumulator (multiple of 16)
};

template <bool TRANS, int MT, int NT>
__global__ void __launch_bounds__(Cfg<MT, NT>::kThreads, 1)
nf4_tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_act,
                   const __grid_constant__ CUtensorMap tm_lw, const __grid_constant__ CUtensorMap tm_lact,
                   const Params p) {
    using C = Cfg<MT, NT>;
    constexpr int S = C::kStages;
    constexpr int TM = kBM * MT;  // rows of the CTA tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bar0 = sbase + C::kOffBar;
    auto tma_full = [&](int s) { return bar0 + 8u * s; };
    auto code_full = [&](int s) { return bar0 + 8u * (S + s); };
    auto dec_full = [&](int s) { return bar0 + 8u * (2 * S + s); };
    auto empty = [&](int s) { return bar0 + 8u * (3 * S + s); };
    const uint32_t accum_full = bar0 + 8u * (4 * S);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffMisc + 4);
    volatile int *epi_go = reinterpret_cast<volatile int *>(smem + C::kOffMisc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * NT * p.BN;  // NT accumulators of BN tokens each
    const int64_t m0 = (int64_t)blockIdx.y * TM;
    const int nsteps = p.KT + p.RT;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(tma_full(s), 1);
            mbar_init(code_full(s), 1);
            mbar_init(dec_full(s), C::kDecThreads);
            mbar_init(empty(s), 1);
        }
        mbar_init(accum_full, 1);
        *abort_flag = 0;
        mbar_fence_init();
        tma_prefetch_map(&tm_codes);
        tma_prefetch_map(&tm_act);
        tma_prefetch_map(&tm_lw);
        tma_prefetch_map(&tm_lact);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;
    // Barriers, descriptors and TMEM are set up while the previous kernel on
    // the stream finishes; every global access comes after this wait.
    qln::pdl_wait();
    qln::pdl_trigger();

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicExch(p.status, (int)QLN_ERR_TIMEOUT);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint32_t bsub = (uint32_t)p.BN * kBK * 2;  // one token sub-tile
            const uint32_t bbytes = NT * bsub;
            int issued = 0;
            for (int kt = 0; kt < nsteps; ++kt) {
                const int s = kt % S;
                const uint32_t ph = (uint32_t)(kt / S) & 1u;
                if (!mbar_wait_bounded(empty(s), ph ^ 1u, abort_flag, kWaitLimitNs)) {
                    give_up();
                    break;
                }
                const uint32_t sA = sbase + C::kOffA + s * C::kABytes;
                const uint32_t sB = sbase + C::kOffB + s * C::kBBytes;
                const uint32_t sC = sbase + C::kOffC + s * C::kCBytes;
                if (kt < p.KT) {
                    mbar_arrive_expect_tx(code_full(s), C::kCBytes);
                    if (!TRANS) {  // TM rows x 32 bytes
                        tma_load_2d(sC, &tm_codes, kt * 32, (int32_t)m0, code_full(s));
                    } else {       // 2*MT boxes of 64 rows x 32 bytes: [column block][row][32 B]
#pragma unroll
                        for (int d = 0; d < 2 * MT; ++d)
                            tma_load_2d(sC + 2048 * d, &tm_codes, (int32_t)(m0 / 2) + 32 * d, kt * kBK, code_full(s));
                    }
                    mbar_arrive_expect_tx(tma_full(s), bbytes);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        tma_load_2d(sB + nt * bsub, &tm_act, kt * kBK, (int32_t)(t0 + nt * p.BN), tma_full(s));
                } else {
                    const int a = kt - p.KT;
                    mbar_arrive_expect_tx(tma_full(s), C::kABytes + bbytes);
                    if (!TRANS) {
                        tma_load_2d(sA, &tm_lw, a * kBK, (int32_t)m0, tma_full(s));  // TM rows x 64
                    } else {
#pragma unroll
                        for (int d = 0; d < 2 * MT; ++d)
                            tma_load_2d(sA + 8192 * d, &tm_lw, (int32_t)m0 + 64 * d, a * kBK, tma_full(s));
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        tma_load_2d(sB + nt * bsub, &tm_lact, a * kBK, (int32_t)(t0 + nt * p.BN), tma_full(s));
                }
                issued = kt + 1;
            }
            // Drain: every issued copy has landed before the CTA may exit.
            for (int kt = (issued > S ? issued - S : 0); kt < issued; ++kt) {
                const int s = kt % S;
                const uint32_t ph = (uint32_t)(kt / S) & 1u;
                if (!mbar_wait_bounded(tma_full(s), ph, nullptr, kWaitLimitNs)) give_up();
                if (kt < p.KT && !mbar_wait_bounded(code_full(s), ph, nullptr, kWaitLimitNs)) give_up();
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kBM, p.BN, TRANS, false);
            for (int kt = 0; kt < nsteps; ++kt) {
                const int s = kt % S;
                const uint32_t ph = (uint32_t)(kt / S) & 1u;
                if (!mbar_wait_bounded(tma_full(s), ph, abort_flag, kWaitLimitNs) ||
                    !mbar_wait_bounded(dec_full(s), ph, abort_flag, kWaitLimitNs)) {
                    give_up();
                    break;
                }
                tc_fence_after();
                const uint32_t sA = sbase + C::kOffA + s * C::kABytes;
                const uint32_t sB = sbase + C::kOffB + s * C::kBBytes;
#pragma unroll
                for (int sub = 0; sub < MT; ++sub) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k) {
                            // K-major: next 16 K elements are 32 bytes further inside the
                            // swizzled 128-byte rows.  MN-major: next two 8-row K groups.
                            const uint32_t aS = sA + sub * 16384;
                            const uint64_t adesc = TRANS ? smem_desc_sw128(aS + k * 2048, 8192, 1024)
                                                         : smem_desc_sw128(aS + k * 32, 16, 1024);
                            const uint64_t bdesc = smem_desc_sw128(sB + nt * p.BN * 128 + k * 32, 16, 1024);
                            tc_mma_ss(tmem_d + (sub * NT + nt) * 256, adesc, bdesc, idesc, (kt | k) != 0 ? 1u : 0u);
                        }
                    }
                }
                tc_commit(empty(s));
            }
            tc_commit(accum_full);
        }
    } else {
        // ------------------------------------------------------------ decoders
        // One thread per 64-wide row block of the A tile.
        //   fwd: block = W row m0 + dt, column block kt.
        //   dX : block = W row 64*kt + dt%64, column block m0/64 + dt/64.
        const int dt = threadIdx.x - 64;
        const int64_t bpr = p.cols / 64;
        const int drow = TRANS ? (dt & 63) : dt;
        const int dcol = TRANS ? (dt >> 6) : 0;
        const float mu = p.qabs ? __ldg(p.dq_mean) : 0.f;
        auto block_index = [&](int kt) -> int64_t {
            return TRANS ? ((int64_t)kt * kBK + drow) * bpr + (m0 / 64) + dcol : (m0 + drow) * bpr + kt;
        };
        // Raw block constants are fetched two k-steps before use so that their
        // L2 latency hides behind the decode of the steps in between.
        struct Raw {
            float v;     // absmax (plain) or DQ scale b_g
            int32_t q;   // DQ code rhat_j
        };
        auto fetch = [&](int kt) -> Raw {
            Raw r{0.f, 0};
            if (kt < p.KT) {
                const int64_t jb = block_index(kt);
                if (p.qabs) {
                    r.q = __ldg(p.qabs + jb);
                    r.v = __ldg(p.dq_scale + (jb >> 8));
                } else {
                    r.v = __ldg(p.absmax + jb);
                }
            }
            return r;
        };
        Raw r0 = fetch(0), r1 = fetch(1);
        // This thread's 32 code bytes sit at a 32-byte stride; the two 16-byte
        // halves are read in an order that keeps each 8-thread phase on
        // distinct banks (half `cfirst` first).
        const uint32_t cfirst = (drow >> 2) & 1;
        const uint32_t code_off = (TRANS ? dcol * 2048 : 0) + drow * 32;
        const uint32_t r8 = drow & 7;
        // fwd (K-major): row drow at (drow/8)*1024 + (drow%8)*128, chunk c (K 8c..8c+7).
        // dX (MN-major): atom (dcol, drow/8) at dcol*8192 + (drow/8)*1024, K-row drow%8,
        //   chunk c = M elements 8c..8c+7.  Both: chunk c at byte (c ^ (row % 8)) * 16
        // of the row.  Bits 4-6 of the row's address are zero, so the chunk
        // address is (row address + 16*r8) XOR 16*c; the half read first
        // holds chunks 4*cfirst.. , folded into the XOR base as well.
        const uint32_t row_off = (TRANS ? dcol * 8192 : 0) + (drow >> 3) * 1024 + r8 * 128;
        const uint32_t sA0 = smem_addr(smem + C::kOffA) + row_off + (r8 << 4);
        for (int kt = 0; kt < nsteps; ++kt) {
            const int s = kt % S;
            const uint32_t ph = (uint32_t)(kt / S) & 1u;
            const float ah = p.qabs ? dq_restore((uint32_t)r0.q, r0.v, mu, p.e4m3) : r0.v;
            r0 = r1;
            r1 = fetch(kt + 2);
            if (!mbar_wait_bounded(empty(s), ph ^ 1u, abort_flag, kWaitLimitNs)) {
                give_up();
                break;
            }
            if (kt < p.KT) {
                if (!mbar_wait_bounded(code_full(s), ph, abort_flag, kWaitLimitNs)) {
                    give_up();
                    break;
                }
                const uint8_t *cptr = smem + C::kOffC + s * C::kCBytes + code_off;
                const uint4 ca = *reinterpret_cast<const uint4 *>(cptr + 16 * cfirst);
                const uint4 cb = *reinterpret_cast<const uint4 *>(cptr + 16 * (cfirst ^ 1));
                const NF4Table tab = nf4_table(ah);
                const uint32_t xa = (sA0 + s * C::kABytes) ^ (cfirst << 6);  // chunks of ca: 4*cfirst + i
                const uint32_t xb = xa ^ 64u;                                  // chunks of cb
                st_shared_v4(xa ^ 0u, nf4_decode8(ca.x, tab));
                st_shared_v4(xa ^ 16u, nf4_decode8(ca.y, tab));
                st_shared_v4(xa ^ 32u, nf4_decode8(ca.z, tab));
                st_shared_v4(xa ^ 48u, nf4_decode8(ca.w, tab));
                st_shared_v4(xb ^ 0u, nf4_decode8(cb.x, tab));
                st_shared_v4(xb ^ 16u, nf4_decode8(cb.y, tab));
                st_shared_v4(xb ^ 32u, nf4_decode8(cb.z, tab));
                st_shared_v4(xb ^ 48u, nf4_decode8(cb.w, tab));
                fence_proxy_async_smem();
            }
            mbar_arrive(dec_full(s));
        }

        // ------------------------------------------------------------ epilogue
        // The go / no-go decision is made uniform across the decoder threads
        // (tcgen05.ld is warp-collective, named barrier 1 counts all of them).
        if (*abort_flag || !mbar_wait_bounded(accum_full, 0, abort_flag, kWaitLimitNs)) give_up();
        asm volatile("bar.sync 1, %0;" ::"n"(C::kDecThreads) : "memory");
        if (dt == 0) *epi_go = *abort_flag ? 0 : 1;
        asm volatile("bar.sync 1, %0;" ::"n"(C::kDecThreads) : "memory");
        if (*epi_go) {
            tc_fence_after();
            const int q = warp & 3;              // TMEM lane quadrant of this warp
            const int sub = (warp - 2) >> 2;     // weight sub-tile of this warp
            uint16_t *Os = reinterpret_cast<uint16_t *>(smem);  // [NT*BN][TM] bf16; all MMAs are done
            const int m = sub * kBM + q * 32 + lane;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                for (int c0 = 0; c0 < p.BN; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem_d + ((uint32_t)(q * 32) << 16) + (uint32_t)((sub * NT + nt) * 256 + c0), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c0 + j < p.BN)
                            Os[(nt * p.BN + c0 + j) * TM + m] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
                }
            }
            asm volatile("bar.sync 1, %0;" ::"n"(C::kDecThreads) : "memory");
            constexpr int kChunksPerRow = TM / 8;
            const int chunks = NT * p.BN * kChunksPerRow;
            for (int idx = dt; idx < chunks; idx += C::kDecThreads) {
                const int row = idx / kChunksPerRow, ch = idx % kChunksPerRow;
                const int64_t t = t0 + row;
                if (t < p.n)
                    *reinterpret_cast<uint4 *>(p.out + t * p.out_ld + m0 + 8 * ch) =
                        *reinterpret_cast<const uint4 *>(Os + row * TM + 8 * ch);
            }
        }
    }

    // Teardown: all MMAs must have retired before TMEM is released.
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        if (lane == 0 && !mbar_wait_bounded(accum_full, 0, nullptr, kWaitLimitNs)) give_up();
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_d, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps (driver entry point fetched through the runtime, so
// the library does not link libcuda), tile-shape choice, launch.
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2D map over a row-major [outer][inner] array.
static bool make_map(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, uint64_t inner,
                     uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * (uint64_t)esize};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

bool make_tensor_map_2d(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, uint64_t inner,
                        uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    return tc::make_map(m, dt, esize, base, inner, outer, box_inner, box_outer, sw);
}

namespace tc {

// Tile shape per call.  Candidates: MT weight sub-tiles of 128 rows and NT
// token sub-tiles of BN tokens (MT * NT <= 2, BN a multiple of 16).  A simple
// cost model picks the fastest: one CTA per SM; a k-step costs the larger of
// its tensor time (at the measured dense rate, about 5700 FLOP per cycle per
// SM) and its decode time (about 0.12 cycle per decoded weight, integer-pipe
// bound), plus a fixed cost per tile; waves are counted whole.
struct TileShape {
    int MT, NT, BN;
};

static TileShape choose_shape(int64_t M, int64_t K, int64_t n, int num_sms) {
    const int64_t ksteps = K / kBK + 1;
    TileShape best{1, 1, 128};
    double best_cost = 1e300;
    const int shapes[3][2] = {{2, 1}, {1, 2}, {1, 1}};
    for (const auto &sh : shapes) {
        const int MT = sh[0], NT = sh[1];
        if ((M % (kBM * MT)) != 0) continue;
        const int maxbn = NT == 1 ? 256 : 208;
        for (int bn = maxbn; bn >= 16; bn -= 16) {
            if (bn < 128 && (int64_t)NT * bn < n) break;  // narrow tiles only for small n
            const int64_t tile_tok = (int64_t)NT * bn;
            const int64_t ttiles = (n + tile_tok - 1) / tile_tok;
            const int64_t tiles = ttiles * (M / (kBM * MT));
            const int64_t rounds = (tiles + num_sms - 1) / num_sms;
            const double mma = 2.0 * kBM * MT * tile_tok * kBK / 5700.0;
            const double dec = 0.12 * 8192.0 * MT;
            const double tile = ksteps * (mma > dec ? mma : dec) + 4000.0;
            // ties go to the fewest padded tokens
            const double cost = rounds * tile * (1.0 + 1e-4 * (double)(ttiles * tile_tok - n) / (double)n);
            if (cost < best_cost * 0.999) {
                best_cost = cost;
                best = TileShape{MT, NT, bn};
            }
        }
    }
    return best;
}

template <bool TRANS, int MT, int NT>
static cudaError_t launch_t(const CUtensorMap &m_codes, const CUtensorMap &m_act, const CUtensorMap &m_lw,
                            const CUtensorMap &m_lact, const Params &p, dim3 grid, cudaStream_t st) {
    using C = Cfg<MT, NT>;
    cudaError_t e = cudaFuncSetAttribute(nf4_tc_gemm_kernel<TRANS, MT, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    return qln::launch_pdl(nf4_tc_gemm_kernel<TRANS, MT, NT>, grid, dim3(C::kThreads), (size_t)C::kSmemBytes, st,
                           m_codes, m_act, m_lw, m_lact, p);
}

}  // namespace tc

bool nf4_tc_gemm_supported(const qln_nf4_weight *w, bool trans, int64_t n, int r) {
    const int64_t M = trans ? w->cols : w->rows;
    const int64_t K = trans ? w->rows : w->cols;
    return n >= 64 && (M % tc::kBM) == 0 && (K % tc::kBK) == 0 && r >= 8 && r <= 128 && (r % 8) == 0 &&
           tc::encode_fn() != nullptr;
}

int64_t nf4_tc_gemm_ctas(const qln_nf4_weight *w, bool trans, int64_t n, int r, int num_sms) {
    if (!nf4_tc_gemm_supported(w, trans, n, r)) return 0;
    const int64_t M = trans ? w->cols : w->rows;
    const int64_t K = trans ? w->rows : w->cols;
    const tc::TileShape shape = tc::choose_shape(M, K, n, num_sms > 0 ? num_sms : 148);
    return ((n + (int64_t)shape.NT * shape.BN - 1) / ((int64_t)shape.NT * shape.BN)) * (M / (tc::kBM * shape.MT));
}

cudaError_t launch_nf4_tc_gemm(const qln_nf4_weight *w, bool trans, const uint16_t *act, int64_t n,
                               const uint16_t *lact, const uint16_t *lw, int r, uint16_t *out, int *status,
                               cudaStream_t st, int num_sms) {
    using namespace tc;
    const int64_t rows = w->rows, cols = w->cols;
    const int64_t M = trans ? cols : rows;
    const int64_t K = trans ? rows : cols;
    const TileShape shape = choose_shape(M, K, n, num_sms > 0 ? num_sms : 148);
    const int MT = shape.MT, NT = shape.NT, BN = shape.BN;
    const int TM = kBM * MT;
    CUtensorMap m_codes, m_act, m_lw, m_lact;
    bool ok = true;
    // codes as bytes [rows][cols/2]
    if (!trans) ok &= make_map(&m_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, cols / 2, rows, 32, TM,
                               CU_TENSOR_MAP_SWIZZLE_NONE);
    else ok &= make_map(&m_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, cols / 2, rows, 32, kBK,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    ok &= make_map(&m_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, act, K, n, kBK, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!trans) ok &= make_map(&m_lw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lw, r, rows, kBK, TM,
                               CU_TENSOR_MAP_SWIZZLE_128B);                       // B [rows][r]
    else ok &= make_map(&m_lw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lw, cols, r, 64, kBK,
                        CU_TENSOR_MAP_SWIZZLE_128B);                               // A [r][cols]
    ok &= make_map(&m_lact, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lact, r, n, kBK, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;

    Params p;
    p.qabs = w->qabs;
    p.e4m3 = w->dq_format == QLN_DQ_E4M3;
    p.absmax = w->absmax;
    p.dq_scale = w->dq_scale;
    p.dq_mean = w->dq_mean;
    p.cols = cols;
    p.n = n;
    p.out = out;
    p.out_ld = M;
    p.status = status;
    p.KT = (int)(K / kBK);
    p.RT = (r + kBK - 1) / kBK;
    p.BN = BN;
    dim3 grid((unsigned)((n + (int64_t)NT * BN - 1) / ((int64_t)NT * BN)), (unsigned)(M / TM));
    if (trans) {
        if (MT == 2) return launch_t<true, 2, 1>(m_codes, m_act, m_lw, m_lact, p, grid, st);
        if (NT == 2) return launch_t<true, 1, 2>(m_codes, m_act, m_lw, m_lact, p, grid, st);
        return launch_t<true, 1, 1>(m_codes, m_act, m_lw, m_lact, p, grid, st);
    }
    if (MT == 2) return launch_t<false, 2, 1>(m_codes, m_act, m_lw, m_lact, p, grid, st);
    if (NT == 2) return launch_t<false, 1, 2>(m_codes, m_act, m_lw, m_lact, p, grid, st);
    return launch_t<false, 1, 1>(m_codes, m_act, m_lw, m_lact, p, grid, st);
}

}  // namespace qln
