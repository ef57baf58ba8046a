// NF4 codec kernels: blockwise quantize (K1), double quantization (K2 + K3),
// doubleDequant to BF16 (K4).  All HBM-bound streaming kernels.
//
// Method: jjjymmm.cn 2024/03 QLoRA post, "4-bit NormalFloat(NF4)" (divide by
// the block ABSMAX, snap to the nearest book entry; dequantize = book value),
// "Double Quantization" and "QLoRA" (doubleDequant: constants first);
// "LoRA 与 QLoRA" section QLoRA 2 (a_j = max|W_j| per 64 weights,
// r_j = (a_j - mu)/b, 8-bit rhat_j, ahat_j = mu + b rhat_j).
#include <atomic>

#include <cuda_fp16.h>

#include "qln_common.cuh"
#include "qln_internal.h"

namespace qln {

// ===========================================================================
// K1: quantize.  Lane l of a warp owns 8 consecutive weights, so 8 lanes hold
// one 64-weight block and a warp takes 4 blocks (a 256-weight chunk) at a
// time.  Each 8-lane group reduces its block's absmax with three xor-shuffles;
// x = w / absmax is the IEEE fp32 quotient, in [-1, 1].
//
// Snap, almost always without a division and without a 15-way compare:
//  * y = w * inv, with inv the hardware reciprocal of the absmax, stands in
//    for x (the near-threshold rule below makes the result exactly x's code);
//  * y' = y/2 + 3 lies in [2, 4) for every |y| <= 1, where fp32 has a single
//    exponent, so byte 2 of y' (its top 7 mantissa bits) is a uniform bucket
//    of width 1/32 in y.  Thresholds are at least 0.08 apart, so a bucket
//    holds at most one;
//  * a 256-entry table gives, per bucket, the number of thresholds below the
//    bucket ("base", 0..15) and the bucket's threshold (or a huge value); the
//    code is base + (y > threshold).  The table is replicated once per lane
//    (entry-major, 128 bytes per bucket), so the lookup never has a bank
//    conflict, and any byte value indexes in bounds.
// An entry is one word: the threshold's fp32 bits with the low 4 mantissa
// bits replaced by base.  That moves the threshold by at most 15 ulps
// (< 2^-20 for |t| < 1), which the near window below absorbs.
// ===========================================================================
namespace snap_build {

// 2^i for i in [-160, 160], exactly, as binary64.
struct Pow2 {
    double v[321];
};
constexpr Pow2 make_pow2() {
    Pow2 p{};
    p.v[160] = 1.0;
    for (int i = 1; i <= 160; ++i) {
        p.v[160 + i] = p.v[159 + i] * 2.0;
        p.v[160 - i] = p.v[161 - i] * 0.5;
    }
    return p;
}
constexpr Pow2 kPow2 = make_pow2();
constexpr double pow2(int i) { return kPow2.v[160 + i]; }

// The exact value of a finite, normal-or-zero fp32 bit pattern.
constexpr double f32_value(uint32_t b) {
    const int e = (int)((b >> 23) & 0xffu);
    const uint32_t m = b & 0x7fffffu;
    const double v = e == 0 ? (double)m * pow2(-149) : (double)(m | 0x800000u) * pow2(e - 150);
    return (b >> 31) ? -v : v;
}

// The largest fp32 value <= s (s a nonzero binary64 in the normal fp32 range).
constexpr uint32_t f32_round_down_bits(double s) {
    const bool neg = s < 0;
    const double a = neg ? -s : s;
    int E = 0;
    while (a >= pow2(E + 1)) ++E;
    while (a < pow2(E)) --E;
    const double q = a * pow2(23 - E);  // exact: a power-of-two scaling, q in [2^23, 2^24)
    uint64_t mi = (uint64_t)q;
    if (neg && (double)mi != q) ++mi;  // rounding toward -inf rounds a negative magnitude up
    if (mi == (1ull << 24)) {
        mi = 1ull << 23;
        ++E;
    }
    return (neg ? 0x80000000u : 0u) | ((uint32_t)(E + 127) << 23) | (uint32_t)(mi - (1ull << 23));
}

// t_k = RD((c_k + c_{k+1}) / 2); the sum of two book values is exact in binary64.
constexpr uint32_t threshold_bits(int k) {
    return f32_round_down_bits(0.5 * f32_value(nf4_bits(k)) + 0.5 * f32_value(nf4_bits(k + 1)));
}

struct Thresholds {
    uint32_t bits[15];
    double value[15];
};
constexpr Thresholds make_thresholds() {
    Thresholds t{};
    for (int k = 0; k < 15; ++k) {
        t.bits[k] = threshold_bits(k);
        t.value[k] = f32_value(t.bits[k]);
    }
    return t;
}
constexpr Thresholds kThr = make_thresholds();

// Bucket b (byte 2 of y' = y/2 + 3, b < 128) holds y in [b/32 - 2, (b+1)/32 - 2).
constexpr double bucket_lo(int b) { return b / 32.0 - 2.0; }
constexpr uint32_t kNoThreshold = 0x7f000000u;  // 2^127: above every y

struct Table {
    uint32_t e[256];
};
constexpr Table make_table() {
    Table t{};
    for (int b = 0; b < 256; ++b) {
        if (b >= 128) {  // bit 23 of y' set: not reached from |y| <= 1.03
            t.e[b] = kNoThreshold | 7u;
            continue;
        }
        const double lo = bucket_lo(b), hi = bucket_lo(b + 1);
        uint32_t base = 0, thr = kNoThreshold;
        for (int k = 0; k < 15; ++k) {
            if (kThr.value[k] < lo) ++base;
            else if (kThr.value[k] < hi) thr = kThr.bits[k] & ~0xfu;
        }
        t.e[b] = thr | base;
    }
    return t;
}

// What the snap argument needs, checked here: at most one threshold per
// bucket; every threshold more than 2^-16 from a bucket edge (so a y within
// the near window of a threshold has that threshold's bucket even after
// y' rounds); the 4-bit base substitution moves no threshold by 2^-20 or more.
constexpr bool snap_table_sound() {
    for (int k = 0; k < 15; ++k) {
        const double tk = kThr.value[k];
        if (!(f32_value(nf4_bits(k)) < tk && tk < f32_value(nf4_bits(k + 1)))) return false;
        if (k > 0 && !(tk - kThr.value[k - 1] > 1.0 / 32)) return false;
        const double pos = (tk + 2.0) * 32.0;  // bucket coordinate
        const double frac = pos - (double)(int64_t)pos;
        if (!(frac * (1.0 / 32) > pow2(-16) && (1.0 - frac) * (1.0 / 32) > pow2(-16))) return false;
        const double moved = f32_value(kThr.bits[k] & ~0xfu);
        const double diff = moved > tk ? moved - tk : tk - moved;
        if (!(diff < pow2(-20))) return false;
    }
    return true;
}
static_assert(snap_table_sound(), "snap bucket table assumptions");
static_assert(threshold_bits(6) == 0xbd3a7869u && threshold_bits(7) == 0x3d22fb01u,
              "the thresholds next to zero are the halved neighbours of the zero code");

}  // namespace snap_build

constexpr snap_build::Table kSnapTableHost = snap_build::make_table();  // evaluated by the compiler
__device__ const snap_build::Table kSnapTable = kSnapTableHost;
__constant__ uint32_t kSnapThresholdBits[15] = {
    snap_build::kThr.bits[0],  snap_build::kThr.bits[1],  snap_build::kThr.bits[2],  snap_build::kThr.bits[3],
    snap_build::kThr.bits[4],  snap_build::kThr.bits[5],  snap_build::kThr.bits[6],  snap_build::kThr.bits[7],
    snap_build::kThr.bits[8],  snap_build::kThr.bits[9],  snap_build::kThr.bits[10], snap_build::kThr.bits[11],
    snap_build::kThr.bits[12], snap_build::kThr.bits[13], snap_build::kThr.bits[14]};

__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// Codes of 8 weights w (block absmax a, inv = hardware reciprocal of a when a
// is normal and below 2^126, else 0) as one little-endian word: byte i holds
// weight 2i in its high nibble and weight 2i+1 in its low nibble.
// Near-threshold rule: y = RN(w * inv) differs from w/a by at most
// |w/a| (2^-23 + 2^-24) < 1.8e-7 and x = RN(w/a) is within 2^-25 of w/a, so
// whenever y is 2^-19 or more from every threshold, y and x lie on the same
// side of all of them.  The test compares y with its bucket's (moved)
// threshold t': |t' - y| >= 2^-18 gives |t - y| > 2^-18 - 2^-20 > 2^-19, and
// then also sign(t' - y) = sign(t - y).  Thresholds of other buckets are more
// than 2^-16 away.  Otherwise the group is redone with the IEEE quotient and
// a plain count of the thresholds below it.  The sign of RN(t' - y) is that
// of the exact difference (and +0 on equality: a tie goes to the lower code).
__device__ __forceinline__ uint32_t snap8(const float (&w)[8], float a, float inv, uint32_t lut_lane) {
    if (!(a > 0.f)) return 0x77777777u;  // all-zero block: the exact zero
    float y[8], yb[8];
    const uint64_t inv2 = f32x2_pack(inv, inv);
    const uint64_t half_inv2 = f32x2_pack(0.5f * inv, 0.5f * inv);
    const uint64_t three2 = f32x2_pack(3.0f, 3.0f);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const uint64_t w2 = f32x2_pack(w[i], w[i + 1]);
        uint64_t p, q;
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(p) : "l"(w2), "l"(inv2));
        asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(w2), "l"(half_inv2), "l"(three2));
        f32x2_unpack(p, y[i], y[i + 1]);
        f32x2_unpack(q, yb[i], yb[i + 1]);
    }
    // Nibble j of the word (bits 4j..4j+3) is weight order[j]; a funnel shift
    // pushes each new nibble in at the top.
    constexpr int order[8] = {1, 0, 3, 2, 5, 4, 7, 6};
    uint32_t word = 0;
    float dmin = 1.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int i = order[j];
        const uint32_t bucket = __byte_perm(__float_as_uint(yb[i]), 0u, 0x4442u);
        uint32_t e;
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(e) : "r"(lut_lane + (bucket << 7)));
        const float d = __fsub_rn(__uint_as_float(e), y[i]);
        dmin = fminf(dmin, fabsf(d));
        e += __float_as_uint(d) >> 31;  // base + (y > t'); base <= 14 wherever a threshold exists
        word = __funnelshift_r(word, e, 4);
    }
    if (dmin < 0x1p-18f || inv == 0.f) {  // rare: redo the group with the exact quotient
        word = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float x = __fdiv_rn(w[order[j]], a);
            uint32_t q = 0;
#pragma unroll
            for (int k = 0; k < 15; ++k) q += (x > __uint_as_float(kSnapThresholdBits[k])) ? 1u : 0u;
            word = __funnelshift_r(word, q, 4);
        }
    }
    return word;
}

// Input element types of K1: fp32, or 16-bit weights (bf16 / fp16) widened
// exactly to fp32 in registers.
struct Bf16In {
    uint16_t bits;
};
struct F16In {
    uint16_t bits;
};
template <typename T> struct QzIn;
template <> struct QzIn<float> {
    static constexpr int kBytes = 4;
    __device__ static void widen(const float *ring8, float (&v)[8]) {
        const float4 lo = *reinterpret_cast<const float4 *>(ring8);
        const float4 hi = *reinterpret_cast<const float4 *>(ring8 + 4);
        v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
        v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
    }
};
template <> struct QzIn<Bf16In> {
    static constexpr int kBytes = 2;
    __device__ static void widen(const float *ring8, float (&v)[8]) {
        const uint4 u = *reinterpret_cast<const uint4 *>(ring8);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // a bf16 is the top half of its fp32 pattern
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <> struct QzIn<F16In> {
    static constexpr int kBytes = 2;
    __device__ static void widen(const float *ring8, float (&v)[8]) {
        const uint4 u = *reinterpret_cast<const uint4 *>(ring8);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // binary16 -> binary32 is exact
            const __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
            const float2 f = __half22float2(h);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
};

constexpr int kQzWarps = 24;       // two CTAs of 24 warps per SM
constexpr int kQzCtasPerSm = 2;
constexpr int kQzStages = 3;       // chunks per warp ring
constexpr int kQzThreads = 32 * kQzWarps;
constexpr int kQzLutBytes = 256 * 128;                                    // 256 buckets x 32 lanes x 4 B

// The weights stream through a private ring of kQzStages chunk slots per warp,
// filled by cp.async: lane l copies (and later reads back) its own 8 weights
// of each chunk, so no lane waits on another's copy.  48 warps per SM with
// two chunks requested ahead keep about 96 KB per SM in flight (fp32) --
// what HBM latency asks for at full bandwidth -- without holding them in
// registers, and enough warps to cover the snap's shared-memory and shuffle
// latencies.  Weights past numel are zero-filled by the copy (a zero weight
// raises no absmax and gets code 7, which is what a ragged tail stores); a
// lane's last partial code word is written byte by byte.  Idx is 32-bit
// whenever every element offset stays below 2^31.
template <typename T, typename Idx>
__global__ void __launch_bounds__(kQzThreads, kQzCtasPerSm) nf4_quantize_kernel(const T *__restrict__ W, Idx numel,
                                                                                uint8_t *__restrict__ codes,
                                                                                float *__restrict__ absmax,
                                                                                bool release_early) {
    constexpr int kB = QzIn<T>::kBytes;
    extern __shared__ __align__(16) unsigned char qz_smem[];
    for (int i = threadIdx.x; i < kQzLutBytes / 4; i += kQzThreads)  // bucket i/32, lane i%32
        reinterpret_cast<uint32_t *>(qz_smem)[i] = kSnapTable.e[i >> 5];
    __syncthreads();
    pdl_wait();  // W may come from the previous kernel; codes/absmax may still be read by it
    // This kernel writes a weight (codes, absmax), and a forward may read its
    // weight before its own dependency wait; so the next kernel is released
    // early only when it is known to wait first.
    if (release_early) pdl_trigger();

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int sub = lane >> 3;  // block of the lane within a 4-block chunk
    const uint32_t lut_lane = smem_u32(qz_smem) + 4u * lane;
    unsigned char *ring = qz_smem + kQzLutBytes + warp * (kQzStages * 256 * kB) + lane * (8 * kB);
    const Idx nfull = numel / 256;           // chunks of 256 weights inside numel
    const Idx nchunks = (numel + 255) / 256;  // plus at most one ragged chunk
    const Idx nwarps = (Idx)gridDim.x * kQzWarps;
    const Idx c0 = (Idx)blockIdx.x * kQzWarps + warp;

    auto issue = [&](int slot, Idx c) {  // one commit group per chunk, empty past the end
        const Idx e = 256 * c + 8 * lane;
        unsigned char *dst = ring + slot * (256 * kB);
        const unsigned char *src = reinterpret_cast<const unsigned char *>(W + e);
        if (c < nfull) {
#pragma unroll
            for (int p = 0; p < 8 * kB / 16; ++p) cp_async16(dst + 16 * p, src + 16 * p);
        } else if (c < nchunks && e < numel) {  // the ragged chunk: zero-fill past numel
            const int valid = e + 8 <= numel ? 8 * kB : (int)(numel - e) * kB;
#pragma unroll
            for (int p = 0; p < 8 * kB / 16; ++p) {
                const int n = valid - 16 * p;
                if (n > 0) cp_async16_zfill(dst + 16 * p, src + 16 * p, n < 16 ? n : 16);
                else *reinterpret_cast<uint4 *>(dst + 16 * p) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        cp_async_commit();
    };
#pragma unroll
    for (int d = 0; d < kQzStages; ++d) issue(d, c0 + d * nwarps);

    int slot = 0;
    for (Idx c = c0; c < nchunks; c += nwarps) {
        cp_async_wait<kQzStages - 1>();  // this lane's copies of chunk c have landed
        const Idx e = 256 * c + 8 * lane;
        const bool full = c < nfull;  // warp-uniform
        float v[8];
        if (full || e < numel) {
            QzIn<T>::widen(reinterpret_cast<const float *>(ring + slot * (256 * kB)), v);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.f;
        }
        float m;
        {
            float t[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) t[i] = fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1]));
            m = fmaxf(fmaxf(t[0], t[1]), fmaxf(t[2], t[3]));
        }
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const float a = m;  // the block absmax (a max is exact)
        float inv = 0.f;
        if (a >= 0x1p-126f && a < 0x1p126f) asm("rcp.approx.f32 %0, %1;" : "=f"(inv) : "f"(a));
        const uint32_t word = snap8(v, a, inv, lut_lane);
        if (full) {
            __stcs(reinterpret_cast<uint32_t *>(codes) + (e >> 3), word);
            if ((lane & 7) == 0) absmax[4 * c + sub] = a;
        } else if (e < numel) {
            if (e + 8 <= numel) {
                __stcs(reinterpret_cast<uint32_t *>(codes) + (e >> 3), word);
            } else {  // ceil((numel - e) / 2) bytes
                const int nbytes = (int)((numel - e + 1) / 2);
                for (int i = 0; i < nbytes; ++i) codes[(e >> 1) + i] = (uint8_t)(word >> (8 * i));
            }
            if ((lane & 7) == 0) absmax[4 * c + sub] = a;
        }
        issue(slot, c + kQzStages * nwarps);  // after v has been consumed
        slot = (slot + 1 == kQzStages) ? 0 : slot + 1;
    }
    cp_async_wait<0>();
}

template <typename T, typename Idx>
static cudaError_t launch_quantize_t(const T *W, int64_t numel, uint8_t *codes, float *absmax, cudaStream_t st,
                                     int num_sms) {
    const int64_t nchunks = ((numel + 63) / 64 + 3) / 4;
    int64_t grid = (nchunks + kQzWarps - 1) / kQzWarps;
    if (grid > (int64_t)kQzCtasPerSm * num_sms) grid = (int64_t)kQzCtasPerSm * num_sms;
    if (grid < 1) grid = 1;
    const int smem = kQzLutBytes + kQzWarps * kQzStages * 256 * QzIn<T>::kBytes;
    cudaError_t e =
        cudaFuncSetAttribute(nf4_quantize_kernel<T, Idx>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(nf4_quantize_kernel<T, Idx>, dim3((unsigned)grid), dim3(kQzThreads), (size_t)smem, st, W,
                      (Idx)numel, codes, absmax, false);
}

template <typename T>
static cudaError_t launch_quantize_any(const void *W, int64_t numel, uint8_t *codes, float *absmax, cudaStream_t st,
                                       int num_sms) {
    const T *w = static_cast<const T *>(W);
    // 32-bit indices while every element offset (and a chunk look-ahead per warp) stays below 2^31
    if (numel + (int64_t)256 * (kQzStages + 1) * kQzCtasPerSm * num_sms * kQzWarps < ((int64_t)1 << 31))
        return launch_quantize_t<T, uint32_t>(w, numel, codes, absmax, st, num_sms);
    return launch_quantize_t<T, int64_t>(w, numel, codes, absmax, st, num_sms);
}

cudaError_t launch_nf4_quantize(const void *W, int dtype, int64_t numel, uint8_t *codes, float *absmax,
                                cudaStream_t st, int num_sms) {
    switch (dtype) {
        case QLN_DTYPE_BF16: return launch_quantize_any<Bf16In>(W, numel, codes, absmax, st, num_sms);
        case QLN_DTYPE_F16: return launch_quantize_any<F16In>(W, numel, codes, absmax, st, num_sms);
        default: return launch_quantize_any<float>(W, numel, codes, absmax, st, num_sms);
    }
}

// ===========================================================================
// K2: partial sums for mu.  CTA c sums the block constants a[C c, C (c+1)) as
// a perfect binary tree in binary64 (zero-padded), C = 2048 * NG: thread t
// folds its 8 * NG consecutive leaves (8 at a time, the 8-leaf sums merged
// like a binary counter, which is the tree order), a warp xor-butterfly adds
// lane pairs level by level (addition is commutative, so both lanes of a pair
// hold the same node), and the 8 warp roots are folded pairwise.  The result
// is exactly the aligned subtree of the whole-tensor tree.  C grows with nb so
// that there are at most kMaxPartials partial sums.
// ===========================================================================
constexpr int kMeanThreads = 256;
constexpr int kMaxPartials = 1024;
constexpr int64_t kMeanMaxBlocks = (int64_t)1 << 25;  // nb limit: C <= 32768

__device__ __forceinline__ double tree8(const float (&v)[8]) {
    const double s01 = __dadd_rn((double)v[0], (double)v[1]), s23 = __dadd_rn((double)v[2], (double)v[3]);
    const double s45 = __dadd_rn((double)v[4], (double)v[5]), s67 = __dadd_rn((double)v[6], (double)v[7]);
    return __dadd_rn(__dadd_rn(s01, s23), __dadd_rn(s45, s67));
}

// 8 consecutive constants starting at j (zeros past nb).
__device__ __forceinline__ void load8_const(float (&v)[8], const float *__restrict__ a, int64_t j, int64_t nb) {
    if (j + 8 <= nb) {
        const float4 x = __ldg(reinterpret_cast<const float4 *>(a + j));
        const float4 y = __ldg(reinterpret_cast<const float4 *>(a + j + 4));
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
        v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = (j + i < nb) ? a[j + i] : 0.f;
    }
}

__device__ __forceinline__ double warp_butterfly_sum(double s, int levels) {
    for (int l = 0; l < levels; ++l) s = __dadd_rn(s, __shfl_xor_sync(0xffffffffu, s, 1 << l));
    return s;
}

template <int NG>
__global__ void __launch_bounds__(kMeanThreads) dq_partial_kernel(const float *__restrict__ a, int64_t nb,
                                                                  double *__restrict__ partial) {
    __shared__ double warp_root[kMeanThreads / 32];
    pdl_wait();
    pdl_trigger();
    const int64_t base = ((int64_t)blockIdx.x * kMeanThreads + threadIdx.x) * (8 * NG);
    float v[NG][8];
#pragma unroll
    for (int g = 0; g < NG; ++g) load8_const(v[g], a, base + 8 * g, nb);  // all loads in flight at once
    double level[5];  // level[k]: a pending subtree of 8 * 2^k leaves (binary counter over g)
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        double s = tree8(v[g]);
        int k = 0;
#pragma unroll
        for (int t = g; t & 1; t >>= 1, ++k) s = __dadd_rn(level[k], s);
        level[k] = s;
    }
    constexpr int top = NG == 1 ? 0 : NG == 2 ? 1 : NG == 4 ? 2 : NG == 8 ? 3 : 4;
    const double s = warp_butterfly_sum(level[top], 5);
    if ((threadIdx.x & 31) == 0) warp_root[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        const double w01 = __dadd_rn(warp_root[0], warp_root[1]), w23 = __dadd_rn(warp_root[2], warp_root[3]);
        const double w45 = __dadd_rn(warp_root[4], warp_root[5]), w67 = __dadd_rn(warp_root[6], warp_root[7]);
        partial[blockIdx.x] = __dadd_rn(__dadd_rn(w01, w23), __dadd_rn(w45, w67));
    }
}

// One group of 256 block constants, one warp, 8 consecutive constants per
// lane (e, starting at j0): d = fp32(a - mu), b = fp32(max|d| / 127 or 448),
// rhat = clamp(rint(fp32(d / b)), -127, 127) or E4M3(fp32(d / b)); 0 if b == 0.
__device__ __forceinline__ void dq_quantize_group(const float (&e)[8], int64_t j0, int64_t nb, float mu, bool e4m3,
                                                  int lane, int64_t g, int8_t *__restrict__ qabs,
                                                  float *__restrict__ scale) {
    float d[8], m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        d[i] = __fsub_rn(e[i], mu);
        if (j0 + i < nb) m = fmaxf(m, fabsf(d[i]));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float b = __fdiv_rn(m, e4m3 ? 448.0f : 127.0f);  // 448: the largest E4M3 value
    if (lane == 0) scale[g] = b;
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t r = 0;
        if (b != 0.f) {
            const float x = __fdiv_rn(d[i], b);
            r = e4m3 ? (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3)  // nearest-even, saturating
                     : (uint32_t)((int)fminf(fmaxf(rintf(x), -127.f), 127.f) & 0xff);
        }
        w[i >> 2] |= (r & 0xffu) << (8 * (i & 3));
    }
    if (j0 + 8 <= nb) {
        *reinterpret_cast<uint32_t *>(qabs + j0) = w[0];
        *reinterpret_cast<uint32_t *>(qabs + j0 + 4) = w[1];
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (j0 + i < nb) qabs[j0 + i] = (int8_t)((w[i >> 2] >> (8 * (i & 3))) & 0xff);
    }
}

// ===========================================================================
// K3: each warp quantizes one group of 256 constants: d = fp32(a - mu),
// b = fp32(max|d| / 127), rhat = clamp(rint(fp32(d / b)), -127, 127).  Every
// CTA first folds the np K2 partials (zero-padded to P = a power of two >= 8)
// into S and mu = fp32(S / nb) -- the top of the same tree, so mu is
// bit-exact: warp w folds the aligned slice [w P/8, (w+1) P/8) (lane-local
// pairs, then a butterfly) and one thread folds the 8 slice sums.  The
// group's constants are requested before the fold.
// ===========================================================================
constexpr int kDqThreads = 256;

__global__ void __launch_bounds__(kDqThreads) dq_quant_kernel(const float *__restrict__ a, int64_t nb,
                                                              const double *__restrict__ partial, int np,
                                                              int P, int8_t *__restrict__ qabs,
                                                              float *__restrict__ scale, float *__restrict__ mu_out,
                                                              bool e4m3) {
    __shared__ double slice[kDqThreads / 32];
    __shared__ float mu_s;
    pdl_wait();
    // writes the DQ constants of a weight: no early release (see the quantize kernel)
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t g = (int64_t)blockIdx.x * (kDqThreads / 32) + warp;
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    const int64_t j0 = g * kDqGroup + 8 * lane;  // this lane's 8 consecutive constants
    float e[8];
    load8_const(e, a, g < ng ? j0 : nb, nb);

    {   // the partial sums: L leaves per warp, c per lane (P <= 1024, so c <= 4)
        const int L = P / 8;
        const int c = L >= 32 ? L / 32 : 1;
        const int first = warp * L + lane * c;
        double s = 0.0;
        if (lane * c < L) {
            double t[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) t[i] = (i < c && first + i < np) ? __ldcg(partial + first + i) : 0.0;
            s = c == 1 ? t[0] : c == 2 ? __dadd_rn(t[0], t[1]) : __dadd_rn(__dadd_rn(t[0], t[1]), __dadd_rn(t[2], t[3]));
        }
        int levels = 0;
        for (int span = L / c; span > 1 && levels < 5; span >>= 1) ++levels;
        s = warp_butterfly_sum(s, levels);
        if (lane == 0) slice[warp] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const double w01 = __dadd_rn(slice[0], slice[1]), w23 = __dadd_rn(slice[2], slice[3]);
        const double w45 = __dadd_rn(slice[4], slice[5]), w67 = __dadd_rn(slice[6], slice[7]);
        const double S = __dadd_rn(__dadd_rn(w01, w23), __dadd_rn(w45, w67));
        const float mu = __double2float_rn(__ddiv_rn(S, (double)nb));
        mu_s = mu;
        if (blockIdx.x == 0) *mu_out = mu;
    }
    __syncthreads();
    const float mu = mu_s;
    if (g >= ng) return;
    dq_quantize_group(e, j0, nb, mu, e4m3, lane, g, qabs, scale);
}

// ===========================================================================
// Fused double quantization (the workspace entry point): one launch that
// forms the mean, waits on a grid-wide barrier and quantizes.
//  1. CTA c owns the 8 * GPW groups [8 GPW c, 8 GPW (c + 1)) -- an aligned
//     subtree of 2048 GPW block constants.  Each warp keeps its GPW groups'
//     constants in registers, sums each group as a binary64 perfect tree (8
//     leaves per lane, then a butterfly), folds its groups and the CTA folds
//     its 8 warps, both pairwise: the CTA's partial is exactly that subtree of
//     the whole-tensor tree.  It is published in the workspace.
//  2. Barrier: the CTA counts itself in (release) and waits, bounded by
//     kDqfWaitNs, until all G CTAs have (acquire).  G never exceeds the CTAs
//     the device holds at once, so every CTA is resident.
//  3. Every CTA folds the G partials (zero-padded to P, the top of the same
//     tree: mu is bit-exact), then quantizes its groups from registers.
// The workspace header holds the status word (offset 0), the arrival counter
// (64) and the departure counter (128); the last CTA to leave puts both
// counters back to zero, so every call starts from and leaves a zeroed header.
// ===========================================================================
constexpr int kDqfArriveOffset = 64;
constexpr int kDqfLeaveOffset = 128;
constexpr uint64_t kDqfWaitNs = 2000000000ull;

__device__ __forceinline__ int dqf_ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint64_t dqf_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

template <int GPW>
__global__ void __launch_bounds__(kDqThreads) dq_fused_kernel(const float *__restrict__ a, int64_t nb,
                                                              int8_t *__restrict__ qabs, float *__restrict__ scale,
                                                              float *__restrict__ mu_out, unsigned char *ws, int G,
                                                              int P, bool e4m3) {
    __shared__ double wsum[kDqThreads / 32];
    __shared__ float mu_s;
    __shared__ int ok_s;
    int *status = reinterpret_cast<int *>(ws);
    int *arrive = reinterpret_cast<int *>(ws + kDqfArriveOffset);
    int *leave = reinterpret_cast<int *>(ws + kDqfLeaveOffset);
    double *partial = reinterpret_cast<double *>(ws + 256);
    pdl_wait();  // the constants come from the previous kernel (the quantize)
    // writes the DQ constants of a weight: no early release (see the quantize kernel)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    const int64_t g0 = ((int64_t)blockIdx.x * (kDqThreads / 32) + warp) * GPW;
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = QLN_OK;

    // ---- 1. this CTA's subtree of the mean -----------------------------------
    float e[GPW][8];
    double gs[GPW];
#pragma unroll
    for (int i = 0; i < GPW; ++i) {
        const int64_t j0 = (g0 + i) * kDqGroup + 8 * lane;
        load8_const(e[i], a, (g0 + i) < ng ? j0 : nb, nb);
        gs[i] = warp_butterfly_sum(tree8(e[i]), 5);
    }
#pragma unroll
    for (int len = GPW; len > 1; len >>= 1)
#pragma unroll
        for (int i = 0; i < len / 2; ++i) gs[i] = __dadd_rn(gs[2 * i], gs[2 * i + 1]);
    if (lane == 0) wsum[warp] = gs[0];
    __syncthreads();
    if (threadIdx.x == 0) {
        const double w01 = __dadd_rn(wsum[0], wsum[1]), w23 = __dadd_rn(wsum[2], wsum[3]);
        const double w45 = __dadd_rn(wsum[4], wsum[5]), w67 = __dadd_rn(wsum[6], wsum[7]);
        __stcg(partial + blockIdx.x, __dadd_rn(__dadd_rn(w01, w23), __dadd_rn(w45, w67)));
        __threadfence();
        atomicAdd(arrive, 1);
        // ---- 2. grid barrier, bounded -------------------------------------------
        bool ok = dqf_ld_acquire(arrive) >= G;
        if (!ok) {
            const uint64_t t0 = dqf_timer_ns();
            for (uint32_t it = 0; !ok; ++it) {
                ok = dqf_ld_acquire(arrive) >= G;
                if (!ok && (it & 63u) == 63u && dqf_timer_ns() - t0 > kDqfWaitNs) break;
            }
        }
        if (!ok) atomicExch(status, (int)QLN_ERR_TIMEOUT);
        ok_s = ok;
    }
    __syncthreads();
    const bool ok = ok_s != 0;

    // ---- 3. mu from the G partials, then the groups ----------------------------
    if (ok) {
        const int L = P / 8;  // leaves per warp slice; P <= 2048, so c <= 8
        const int c = L >= 32 ? L / 32 : 1;
        const int first = warp * L + lane * c;
        double s = 0.0;
        if (lane * c < L) {
            double t[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) t[i] = (i < c && first + i < G) ? __ldcg(partial + first + i) : 0.0;
#pragma unroll
            for (int len = 8; len > 1; len >>= 1)
#pragma unroll
                for (int i = 0; i < len / 2; ++i) t[i] = __dadd_rn(t[2 * i], t[2 * i + 1]);
            // leaves past c are zero, so the 8-leaf tree equals the c-leaf one
            s = t[0];
        }
        int levels = 0;
        for (int span = L / c; span > 1 && levels < 5; span >>= 1) ++levels;
        s = warp_butterfly_sum(s, levels);
        __syncthreads();  // wsum is reused
        if (lane == 0) wsum[warp] = s;
        __syncthreads();
        if (threadIdx.x == 0) {
            const double w01 = __dadd_rn(wsum[0], wsum[1]), w23 = __dadd_rn(wsum[2], wsum[3]);
            const double w45 = __dadd_rn(wsum[4], wsum[5]), w67 = __dadd_rn(wsum[6], wsum[7]);
            const double S = __dadd_rn(__dadd_rn(w01, w23), __dadd_rn(w45, w67));
            const float mu = __double2float_rn(__ddiv_rn(S, (double)nb));
            mu_s = mu;
            if (blockIdx.x == 0) *mu_out = mu;
        }
        __syncthreads();
        const float mu = mu_s;
#pragma unroll
        for (int i = 0; i < GPW; ++i)
            if (g0 + i < ng) dq_quantize_group(e[i], (g0 + i) * kDqGroup + 8 * lane, nb, mu, e4m3, lane, g0 + i, qabs,
                                               scale);
    }
    // ---- leave: the last CTA out zeroes the counters for the next call --------
    if (threadIdx.x == 0 && ok && atomicAdd(leave, 1) == G - 1) {
        *arrive = 0;
        *leave = 0;
    }
}

// Leaves per K2 CTA: 2048 * NG with NG the smallest power of two (<= 16) that
// keeps the partial count within kMaxPartials.
static int dq_groups_per_thread(int64_t nb) {
    int ng = 1;
    while (ng < 16 && (nb + 2048LL * ng - 1) / (2048LL * ng) > kMaxPartials) ng <<= 1;
    return ng;
}

static int64_t dq_partial_count(int64_t nb) {
    const int64_t C = 2048LL * dq_groups_per_thread(nb);
    return (nb + C - 1) / C;
}

size_t dq_workspace_bytes(int64_t nb) {
    const int64_t fused = ((nb + kDqGroup - 1) / kDqGroup + 7) / 8;  // one partial per CTA of the fused kernel
    const int64_t np = dq_partial_count(nb) > fused ? dq_partial_count(nb) : fused;
    return (size_t)(256 + ((np * 8 + 255) / 256) * 256);
}

// CTAs of the fused kernel the device holds at once (cached per variant).
template <int GPW>
static int dq_fused_capacity(int num_sms) {
    static std::atomic<int> cached{0};
    int per_sm = cached.load(std::memory_order_relaxed);
    if (per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dq_fused_kernel<GPW>, kDqThreads, 0) !=
            cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        cached.store(per_sm, std::memory_order_relaxed);
    }
    return per_sm * num_sms;
}

// The fused kernel when its grid fits on the device at once; false when it
// does not (then the two-kernel path runs).
template <int GPW>
static bool try_dq_fused(const float *absmax, int64_t nb, int8_t *qabs, float *scale, float *mu, void *ws, bool e4m3,
                         cudaStream_t st, int num_sms, cudaError_t *err) {
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    const int64_t G = (ng + 8 * GPW - 1) / (8 * GPW);
    if (G > dq_fused_capacity<GPW>(num_sms)) return false;
    int P = 8;
    while (P < G) P <<= 1;
    if (P > 2048) return false;
    *err = launch_pdl(dq_fused_kernel<GPW>, dim3((unsigned)G), dim3(kDqThreads), 0, st, absmax, nb, qabs, scale, mu,
                      static_cast<unsigned char *>(ws), (int)G, P, e4m3);
    return true;
}

int64_t dq_max_blocks() { return kMeanMaxBlocks; }

// K2 then K3, each launched as a programmatic dependent of the kernel before it.
static cudaError_t launch_dq_pair(const float *absmax, int64_t nb, double *partial, int8_t *qabs, float *scale,
                                  float *mu, bool e4m3, cudaStream_t st) {
    const int NG = dq_groups_per_thread(nb);
    const int np = (int)dq_partial_count(nb);
    int P = 8;
    while (P < np) P <<= 1;
    cudaError_t e;
    const dim3 g2((unsigned)np), b2(kMeanThreads);
    switch (NG) {
        case 1: e = launch_pdl(dq_partial_kernel<1>, g2, b2, 0, st, absmax, nb, partial); break;
        case 2: e = launch_pdl(dq_partial_kernel<2>, g2, b2, 0, st, absmax, nb, partial); break;
        case 4: e = launch_pdl(dq_partial_kernel<4>, g2, b2, 0, st, absmax, nb, partial); break;
        case 8: e = launch_pdl(dq_partial_kernel<8>, g2, b2, 0, st, absmax, nb, partial); break;
        default: e = launch_pdl(dq_partial_kernel<16>, g2, b2, 0, st, absmax, nb, partial); break;
    }
    if (e != cudaSuccess) return e;
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    const int64_t grid = (ng + (kDqThreads / 32) - 1) / (kDqThreads / 32);
    return launch_pdl(dq_quant_kernel, dim3((unsigned)grid), dim3(kDqThreads), 0, st, absmax, nb,
                      (const double *)partial, np, P, qabs, scale, mu, e4m3);
}

cudaError_t launch_nf4_double_quant(const float *absmax, int64_t nb, int8_t *qabs, float *scale, float *mu,
                                    void *ws, bool e4m3, cudaStream_t st, int num_sms) {
    cudaError_t e = cudaSuccess;
    // Measured on B200 (CUDA graphs, after the quantize): the single launch with
    // one group per warp saves ~1.7 us on an 11008 x 4096 weight and is within
    // 0.2 us of the two kernels on 4096 x 4096; more groups per warp serialise
    // each warp's work (8 per warp: 12.9 us against 4.9 us), so weights too
    // large for one group per warp take the two kernels.
    if (try_dq_fused<1>(absmax, nb, qabs, scale, mu, ws, e4m3, st, num_sms, &e)) return e;
    double *partial = reinterpret_cast<double *>(reinterpret_cast<char *>(ws) + 256);
    return launch_dq_pair(absmax, nb, partial, qabs, scale, mu, e4m3, st);
}

// ===========================================================================
// Allocation-free double quantization.  The only scratch K2/K3 need is the
// binary64 partial sums of mu (at most kMaxPartials of them).  This variant
// keeps them in a fixed, file-scope device array instead of a caller
// workspace, so a caller that cannot allocate device memory can still run the
// path.  The array is 8 KB; the entry point accepts nb up to 1024 * 8192 =
// 8,388,608 blocks (536,870,912 weights); every GPU that loads the library
// holds it until the process exits.  Each call overwrites every partial it
// reads before reading it, so nothing has to be cleared between calls; two
// calls that overlap on the GPU (different streams, no ordering) share the
// array and race.
// ===========================================================================
constexpr int kStaticPartials = kMaxPartials;
static __device__ __align__(256) double g_dq_static_partials[kStaticPartials];
static std::atomic<double *> g_dq_static_ptr[64];

int64_t dq_static_max_blocks() { return (int64_t)1024 * 8192; }

// Device address of the array on the current device.  In host code the
// symbol names a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
static cudaError_t dq_static_partials(double **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    double *p = g_dq_static_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        void *addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_dq_static_partials);
        if (e != cudaSuccess) return e;
        p = static_cast<double *>(addr);
        g_dq_static_ptr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return cudaSuccess;
}

cudaError_t launch_nf4_double_quant_static(const float *absmax, int64_t nb, int8_t *qabs, float *scale, float *mu,
                                           cudaStream_t st) {
    double *partial = nullptr;
    cudaError_t e = dq_static_partials(&partial);
    if (e != cudaSuccess) return e;
    return launch_dq_pair(absmax, nb, partial, qabs, scale, mu, false, st);
}

// ===========================================================================
// K4: doubleDequant to BF16.  A warp takes 1024 consecutive weights at a time
// (512 bytes of codes, 16 blocks): lane l loads 16 bytes, 32 weights of block
// l/2.  The code bytes and constants of the warp's next two chunks are
// requested before the current one is decoded.  The decode is register-only:
// the 16 products bf16_RN(fp32(ahat * c[q])) of the block are built once and
// split into byte tables, and a byte permute looks up four codes at a time --
// exactly w' = bf16_RN(fp32(ahat * c[q])).  The 2 KB of BF16 go through a
// per-warp shared buffer (16-byte pieces rotated so that neither side has
// bank conflicts) and leave as four 512-byte rows, one contiguous store
// instruction each.
// ===========================================================================
struct DeqIn {
    uint4 cw;   // 32 codes
    int8_t q;   // DQ code of the block (or unused)
    float v;    // DQ scale of the block's group, or the plain absmax
};

__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint4 *__restrict__ codes128,
                                                          const float *__restrict__ absmax,
                                                          const int8_t *__restrict__ qabs,
                                                          const float *__restrict__ scale,
                                                          const float *__restrict__ mu_p, int64_t nchunks,
                                                          uint4 *__restrict__ out, bool e4m3) {
    __shared__ __align__(16) uint4 stage[8][128];  // per warp 2 KB
    pdl_wait();  // the weight may come from the previous kernel on the stream
    pdl_trigger();
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    uint4 *buf = stage[wib];
    const float mu = qabs ? __ldg(mu_p) : 0.f;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    auto fetch = [&](int64_t ch, DeqIn &d) {
        if (ch < nchunks) {
            const int64_t i = ch * 32 + lane;  // 32-weight group
            const int64_t j = i >> 1;          // two groups per block
            d.cw = __ldcs(codes128 + i);
            if (qabs) {
                d.q = __ldg(qabs + j);
                d.v = __ldg(scale + (j >> 8));
            } else {
                d.q = 0;
                d.v = __ldg(absmax + j);
            }
        }
    };
    int64_t ch = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib;
    DeqIn d0, d1, d2;
    fetch(ch, d0);
    fetch(ch + nwarps, d1);
    for (; ch < nchunks; ch += nwarps) {
        fetch(ch + 2 * nwarps, d2);
        const float ah = qabs ? dq_restore((uint32_t)d0.q, d0.v, mu, e4m3) : d0.v;
        const NF4Table t = nf4_table(ah);
        // piece w of lane l (bytes 64 l + 16 w of the chunk) sits at slot 4 l + ((w + l/2) & 3)
        const int rot = lane >> 1;
        buf[4 * lane + ((0 + rot) & 3)] = nf4_decode8(d0.cw.x, t);
        buf[4 * lane + ((1 + rot) & 3)] = nf4_decode8(d0.cw.y, t);
        buf[4 * lane + ((2 + rot) & 3)] = nf4_decode8(d0.cw.z, t);
        buf[4 * lane + ((3 + rot) & 3)] = nf4_decode8(d0.cw.w, t);
        __syncwarp();
        uint4 *o = out + ch * 128;
#pragma unroll
        for (int row = 0; row < 4; ++row) {
            const int piece = 32 * row + lane;            // 16-byte piece of the chunk
            const int src = piece >> 2, w = piece & 3;    // written by lane src as its piece w
            __stcs(o + piece, buf[4 * src + ((w + (src >> 1)) & 3)]);
        }
        __syncwarp();
        d0 = d1;
        d1 = d2;
    }
}

// The last (numel mod 1024) weights: one thread per 32-weight group.
__global__ void nf4_dequant_tail_kernel(const uint4 *__restrict__ codes128, const float *__restrict__ absmax,
                                        const int8_t *__restrict__ qabs, const float *__restrict__ scale,
                                        const float *__restrict__ mu_p, int64_t g0, int64_t ng,
                                        uint4 *__restrict__ out, bool e4m3) {
    const int64_t k = threadIdx.x;
    if (k >= ng) return;
    const int64_t i = g0 + k, j = i >> 1;
    const float ah = qabs ? dq_restore((uint32_t)__ldg(qabs + j), __ldg(scale + (j >> 8)), __ldg(mu_p), e4m3)
                          : __ldg(absmax + j);
    const NF4Table t = nf4_table(ah);
    const uint4 cw = __ldg(codes128 + i);
    out[4 * i + 0] = nf4_decode8(cw.x, t);
    out[4 * i + 1] = nf4_decode8(cw.y, t);
    out[4 * i + 2] = nf4_decode8(cw.z, t);
    out[4 * i + 3] = nf4_decode8(cw.w, t);
}

// Ragged end of a flat weight: one thread per weight, w' = bf16_RN(fp32(ahat * c[q])).
__global__ void nf4_dequant_elem_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ absmax,
                                        const int8_t *__restrict__ qabs, const float *__restrict__ scale,
                                        const float *__restrict__ mu_p, int64_t e0, int64_t numel,
                                        uint16_t *__restrict__ out, bool e4m3) {
    const int64_t e = e0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= numel) return;
    const int64_t j = e >> 6;
    const float ah = qabs ? dq_restore((uint32_t)__ldg(qabs + j), __ldg(scale + (j >> 8)), __ldg(mu_p), e4m3)
                          : __ldg(absmax + j);
    const uint32_t byte = __ldg(codes + (e >> 1));
    const int q = (e & 1) ? (int)(byte & 15u) : (int)(byte >> 4);
    const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(ah, nf4_value(q)));
    out[e] = *reinterpret_cast<const uint16_t *>(&b);
}

static cudaError_t launch_dequant_numel(const qln_nf4_weight *w, int64_t numel, uint16_t *out, cudaStream_t st,
                                        int num_sms);

cudaError_t launch_nf4_dequant(const qln_nf4_weight *w, uint16_t *out, cudaStream_t st, int num_sms) {
    return launch_dequant_numel(w, w->rows * w->cols, out, st, num_sms);
}

cudaError_t launch_nf4_dequant_flat(const qln_nf4_weight *w, int64_t numel, uint16_t *out, cudaStream_t st,
                                    int num_sms) {
    return launch_dequant_numel(w, numel, out, st, num_sms);
}

static cudaError_t launch_dequant_numel(const qln_nf4_weight *w, int64_t numel, uint16_t *out, cudaStream_t st,
                                        int num_sms) {
    const bool e4m3 = w->dq_format == QLN_DQ_E4M3;
    const int64_t nchunks = numel / 1024;  // weights come in whole 64-blocks; chunks of 1024 + a tail below
    const int64_t tail = numel - nchunks * 1024;
    int64_t grid = (nchunks + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 6;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    if (nchunks > 0) {
        cudaError_t e = launch_pdl(nf4_dequant_kernel, dim3((unsigned)grid), dim3(256), 0, st,
                                   reinterpret_cast<const uint4 *>(w->codes), w->absmax, w->qabs, w->dq_scale,
                                   w->dq_mean, nchunks, reinterpret_cast<uint4 *>(out), e4m3);
        if (e != cudaSuccess) return e;
    }
    const int64_t whole = (tail / 32) * 32;  // 32-weight groups of the tail: 16-byte stores
    if (whole > 0) {
        const int64_t g0 = nchunks * 32, ng = whole / 32;
        nf4_dequant_tail_kernel<<<1, 64, 0, st>>>(reinterpret_cast<const uint4 *>(w->codes), w->absmax, w->qabs,
                                                   w->dq_scale, w->dq_mean, g0, ng, reinterpret_cast<uint4 *>(out),
                                                   e4m3);
        note_launch();
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (tail > whole) {  // fewer than 32 weights: one thread each
        nf4_dequant_elem_kernel<<<1, 32, 0, st>>>(w->codes, w->absmax, w->qabs, w->dq_scale, w->dq_mean,
                                                   nchunks * 1024 + whole, numel, out, e4m3);
        note_launch();
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace qln
