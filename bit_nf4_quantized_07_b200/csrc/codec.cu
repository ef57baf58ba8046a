// NF4 codec kernels: blockwise quantize (K1), double quantization (K2 + K3),
// doubleDequant to BF16 (K4).  All HBM-bound streaming kernels.
//
// Method: jjjymmm.cn 2024/03 QLoRA post, "4-bit NormalFloat(NF4)" (divide by
// the block ABSMAX, snap to the nearest book entry; dequantize = book value),
// "Double Quantization" and "QLoRA" (doubleDequant: constants first);
// "LoRA 与 QLoRA" section QLoRA 2 (a_j = max|W_j| per 64 weights,
// r_j = (a_j - mu)/b, 8-bit rhat_j, ahat_j = mu + b rhat_j).
#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include <cuda.h>
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

// ===========================================================================
// The DQ mean mu: the binary32 value nearest to the exact mean of the block
// constants, ties to even ("LoRA 与 QLoRA", section 2: subtract the mean mu;
// mu is kept in 32 bits).
//
// Exact sums.  Every finite binary32 value is an integer number of units of
// 2^-149: |a| = m * 2^s units with m < 2^24 and s = max(exponent field, 1) - 1
// in [0, 253].  A sum is held as kXLimbs signed 64-bit limbs, limb k weighing
// 2^(32 k) units.  A thread keeps a run of values that fall on the same limb
// pair in one 64-bit word (at most 64 values of < 2^55 each), and a run is
// added to the limbs as a low part (< 2^32) on limb k and a high part on limb
// k + 1.  Integer addition is associative, so the result does not depend on the
// order in which threads, warps or CTAs add their parts, and no limb can
// overflow for fewer than 2^30 values.
// ===========================================================================
constexpr int kXLimbs = 10;  // 320 bits: a value reaches bit 277; the rest holds carries and the sign
constexpr int64_t kMeanMaxBlocks = (int64_t)1 << 25;  // nb limit (numel 2^31); the limbs stay exact to 2^30

struct XRun {
    long long acc = 0;  // sum of the run, in units of 2^(32 k)
    int k = -1;         // limb of the run (-1: empty)
    int cnt = 0;
};

__device__ __forceinline__ void xsum_flush_lane(XRun &x, unsigned long long *lim) {
    if (x.k >= 0 && x.acc != 0) {
        atomicAdd(&lim[x.k], (unsigned long long)(x.acc & 0xffffffffll));
        atomicAdd(&lim[x.k + 1], (unsigned long long)(x.acc >> 32));
    }
    x.acc = 0;
    x.k = -1;
    x.cnt = 0;
}

// Adds one binary32 value (finite) to this thread's run; a value on another
// limb pair (rare: the constants of one weight are close in magnitude) first
// sends the run to the shared limbs.
__device__ __forceinline__ void xsum_add(XRun &x, float v, unsigned long long *lim) {
    const uint32_t b = __float_as_uint(v);
    const int e = (int)((b >> 23) & 0xffu);
    const uint32_t m = (b & 0x7fffffu) | (e ? 0x800000u : 0u);
    if (m == 0) return;
    const int s = (e > 1 ? e : 1) - 1;
    const int k = s >> 5;
    if (k != x.k || x.cnt == 64) {
        xsum_flush_lane(x, lim);
        x.k = k;
    }
    const long long t = (long long)m << (s & 31);
    x.acc += (b >> 31) ? -t : t;
    ++x.cnt;
}

// A warp's runs into the shared limbs: one pair of atomics per warp when every
// lane's run sits on the same limb pair (the usual case), else one per lane.
__device__ __forceinline__ void xsum_flush_warp(XRun &x, unsigned long long *lim) {
    const int kk = x.acc != 0 ? x.k : -1;
    const int k0 = (int)__reduce_max_sync(0xffffffffu, (unsigned)(kk + 1)) - 1;
    if (__all_sync(0xffffffffu, kk == -1 || kk == k0)) {
        long long lo = kk >= 0 ? (x.acc & 0xffffffffll) : 0, hi = kk >= 0 ? (x.acc >> 32) : 0;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            lo += __shfl_xor_sync(0xffffffffu, lo, o);
            hi += __shfl_xor_sync(0xffffffffu, hi, o);
        }
        if ((threadIdx.x & 31) == 0 && k0 >= 0) {
            atomicAdd(&lim[k0], (unsigned long long)lo);
            atomicAdd(&lim[k0 + 1], (unsigned long long)hi);
        }
        x.acc = 0;
        x.k = -1;
        x.cnt = 0;
    } else {
        xsum_flush_lane(x, lim);
    }
}

// mu = the binary32 value nearest to (limbs / nb) units, ties to even, by one
// thread.  The limbs are carried into 32-bit digits d (two's complement over
// the digits for a negative sum) and the magnitude S is cut to its top 64
// bits, S = T 2^sh + R with T >= 2^63 when sh > 0 (and R < 2^sh), or T = S and
// sh = 0.  Then S / nb = (T div nb) 2^sh + (rem 2^sh + R) / nb: the quotient
// q = T div nb has at least 39 bits when sh > 0 (nb < 2^25), and the exact
// mean has bits below q's last exactly when rem or R is nonzero -- enough for
// 24 significant bits, the guard bit and the sticky bit, from one 64-bit
// division.
__device__ float xsum_mean(const unsigned long long (&limb)[kXLimbs], uint32_t nb) {
    uint32_t d[kXLimbs];
    long long carry = 0;
#pragma unroll
    for (int k = 0; k < kXLimbs; ++k) {
        const long long v = (long long)limb[k] + carry;
        d[k] = (uint32_t)v;
        carry = (v - (long long)(uint32_t)v) >> 32;
    }
    const bool neg = carry < 0;
    if (neg) {  // magnitude of a negative two's complement number
        uint32_t c = 1;
#pragma unroll
        for (int k = 0; k < kXLimbs; ++k) {
            const uint64_t t = (uint64_t)(~d[k]) + c;
            d[k] = (uint32_t)t;
            c = (uint32_t)(t >> 32);
        }
    }
    int t = 0;  // top nonzero digit (0 for a zero sum)
#pragma unroll
    for (int k = 1; k < kXLimbs; ++k)
        if (d[k] != 0) t = k;
    uint64_t T;
    int sh = 0;
    bool R = false;  // a nonzero bit of S below T
    if (t < 2) {
        T = ((uint64_t)d[1] << 32) | d[0];
    } else {
        uint32_t d2 = 0, d1 = 0, d0 = 0;
#pragma unroll
        for (int k = 2; k < kXLimbs; ++k) {
            if (k == t) { d2 = d[k]; d1 = d[k - 1]; d0 = d[k - 2]; }
            if (k < t && d[k - 2] != 0) R = true;  // digits below t - 2
        }
        const int z = __clz(d2);  // d2 != 0
        const uint64_t top = ((uint64_t)d2 << 32) | d1;
        T = z ? (top << z) | (d0 >> (32 - z)) : top;  // 64 bits from bit 32 t + 31 - z down
        if (z ? (d0 << z) != 0u : d0 != 0u) R = true;
        sh = 32 * (t - 2) + 32 - z;
    }
    const uint64_t q = T / nb;
    const uint64_t rem = T - q * nb;
    const int lb = q ? 63 - __clzll((long long)q) : -1;
    uint32_t bits;
    if (sh + lb <= 23) {  // below 2^-125 (then sh == 0): the value in units is the pattern itself
        uint32_t k = (uint32_t)q;
        if (2 * rem > nb || (2 * rem == nb && (k & 1u))) ++k;
        bits = k;
    } else {
        const int rs = lb - 23;  // >= 1: q's bits below rs are rounded off
        const uint32_t sig = (uint32_t)(q >> rs) & 0xffffffu;
        const uint64_t below = q & ((1ull << rs) - 1);
        const uint64_t half = 1ull << (rs - 1);
        const bool guard = (below & half) != 0;
        const bool sticky = (below & (half - 1)) != 0 || rem != 0 || R;
        uint32_t m = sig;
        if (guard && (sticky || (m & 1u))) ++m;
        const uint64_t b64 = ((uint64_t)(sh + rs + 1) << 23) + m - (1u << 23);
        bits = b64 >= 0x7f800000ull ? 0x7f800000u : (uint32_t)b64;
    }
    return __uint_as_float(bits | (neg ? 0x80000000u : 0u));
}

// The limbs read by lanes 0..kXLimbs-1 of the calling warp (one coalesced
// request) and mu formed by lane 0; every lane of the warp must call it.
__device__ __forceinline__ float xsum_mean_warp(const unsigned long long *glim, uint32_t nb) {
    const int lane = threadIdx.x & 31;
    const unsigned long long mine = lane < kXLimbs ? __ldcg(glim + lane) : 0ull;
    unsigned long long L[kXLimbs];
#pragma unroll
    for (int k = 0; k < kXLimbs; ++k) L[k] = __shfl_sync(0xffffffffu, mine, k);
    return lane == 0 ? xsum_mean(L, nb) : 0.f;
}

// The DQ scratch (256 bytes): a status word, a generation word, an arrival
// counter and two banks of limbs.  A call reads the generation g at its start
// and sums into bank g % 2, which is zero; the last CTA of the call's summing
// kernel to arrive puts the counter back to zero, zeroes the other bank and
// then advances the generation, so the next call finds its bank zeroed and
// nothing has to be cleared after the last reader.
struct DqScratch {
    int *status;  // null: none (the allocation-free entry point)
    unsigned *gen;
    int *arrive;
    unsigned long long *bank[2];  // [kXLimbs] each
};
constexpr int kDqStatusOffset = 0, kDqGenOffset = 16, kDqArriveOffset = 32, kDqBank0Offset = 64, kDqBank1Offset = 160;
constexpr size_t kDqScratchBytes = 256;
static_assert(kDqBank0Offset + 8 * kXLimbs <= kDqBank1Offset && kDqBank1Offset + 8 * kXLimbs <= (int)kDqScratchBytes,
              "limb banks inside the scratch");

__device__ __forceinline__ DqScratch dq_scratch(unsigned char *ws, bool with_status) {
    DqScratch d;
    d.status = with_status ? reinterpret_cast<int *>(ws + kDqStatusOffset) : nullptr;
    d.gen = reinterpret_cast<unsigned *>(ws + kDqGenOffset);
    d.arrive = reinterpret_cast<int *>(ws + kDqArriveOffset);
    d.bank[0] = reinterpret_cast<unsigned long long *>(ws + kDqBank0Offset);
    d.bank[1] = reinterpret_cast<unsigned long long *>(ws + kDqBank1Offset);
    return d;
}

// The generation, read by thread 0 and shared with the CTA (every thread calls).
__device__ __forceinline__ unsigned dq_read_gen(const DqScratch &sc, unsigned *gen_s) {
    if (threadIdx.x == 0) *gen_s = __ldcg(sc.gen);
    __syncthreads();
    return *gen_s;
}

// Thread 0, after the CTA's limbs are in bank g % 2: count this CTA in; the
// last of G to arrive resets the counter, zeroes the other bank and publishes
// generation g + 1 (a release, after everything it has seen).  Returns whether
// this CTA was the last.
__device__ __forceinline__ bool dq_arrive(const DqScratch &sc, unsigned g, int G) {
    __threadfence();
    if (atomicAdd(sc.arrive, 1) != G - 1) return false;
    *sc.arrive = 0;
    unsigned long long *other = sc.bank[(g + 1) & 1];
#pragma unroll
    for (int k = 0; k < kXLimbs; ++k) other[k] = 0ull;
    __threadfence();
    atomicExch(sc.gen, g + 1);
    return true;
}

// 8 consecutive constants starting at j (zeros past nb), read through L2: they
// come from the previous kernel, which may still have been running when this
// one started (programmatic dependent launch).
__device__ __forceinline__ void load8_const(float (&v)[8], const float *a, int64_t j, int64_t nb) {
    if (j + 8 <= nb) {
        const float4 x = __ldcg(reinterpret_cast<const float4 *>(a + j));
        const float4 y = __ldcg(reinterpret_cast<const float4 *>(a + j + 4));
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
        v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = (j + i < nb) ? __ldcg(a + j + i) : 0.f;
    }
}

// This CTA's constants into its shared limbs, then into the scratch limbs.
// Every thread of the CTA calls it; on return the CTA's part is published.
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

// Grid-wide barrier helpers: an acquiring load of a counter, the global timer.
constexpr uint64_t kDqfWaitNs = 2000000000ull;

__device__ __forceinline__ unsigned dqf_ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint64_t dqf_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

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

//
// kLateWait (the batch entry point, second weight on, buffers of all jobs
// disjoint): the kernel reads only the caller's weight, which was complete
// before the batch's first launch passed its wait, and writes only its own
// outputs, which nothing else in the batch touches; so it releases its
// dependents and starts at once, filling the SMs the previous weight's
// kernels leave, and waits for its predecessor only at its end -- its
// completion then still implies that everything before it in the stream has
// completed.
template <typename T, typename Idx, bool kLateWait>
__global__ void __launch_bounds__(kQzThreads, kQzCtasPerSm) nf4_quantize_kernel(const T *__restrict__ W, Idx numel,
                                                                                uint8_t *__restrict__ codes,
                                                                                float *__restrict__ absmax) {
    constexpr int kB = QzIn<T>::kBytes;
    extern __shared__ __align__(16) unsigned char qz_smem[];
    for (int i = threadIdx.x; i < kQzLutBytes / 4; i += kQzThreads)  // bucket i/32, lane i%32
        reinterpret_cast<uint32_t *>(qz_smem)[i] = kSnapTable.e[i >> 5];
    __syncthreads();
    if (!kLateWait) pdl_wait();  // W may come from the previous kernel; codes/absmax may still be read by it
    pdl_trigger();

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
    if (kLateWait) pdl_wait();
}

// Launch of the quantize kernel: a persistent grid of up to two CTAs per SM,
// as a programmatic dependent.
template <typename T, typename Idx, bool kLateWait>
static cudaError_t launch_quantize_t(const T *W, int64_t numel, uint8_t *codes, float *absmax, cudaStream_t st,
                                     int num_sms) {
    const int64_t nchunks = ((numel + 63) / 64 + 3) / 4;
    int64_t grid = (nchunks + kQzWarps - 1) / kQzWarps;
    if (grid > (int64_t)kQzCtasPerSm * num_sms) grid = (int64_t)kQzCtasPerSm * num_sms;
    if (grid < 1) grid = 1;
    const int smem = kQzLutBytes + kQzWarps * kQzStages * 256 * QzIn<T>::kBytes;
    auto kern = nf4_quantize_kernel<T, Idx, kLateWait>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(kQzThreads), (size_t)smem, st, W, (Idx)numel, codes, absmax);
}

template <typename T, bool kLateWait>
static cudaError_t launch_quantize_any(const void *W, int64_t numel, uint8_t *codes, float *absmax, cudaStream_t st,
                                       int num_sms) {
    const T *w = static_cast<const T *>(W);
    // 32-bit indices while every element offset (and a chunk look-ahead per warp) stays below 2^31
    if (numel + (int64_t)256 * (kQzStages + 1) * kQzCtasPerSm * num_sms * kQzWarps < ((int64_t)1 << 31))
        return launch_quantize_t<T, uint32_t, kLateWait>(w, numel, codes, absmax, st, num_sms);
    return launch_quantize_t<T, int64_t, kLateWait>(w, numel, codes, absmax, st, num_sms);
}

template <bool kLateWait>
static cudaError_t launch_quantize_dtype(const void *W, int dtype, int64_t numel, uint8_t *codes, float *absmax,
                                         cudaStream_t st, int num_sms) {
    switch (dtype) {
        case QLN_DTYPE_BF16: return launch_quantize_any<Bf16In, kLateWait>(W, numel, codes, absmax, st, num_sms);
        case QLN_DTYPE_F16: return launch_quantize_any<F16In, kLateWait>(W, numel, codes, absmax, st, num_sms);
        default: return launch_quantize_any<float, kLateWait>(W, numel, codes, absmax, st, num_sms);
    }
}

cudaError_t launch_nf4_quantize(const void *W, int dtype, int64_t numel, uint8_t *codes, float *absmax,
                                cudaStream_t st, int num_sms) {
    return launch_quantize_dtype<false>(W, dtype, numel, codes, absmax, st, num_sms);
}

template <int P>
__device__ __forceinline__ void dq_add_cta(const float (&e)[P][8], unsigned long long *slim,
                                           unsigned long long *glim) {
    XRun x;
#pragma unroll
    for (int i = 0; i < P; ++i)
#pragma unroll
        for (int u = 0; u < 8; ++u) xsum_add(x, e[i][u], slim);
    xsum_flush_warp(x, slim);
    __syncthreads();
    if (threadIdx.x < kXLimbs && slim[threadIdx.x] != 0ull) atomicAdd(&glim[threadIdx.x], slim[threadIdx.x]);
}

constexpr int kDqThreads = 256;
constexpr int kDqGroupsPerCta = kDqThreads / 32;  // one group of 256 constants per warp

// ===========================================================================
// K2: the exact sum.  Each CTA adds the constants of 8 groups per pass (8 per
// lane) into its shared limbs and then, with one reduction per nonzero limb,
// into the call's bank of the scratch; the last CTA to arrive advances the
// generation.  Nothing waits: K3 reads the bank only after this grid has
// completed.
// ===========================================================================
// CTA `bid` of the `nblk` that sum one weight's constants (slim zeroed and
// visible to the CTA on entry).
__device__ __forceinline__ void dq_sum_part(const float *__restrict__ a, int64_t nb, unsigned char *ws,
                                            bool with_status, int64_t bid, int64_t nblk, unsigned long long *slim,
                                            unsigned *gen_s) {
    const DqScratch sc = dq_scratch(ws, with_status);
    if (bid == 0 && threadIdx.x == 0 && sc.status) *sc.status = QLN_OK;
    const unsigned g0 = dq_read_gen(sc, gen_s);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    XRun x;
    for (int64_t g = bid * kDqGroupsPerCta + warp; g < ng; g += nblk * kDqGroupsPerCta) {
        float e[8];
        load8_const(e, a, g * kDqGroup + 8 * lane, nb);
#pragma unroll
        for (int u = 0; u < 8; ++u) xsum_add(x, e[u], slim);
    }
    xsum_flush_warp(x, slim);
    __syncthreads();
    if (threadIdx.x < kXLimbs && slim[threadIdx.x] != 0ull) atomicAdd(&sc.bank[g0 & 1][threadIdx.x], slim[threadIdx.x]);
    __syncthreads();
    if (threadIdx.x == 0) dq_arrive(sc, g0, (int)nblk);
}

__global__ void __launch_bounds__(kDqThreads) dq_sum_kernel(const float *__restrict__ a, int64_t nb,
                                                            unsigned char *ws, bool with_status) {
    __shared__ unsigned long long slim[kXLimbs];
    __shared__ unsigned gen_s;
    if (threadIdx.x < kXLimbs) slim[threadIdx.x] = 0ull;
    __syncthreads();
    pdl_wait();  // the constants come from the previous kernel (the quantize)
    pdl_trigger();
    dq_sum_part(a, nb, ws, with_status, blockIdx.x, gridDim.x, slim, &gen_s);
}

// ===========================================================================
// K3: the group quantization.  mu is either read (mu_in) or formed here from
// the bank K2 summed into: warp 0 of every CTA reads the limbs and forms mu
// while the other warps load their first groups, and CTA 0 writes it out.  The
// bank is zeroed by the next call's K2 (or single launch), not here.  A warp takes groups warp, warp + 8 gridDim, ... with the next group's
// constants requested before the current one is quantized.
// ===========================================================================
// CTA `bid` of the `nblk` that quantize one weight's groups.
__device__ __forceinline__ void dq_quant_part(const float *__restrict__ a, int64_t nb, int8_t *__restrict__ qabs,
                                              float *__restrict__ scale, const float *__restrict__ mu_in,
                                              float *__restrict__ mu_out, unsigned char *scratch, bool e4m3,
                                              int64_t bid, int64_t nblk, float *mu_sh) {
    float &mu_s = *mu_sh;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    const int64_t gstep = nblk * kDqGroupsPerCta;
    int64_t g = bid * kDqGroupsPerCta + warp;
    float e[8];
    load8_const(e, a, g < ng ? g * kDqGroup + 8 * lane : nb, nb);
    const DqScratch sc = dq_scratch(scratch, false);
    if (warp == 0) {
        if (scratch) {  // K2 advanced the generation: its bank is the other one
            const float mu = xsum_mean_warp(sc.bank[(__ldcg(sc.gen) + 1) & 1], (uint32_t)nb);
            if (lane == 0) {
                mu_s = mu;
                if (bid == 0) *mu_out = mu;
            }
        } else if (lane == 0) {
            mu_s = __ldcg(mu_in);
        }
    }
    __syncthreads();
    const float mu = mu_s;
    for (; g < ng; g += gstep) {
        float nx[8];
        load8_const(nx, a, g + gstep < ng ? (g + gstep) * kDqGroup + 8 * lane : nb, nb);
        dq_quantize_group(e, g * kDqGroup + 8 * lane, nb, mu, e4m3, lane, g, qabs, scale);
#pragma unroll
        for (int u = 0; u < 8; ++u) e[u] = nx[u];
    }
}

__global__ void __launch_bounds__(kDqThreads) dq_quant_kernel(const float *__restrict__ a, int64_t nb,
                                                              int8_t *__restrict__ qabs, float *__restrict__ scale,
                                                              const float *__restrict__ mu_in,
                                                              float *__restrict__ mu_out, unsigned char *scratch,
                                                              bool e4m3) {
    __shared__ float mu_s;
    pdl_wait();
    pdl_trigger();
    dq_quant_part(a, nb, qabs, scale, mu_in, mu_out, scratch, e4m3, blockIdx.x, gridDim.x, &mu_s);
}

// K3's grid: one group per warp up to the CTAs the device holds at once (a
// few per SM), then more groups per warp.
static int64_t dq_quant_grid(int64_t nb, int num_sms) {
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    int64_t grid = (ng + kDqGroupsPerCta - 1) / kDqGroupsPerCta;
    if (grid > 4LL * num_sms) grid = 4LL * num_sms;
    return grid < 1 ? 1 : grid;
}

// ===========================================================================
// Single-launch double quantization (the workspace entry point, when the grid
// fits on the device): CTA c owns P groups per warp, keeps them in registers,
// adds them into the call's bank of limbs, and waits on a grid-wide barrier
// (bounded by kDqfWaitNs) until every CTA has: the last to arrive advances the
// generation, which the others poll.  Then each CTA reads the limbs, forms mu
// itself (every CTA gets the same value) and quantizes its groups.  The launch
// is cooperative, so every CTA is resident whatever else runs on the device.
// ===========================================================================
template <int P>
__global__ void __launch_bounds__(kDqThreads, P == 1 ? 6 : 4) dq_fused_kernel(const float *__restrict__ a, int64_t nb,
                                                              int8_t *__restrict__ qabs, float *__restrict__ scale,
                                                              float *__restrict__ mu_out, unsigned char *ws, int G,
                                                              bool e4m3) {
    __shared__ unsigned long long slim[kXLimbs];
    __shared__ float mu_s;
    __shared__ int ok_s;
    __shared__ unsigned gen_s;
    if (threadIdx.x < kXLimbs) slim[threadIdx.x] = 0ull;
    __syncthreads();
    pdl_wait();  // the constants come from the previous kernel (the quantize)
    pdl_trigger();
    const DqScratch sc = dq_scratch(ws, true);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    if (blockIdx.x == 0 && threadIdx.x == 0) *sc.status = QLN_OK;
    const unsigned g0 = dq_read_gen(sc, &gen_s);
    unsigned long long *bank = sc.bank[g0 & 1];

    // groups c*8P + warp + 8p, p < P: all P loads in flight at once
    float e[P][8];
#pragma unroll
    for (int q = 0; q < P; ++q) {
        const int64_t g = ((int64_t)blockIdx.x * P + q) * kDqGroupsPerCta + warp;
        load8_const(e[q], a, g < ng ? g * kDqGroup + 8 * lane : nb, nb);
    }
    dq_add_cta<P>(e, slim, bank);
    __syncthreads();
    if (threadIdx.x == 0) {  // the grid barrier: the generation moves on when the last CTA arrives
        bool ok = dq_arrive(sc, g0, G) || dqf_ld_acquire_u32(sc.gen) != g0;
        if (!ok) {
            const uint64_t t0 = dqf_timer_ns();
            for (uint32_t it = 0; !ok; ++it) {
                ok = dqf_ld_acquire_u32(sc.gen) != g0;
                if (!ok && (it & 63u) == 63u && dqf_timer_ns() - t0 > kDqfWaitNs) break;
            }
        }
        if (!ok) atomicExch(sc.status, (int)QLN_ERR_TIMEOUT);
        ok_s = ok;
    }
    __syncthreads();
    const bool ok = ok_s != 0;
    if (ok && warp == 0) {
        const float mu = xsum_mean_warp(bank, (uint32_t)nb);
        if (lane == 0) {
            mu_s = mu;
            if (blockIdx.x == 0) *mu_out = mu;
        }
    }
    __syncthreads();
    if (ok) {
#pragma unroll
        for (int q = 0; q < P; ++q) {
            const int64_t g = ((int64_t)blockIdx.x * P + q) * kDqGroupsPerCta + warp;
            if (g < ng) dq_quantize_group(e[q], g * kDqGroup + 8 * lane, nb, mu_s, e4m3, lane, g, qabs, scale);
        }
    }
}

size_t dq_workspace_bytes(int64_t nb) {
    (void)nb;
    return kDqScratchBytes;
}

// CTAs of the fused kernel (P groups per warp) that a cooperative launch can
// hold; the per-SM figure is cached (one device type per process).
template <int P>
static int dq_fused_capacity(int num_sms) {
    static std::atomic<int> cached{0};
    int per_sm = cached.load(std::memory_order_relaxed);
    if (per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dq_fused_kernel<P>, kDqThreads, 0) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        cached.store(per_sm, std::memory_order_relaxed);
    }
    return per_sm * num_sms;
}

template <int P>
static cudaError_t launch_dq_fused(const float *absmax, int64_t nb, int8_t *qabs, float *scale, float *mu, void *ws,
                                   bool e4m3, cudaStream_t st, int G) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)G);
    cfg.blockDim = dim3(kDqThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    // A driver that refuses a cooperative launch with programmatic serialization
    // gets a plain cooperative launch (remembered per process).
    static std::atomic<int> pdl_refused{0};
    cfg.numAttrs = pdl_refused.load(std::memory_order_relaxed) ? 1 : 2;
    note_launch();
    unsigned char *w = static_cast<unsigned char *>(ws);
    cudaError_t err = cudaLaunchKernelEx(&cfg, dq_fused_kernel<P>, absmax, nb, qabs, scale, mu, w, G, e4m3);
    if (err != cudaSuccess && cfg.numAttrs == 2) {
        cudaGetLastError();
        pdl_refused.store(1, std::memory_order_relaxed);
        cfg.numAttrs = 1;
        err = cudaLaunchKernelEx(&cfg, dq_fused_kernel<P>, absmax, nb, qabs, scale, mu, w, G, e4m3);
    }
    return err;
}

// The fused kernel, launched cooperatively (every CTA resident) and as a
// programmatic dependent, with the fewest groups per warp (1, 2 or 4) whose
// grid fits on the device; false when even 4 do not fit.
static bool try_dq_fused(const float *absmax, int64_t nb, int8_t *qabs, float *scale, float *mu, void *ws, bool e4m3,
                         cudaStream_t st, int num_sms, cudaError_t *err) {
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    auto grid = [&](int P) { return (ng + (int64_t)P * kDqGroupsPerCta - 1) / ((int64_t)P * kDqGroupsPerCta); };
    if (grid(1) <= dq_fused_capacity<1>(num_sms)) {
        *err = launch_dq_fused<1>(absmax, nb, qabs, scale, mu, ws, e4m3, st, (int)grid(1));
    } else if (grid(2) <= dq_fused_capacity<2>(num_sms)) {
        *err = launch_dq_fused<2>(absmax, nb, qabs, scale, mu, ws, e4m3, st, (int)grid(2));
    } else if (grid(4) <= dq_fused_capacity<4>(num_sms)) {
        *err = launch_dq_fused<4>(absmax, nb, qabs, scale, mu, ws, e4m3, st, (int)grid(4));
    } else {
        return false;
    }
    return true;
}

int64_t dq_max_blocks() { return kMeanMaxBlocks; }

// K2 then K3 (mu from the limbs), each launched as a programmatic dependent of
// the kernel before it.
static cudaError_t launch_dq_pair(const float *absmax, int64_t nb, unsigned char *scratch, bool with_status,
                                  int8_t *qabs, float *scale, float *mu, bool e4m3, cudaStream_t st, int num_sms) {
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    int64_t g2 = (ng + kDqGroupsPerCta - 1) / kDqGroupsPerCta;
    if (g2 > 4LL * num_sms) g2 = 4LL * num_sms;  // a few passes per CTA for very large weights
    cudaError_t e = launch_pdl(dq_sum_kernel, dim3((unsigned)g2), dim3(kDqThreads), 0, st, absmax, nb, scratch,
                               with_status);
    if (e != cudaSuccess) return e;
    return launch_pdl(dq_quant_kernel, dim3((unsigned)dq_quant_grid(nb, num_sms)), dim3(kDqThreads), 0, st, absmax,
                      nb, qabs, scale, (const float *)nullptr, mu, scratch, e4m3);
}

cudaError_t launch_nf4_double_quant(const float *absmax, int64_t nb, int8_t *qabs, float *scale, float *mu,
                                    void *ws, bool e4m3, cudaStream_t st, int num_sms) {
    cudaError_t e = cudaSuccess;
    if (try_dq_fused(absmax, nb, qabs, scale, mu, ws, e4m3, st, num_sms, &e)) return e;
    return launch_dq_pair(absmax, nb, static_cast<unsigned char *>(ws), true, qabs, scale, mu, e4m3, st, num_sms);
}

// The quantize, then the double quantization of its block constants (the
// single cooperative launch where it fits), each a programmatic dependent of
// the kernel before it: the combined entry point computes exactly what the two
// entry points compute.
cudaError_t launch_nf4_quantize_dq(const void *W, int dtype, int64_t numel, uint8_t *codes, float *absmax,
                                   int8_t *qabs, float *scale, float *mu, void *ws, bool e4m3, cudaStream_t st,
                                   int num_sms) {
    cudaError_t e = launch_nf4_quantize(W, dtype, numel, codes, absmax, st, num_sms);
    if (e != cudaSuccess) return e;
    return launch_nf4_double_quant(absmax, (numel + 63) / 64, qabs, scale, mu, ws, e4m3, st, num_sms);
}

static_assert(kDqScratchBytes == kDqBatchScratchBytes, "one DQ scratch per batch job");

namespace {
struct ByteRange {
    uintptr_t lo, hi;  // [lo, hi)
    int job;           // -1: the workspace
    bool write;
};

// True when no range written by one job (or the workspace) overlaps any range
// of another job: then the quantize kernels of different weights and the
// deferred double quantization may run at the same time.
bool batch_disjoint(const QuantJob *jobs, int njobs, const void *ws) {
    std::vector<ByteRange> r;
    r.reserve((size_t)njobs * 6 + 1);
    auto add = [&](const void *p, size_t n, int job, bool write) {
        if (n) r.push_back({(uintptr_t)p, (uintptr_t)p + n, job, write});
    };
    for (int i = 0; i < njobs; ++i) {
        const QuantJob &q = jobs[i];
        const size_t nb = (size_t)((q.numel + 63) / 64);
        add(q.W, (size_t)q.numel * (q.dtype == QLN_DTYPE_F32 ? 4 : 2), i, false);
        add(q.codes, (size_t)((q.numel + 1) / 2), i, true);
        add(q.absmax, nb * 4, i, true);
        add(q.qabs, nb, i, true);
        add(q.scale, ((nb + kDqGroup - 1) / kDqGroup) * 4, i, true);
        add(q.mu, 4, i, true);
    }
    add(ws, kDqScratchBytes * (size_t)njobs, -1, true);
    std::sort(r.begin(), r.end(), [](const ByteRange &a, const ByteRange &b) { return a.lo < b.lo; });
    // sweep: every range against the earlier ranges still open
    std::vector<size_t> open;
    for (size_t k = 0; k < r.size(); ++k) {
        size_t keep = 0;
        for (size_t t = 0; t < open.size(); ++t) {
            const ByteRange &o = r[open[t]];
            if (o.hi <= r[k].lo) continue;  // closed
            open[keep++] = open[t];
            if (o.job != r[k].job && (o.write || r[k].write)) return false;
        }
        open.resize(keep);
        open.push_back(k);
    }
    return true;
}
}  // namespace

// The double quantization of a disjoint batch after its last quantize: one
// launch sums the constants of up to kTailJobs weights, a second quantizes
// their groups.  A job's CTAs are a contiguous range of the launch (job j owns
// CTAs cta0[j] .. cta0[j+1]-1) and run the single-weight code with that range
// as their grid, so the exact sums and groups are those of separate calls.
// The job table travels as the kernel's parameter (about 7 KB).
constexpr int kTailJobs = 128;
constexpr int kTailPasses = 4;  // groups per warp and CTA, at most
struct DqTailJob {
    const float *absmax;
    int64_t nb;
    unsigned char *ws;
    int8_t *qabs;
    float *scale;
    float *mu;
    int e4m3;
    int cta0;  // first CTA of the job
};
struct DqTail {
    int njobs;
    int status;  // job 0's CTA 0 writes QLN_OK to its scratch status word
    DqTailJob job[kTailJobs];
};

// The job whose CTA range holds CTA b, and the CTA's place in that range.
__device__ __forceinline__ int dq_tail_job(const DqTail &t, int b, int64_t *bid, int64_t *nblk) {
    int lo = 0, hi = t.njobs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (t.job[mid].cta0 <= b) lo = mid;
        else hi = mid - 1;
    }
    *bid = b - t.job[lo].cta0;
    *nblk = (lo + 1 < t.njobs ? t.job[lo + 1].cta0 : (int)gridDim.x) - t.job[lo].cta0;
    return lo;
}

__global__ void __launch_bounds__(kDqThreads) dq_sum_tail_kernel(const __grid_constant__ DqTail t) {
    __shared__ unsigned long long slim[kXLimbs];
    __shared__ unsigned gen_s;
    if (threadIdx.x < kXLimbs) slim[threadIdx.x] = 0ull;
    __syncthreads();
    pdl_wait();  // the constants come from earlier kernels
    pdl_trigger();
    int64_t bid, nblk;
    const int j = dq_tail_job(t, blockIdx.x, &bid, &nblk);
    const DqTailJob &J = t.job[j];
    dq_sum_part(J.absmax, J.nb, J.ws, t.status && j == 0, bid, nblk, slim, &gen_s);
}

__global__ void __launch_bounds__(kDqThreads) dq_quant_tail_kernel(const __grid_constant__ DqTail t) {
    __shared__ float mu_s;
    pdl_wait();  // the sums of the earlier launch
    pdl_trigger();
    int64_t bid, nblk;
    const int j = dq_tail_job(t, blockIdx.x, &bid, &nblk);
    const DqTailJob &J = t.job[j];
    dq_quant_part(J.absmax, J.nb, J.qabs, J.scale, nullptr, J.mu, J.ws, J.e4m3 != 0, bid, nblk, &mu_s);
}

// Sum launches for every kTailJobs jobs, then the group launches.
static cudaError_t launch_dq_tails(const QuantJob *jobs, int njobs, unsigned char *ws, cudaStream_t st) {
    static_assert(sizeof(DqTail) <= 8192, "the job table stays a small kernel parameter");
    for (int pass = 0; pass < 2; ++pass) {
        for (int j0 = 0; j0 < njobs; j0 += kTailJobs) {
            DqTail t{};
            t.njobs = njobs - j0 < kTailJobs ? njobs - j0 : kTailJobs;
            t.status = (j0 == 0) ? 1 : 0;
            int64_t ctas = 0;
            for (int k = 0; k < t.njobs; ++k) {
                const QuantJob &q = jobs[j0 + k];
                DqTailJob &J = t.job[k];
                J.absmax = q.absmax;
                J.nb = (q.numel + 63) / 64;
                J.ws = ws + kDqScratchBytes * (size_t)(j0 + k);
                J.qabs = q.qabs;
                J.scale = q.scale;
                J.mu = q.mu;
                J.e4m3 = q.e4m3 ? 1 : 0;
                J.cta0 = (int)ctas;
                const int64_t ng = (J.nb + kDqGroup - 1) / kDqGroup;
                ctas += (ng + kDqGroupsPerCta * kTailPasses - 1) / (kDqGroupsPerCta * kTailPasses);
            }
            const cudaError_t e = pass == 0
                                      ? launch_pdl(dq_sum_tail_kernel, dim3((unsigned)ctas), dim3(kDqThreads), 0, st, t)
                                      : launch_pdl(dq_quant_tail_kernel, dim3((unsigned)ctas), dim3(kDqThreads), 0, st, t);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

// Batch with disjoint buffers: the quantize kernels back to back (from the
// second on they start early, see kLateWait), then the tail launches of
// launch_dq_tails.  The first tail launch waits for the last quantize, whose
// completion implies that of every earlier one.  Phase kernels running beside
// the quantize kernels instead took the 6.48 B-parameter sweep from 5.35 ms
// to 6.6 ms: their work, on one small CTA per SM, ran longer than the
// quantize of the smaller weights it had to finish within.
// Otherwise (a job reads or writes another job's outputs) each job's
// quantize is followed by its own sum and group launches, every launch
// waiting at its start for the one before it: the order of separate calls.
// Job i's scratch is ws + 256 i; job 0's sum launch writes QLN_OK to the
// status word at ws + 0.
cudaError_t launch_nf4_quantize_dq_batch(const QuantJob *jobs, int njobs, void *ws, cudaStream_t st, int num_sms) {
    unsigned char *w = static_cast<unsigned char *>(ws);
    cudaError_t e = cudaSuccess;
    if (batch_disjoint(jobs, njobs, ws)) {  // the quantize chain alone, then the double quantization of all jobs
        for (int i = 0; i < njobs && e == cudaSuccess; ++i) {
            const QuantJob &q = jobs[i];
            e = i == 0 ? launch_quantize_dtype<false>(q.W, q.dtype, q.numel, q.codes, q.absmax, st, num_sms)
                       : launch_quantize_dtype<true>(q.W, q.dtype, q.numel, q.codes, q.absmax, st, num_sms);
        }
        return e == cudaSuccess ? launch_dq_tails(jobs, njobs, w, st) : e;
    }
    for (int i = 0; i < njobs && e == cudaSuccess; ++i) {  // job by job, as separate calls in order
        const QuantJob &q = jobs[i];
        e = launch_quantize_dtype<false>(q.W, q.dtype, q.numel, q.codes, q.absmax, st, num_sms);
        if (e == cudaSuccess) e = launch_dq_tails(&q, 1, w + kDqScratchBytes * (size_t)i, st);
    }
    return e;
}

// ===========================================================================
// Allocation-free double quantization.  The only scratch the two-kernel path
// needs is the generation word, the arrival counter and the banks of limbs;
// this variant keeps them in a fixed, file-scope device array instead of a
// caller workspace, so a caller that cannot allocate device memory can still
// run the path.  The array is kDqScratchBytes (256 bytes); every GPU that loads
// the library holds it until the process exits.  Each call leaves the bank the
// next call sums into zeroed, so nothing has to be cleared between calls; two
// calls that overlap on the GPU (different streams, no ordering) share the
// array and race.  There is no status word (no workspace to hold it).
// ===========================================================================
static __device__ __align__(256) unsigned char g_dq_static_scratch[kDqScratchBytes];

int64_t dq_static_max_blocks() { return kMeanMaxBlocks; }

// Device address of the array for the current device and context.  In host
// code the symbol names a host-side stand-in, so the address is looked up
// (with the device current) and cached per device together with the context
// it was looked up in: a context torn down and made again may load the module
// elsewhere, so a new context means a new lookup.
struct DqStaticSlot {
    std::mutex mu;
    void *ctx = nullptr;
    unsigned char *ptr = nullptr;
};
static DqStaticSlot g_dq_static_slot[64];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
static CtxGetCurrentFn ctx_get_current_fn() {
    static std::atomic<CtxGetCurrentFn> fn{nullptr};
    CtxGetCurrentFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<CtxGetCurrentFn>(p);
            fn.store(f, std::memory_order_release);
        }
    }
    return f;
}

static cudaError_t dq_static_scratch(unsigned char **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    CtxGetCurrentFn getctx = ctx_get_current_fn();
    if (!getctx) return cudaErrorDeviceUninitialized;
    CUcontext ctx = nullptr;
    if (getctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    DqStaticSlot &slot = g_dq_static_slot[dev];
    std::lock_guard<std::mutex> lock(slot.mu);
    if (slot.ptr == nullptr || ctx == nullptr || slot.ctx != (void *)ctx) {
        void *addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_dq_static_scratch);  // makes the device's context current if needed
        if (e != cudaSuccess) return e;
        if (getctx(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
        slot.ptr = static_cast<unsigned char *>(addr);
        slot.ctx = (void *)ctx;
    }
    *out = slot.ptr;
    return cudaSuccess;
}

cudaError_t launch_nf4_double_quant_static(const float *absmax, int64_t nb, int8_t *qabs, float *scale, float *mu,
                                           cudaStream_t st, int num_sms) {
    unsigned char *scratch = nullptr;
    cudaError_t e = dq_static_scratch(&scratch);
    if (e != cudaSuccess) return e;
    return launch_dq_pair(absmax, nb, scratch, false, qabs, scale, mu, false, st, num_sms);
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
