// Shared device helpers of libqlora_nf4 (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qlora_nf4.h"

namespace qln {

// ---------------------------------------------------------------------------
// The NF4 book: 16 fp32 values, ascending, exact zero at index 7, ends +-1.
// Built (offline, in binary64, then rounded once to binary32) from normal
// quantiles with separate negative and positive halves sharing one zero,
// normalized by the largest quantile: deck "3 QLoRA Finetuning" cards 2-3,
// "LoRA 与 QLoRA" section QLoRA 1 (归一化与匹配).  Positive half: Q_Z at 8 of 9
// probabilities evenly spaced from delta to 1/2; negative half: -Q_Z at 7 of 8;
// delta = 1 - (1/32 + 1/30)/2.  Matches the 4-decimal table printed in the
// jjjymmm.cn post ("4-bit NormalFloat(NF4)").  Stored as bit patterns so the
// values are exact; a CPU test compares them with an independent recomputation.
// ---------------------------------------------------------------------------
__host__ __device__ constexpr uint32_t nf4_bits(int q) {
    return q == 0    ? 0xbf800000u
           : q == 1  ? 0xbf3239b1u
           : q == 2  ? 0xbf066b2eu
           : q == 3  ? 0xbeca329eu
           : q == 4  ? 0xbe91a24bu
           : q == 5  ? 0xbe3d353du
           : q == 6  ? 0xbdba7869u
           : q == 7  ? 0x00000000u
           : q == 8  ? 0x3da2fb01u
           : q == 9  ? 0x3e24cadfu
           : q == 10 ? 0x3e7c04dau
           : q == 11 ? 0x3ead0336u
           : q == 12 ? 0x3ee1a4b5u
           : q == 13 ? 0x3f1007a9u
           : q == 14 ? 0x3f3913b0u
                     : 0x3f800000u;
}

constexpr int kBlock = 64;     // weights per absmax block
constexpr int kDqGroup = 256;  // block constants per DQ scale

__device__ __forceinline__ float nf4_value(int q) { return __uint_as_float(nf4_bits(q)); }

// Snap thresholds: t_k = the largest fp32 value <= (c_k + c_{k+1}) / 2.
// For an fp32 x, x > t_k  <=>  x is strictly closer to c_{k+1} than to c_k,
// so  q = #{k : x > t_k}  is the nearest book entry with ties to the lower
// code.  Halving is exact; __fadd_rd rounds the exact sum toward -inf.
__device__ __forceinline__ float nf4_threshold(int k) {
    return __fadd_rd(0.5f * nf4_value(k), 0.5f * nf4_value(k + 1));
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched with the programmatic
// stream-serialization attribute may start while the previous kernel on the
// stream is still running; pdl_wait() blocks until that kernel has completed
// and its memory operations are visible, so every such kernel calls it before
// its first access to global memory that another kernel reads or writes.
// pdl_trigger() lets the next kernel on the stream be launched (it still
// waits in its own pdl_wait()).  Both are no-ops without the attribute.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ---------------------------------------------------------------------------
// Small conversions.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    // lo -> bits [0,16) (the lower address), hi -> bits [16,32); both RN.
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// The value of an OCP FP8 E4M3 code (exact in fp32): the hardware conversion
// to half, then to float.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)(code & 0xffu), __NV_E4M3);
    return __half2float(__half(h));
}

// doubleDequant of one block constant: ahat = fp32(mu + fp32(b * rhat)), the
// product first, then the sum ("LoRA 与 QLoRA" section 2, reconstruction).
// The low byte of `code` is rhat: an int8 (QLN_DQ_INT8) or an E4M3 code
// (QLN_DQ_E4M3, the "8-bit floats" of deck card 4).
__device__ __forceinline__ float dq_restore(uint32_t code, float b, float mu, bool e4m3) {
    const float r = e4m3 ? e4m3_to_f32(code) : (float)(int8_t)(code & 0xffu);
    return __fadd_rn(mu, __fmul_rn(b, r));
}

// ---------------------------------------------------------------------------
// PTX wrappers: cp.async, ldmatrix, legacy mma.sync (used by the skinny,
// HBM-bound kernels and the small-n path).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
// Zero-filling form: copies src_bytes (0 or 16) and fills the rest with 0.
__device__ __forceinline__ void cp_async16_zfill(void *smem, const void *gmem, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)), "l"(gmem),
                 "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                            const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                                  const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t &r0, uint32_t &r1, const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
                 : "=r"(r0), "=r"(r1)
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t &r0, uint32_t &r1, const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
                 : "=r"(r0), "=r"(r1)
                 : "r"(smem_u32(p)));
}

// D[16x8] += A[16x16] (row) * B[16x8] (col), bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__host__ __device__ constexpr int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

}  // namespace qln

namespace qln {

// ---------------------------------------------------------------------------
// Register-only NF4 decode.  For one block constant ahat the 16 products
// P[q] = bf16_RN(fp32(ahat * c[q])) are formed once and split into a table of
// low bytes L[0..3] and high bytes H[0..3] (4 entries per register); a byte
// permute (prmt) then looks up 4 codes at a time: the low 3 bits of each code
// pick a byte within an 8-entry half-table, bit 3 picks the half.  Exactly the
// doubleDequant value w' = bf16_RN(fp32(ahat * c[q])), with no shared-memory
// traffic.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

struct NF4Table {
    uint32_t L[4], H[4];
};

__device__ __forceinline__ NF4Table nf4_table(float ah) {
    uint32_t T[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) T[i] = pack_bf16x2(__fmul_rn(ah, nf4_value(2 * i)), __fmul_rn(ah, nf4_value(2 * i + 1)));
    NF4Table t;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        t.L[j] = prmt(T[2 * j], T[2 * j + 1], 0x6420u);  // low bytes of P[4j..4j+3]
        t.H[j] = prmt(T[2 * j], T[2 * j + 1], 0x7531u);  // high bytes
    }
    return t;
}

// Four codes held in the low 16 bits of s (nibble order: element 1, 0, 3, 2 of
// the two bytes) -> BF16 pairs (elements 0,1) and (2,3).
__device__ __forceinline__ void nf4_decode4(uint32_t s, const NF4Table &t, uint32_t &e01, uint32_t &e23) {
    const uint32_t i3 = s & 0x7777u;
    const uint32_t sel = ((s >> 1) & 0x4444u) | 0x3210u;
    const uint32_t lo = prmt(prmt(t.L[0], t.L[1], i3), prmt(t.L[2], t.L[3], i3), sel);
    const uint32_t hi = prmt(prmt(t.H[0], t.H[1], i3), prmt(t.H[2], t.H[3], i3), sel);
    e01 = prmt(lo, hi, 0x4051u);
    e23 = prmt(lo, hi, 0x6273u);
}

// One 32-bit word of packed codes (8 weights, first in the high nibble of the
// lowest byte) -> 8 BF16 values in memory order.  The selectors of both
// 16-bit halves come from one mask and one shifted mask of the whole word
// (prmt reads only the low 16 bits of its selector).
__device__ __forceinline__ uint4 nf4_decode8(uint32_t w, const NF4Table &t) {
    const uint32_t i3 = w & 0x77777777u;                           // code & 7, all 8 codes
    const uint32_t sel = ((w >> 1) & 0x44444444u) | 0x32103210u;   // byte j of x0 or of x1 by bit 3
    const uint32_t i3h = i3 >> 16, selh = sel >> 16;
    uint4 o;
    {
        const uint32_t lo = prmt(prmt(t.L[0], t.L[1], i3), prmt(t.L[2], t.L[3], i3), sel);
        const uint32_t hi = prmt(prmt(t.H[0], t.H[1], i3), prmt(t.H[2], t.H[3], i3), sel);
        o.x = prmt(lo, hi, 0x4051u);
        o.y = prmt(lo, hi, 0x6273u);
    }
    {
        const uint32_t lo = prmt(prmt(t.L[0], t.L[1], i3h), prmt(t.L[2], t.L[3], i3h), selh);
        const uint32_t hi = prmt(prmt(t.H[0], t.H[1], i3h), prmt(t.H[2], t.H[3], i3h), selh);
        o.z = prmt(lo, hi, 0x4051u);
        o.w = prmt(lo, hi, 0x6273u);
    }
    return o;
}

}  // namespace qln
