// NF4 codec kernels: blockwise quantize (K1), double quantization (K2 + K3),
// doubleDequant to BF16 (K4).  All HBM-bound streaming kernels.
//
// Method: jjjymmm.cn 2024/03 QLoRA post, "4-bit NormalFloat(NF4)" (divide by
// the block ABSMAX, snap to the nearest book entry; dequantize = book value),
// "Double Quantization" and "QLoRA" (doubleDequant: constants first);
// "LoRA 与 QLoRA" section QLoRA 2 (a_j = max|W_j| per 64 weights,
// r_j = (a_j - mu)/b, 8-bit rhat_j, ahat_j = mu + b rhat_j).
#include <atomic>

#include "qln_common.cuh"
#include "qln_internal.h"

namespace qln {

// ===========================================================================
// K1: quantize.  One warp streams 256 consecutive weights (4 blocks) per step:
// lane l holds float4 #l and #(l+32), i.e. elements 4l..4l+3 of block l/16 and
// of block 2 + l/16.  Each 16-lane half reduces its block's absmax with four
// xor-shuffles and every element is divided by it (IEEE fp32 division, x in
// [-1, 1]).
// Snap without a 15-way compare: the top 12 bits of x (sign, exponent, three
// mantissa bits) name an interval of fp32 values that contains at most one
// snap threshold (the narrowest gap between thresholds, 0.08, is wider than
// any such interval below 1 in magnitude).  A per-CTA table gives, for each
// key, the code of the interval's smallest value and that one threshold (or
// +inf), so  q = base[key] + (x > thr[key])  -- exactly #{k : x > t_k}.
// ===========================================================================
constexpr int kSnapKeys = 4096;

__device__ __forceinline__ uint32_t snap_lut(float x, const uint2 *lut) {
    const uint2 e = lut[__float_as_uint(x) >> 20];
    return e.y + ((x > __uint_as_float(e.x)) ? 1u : 0u);
}

__device__ void build_snap_lut(uint2 *lut) {
    float t[15];
#pragma unroll
    for (int k = 0; k < 15; ++k) t[k] = nf4_threshold(k);
    for (int key = threadIdx.x; key < kSnapKeys; key += blockDim.x) {
        const float a = __uint_as_float((uint32_t)key << 20);
        const float b = __uint_as_float(((uint32_t)key << 20) | 0xFFFFFu);
        const bool neg = (key & 0x800) != 0;
        const float lo = neg ? b : a, hi = neg ? a : b;  // the interval [lo, hi] in value order
        uint32_t base = 0, thr = 0x7f800000u;            // +inf: no threshold inside
#pragma unroll
        for (int k = 0; k < 15; ++k) {
            if (lo > t[k]) ++base;
            else if (t[k] < hi && thr == 0x7f800000u) thr = __float_as_uint(t[k]);
        }
        lut[key] = make_uint2(thr, base);
    }
}

__device__ __forceinline__ uint32_t snap_pair(float w0, float w1, float a, const uint2 *lut) {
    float x0 = 0.f, x1 = 0.f;
    if (a > 0.f) {
        x0 = __fdiv_rn(w0, a);
        x1 = __fdiv_rn(w1, a);
    }
    return (snap_lut(x0, lut) << 4) | snap_lut(x1, lut);  // first element in the high nibble
}

__device__ __forceinline__ float absmax4(float4 v) {
    return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

__global__ void __launch_bounds__(256) nf4_quantize_kernel(const float4 *__restrict__ W, int64_t nb,
                                                           uint16_t *__restrict__ codes16,
                                                           float *__restrict__ absmax) {
    __shared__ uint2 lut[kSnapKeys];
    build_snap_lut(lut);
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t nchunks = (nb + 3) / 4;  // 4 blocks (256 weights) per chunk

    for (int64_t c = warp; c < nchunks; c += nwarps) {
        const int64_t b0 = 4 * c + (lane >> 4);  // block of v0
        const int64_t b1 = b0 + 2;               // block of v1
        float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
        if (b0 < nb) v0 = __ldcs(W + 64 * c + lane);
        if (b1 < nb) v1 = __ldcs(W + 64 * c + 32 + lane);
        float m0 = absmax4(v0), m1 = absmax4(v1);
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) {
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
        }
        if (b0 < nb) {
            uint32_t p = snap_pair(v0.x, v0.y, m0, lut) | (snap_pair(v0.z, v0.w, m0, lut) << 8);
            __stcs(codes16 + 64 * c + lane, (uint16_t)p);
            if ((lane & 15) == 0) absmax[b0] = m0;
        }
        if (b1 < nb) {
            uint32_t p = snap_pair(v1.x, v1.y, m1, lut) | (snap_pair(v1.z, v1.w, m1, lut) << 8);
            __stcs(codes16 + 64 * c + 32 + lane, (uint16_t)p);
            if ((lane & 15) == 0) absmax[b1] = m1;
        }
    }
}

cudaError_t launch_nf4_quantize(const float *W, int64_t numel, uint8_t *codes, float *absmax,
                                cudaStream_t st, int num_sms) {
    const int64_t nb = numel / kBlock;
    const int64_t nchunks = (nb + 3) / 4;
    const int threads = 256;
    int64_t grid = (nchunks + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 4;  // persistent-ish: the table is built once per CTA
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    nf4_quantize_kernel<<<(unsigned)grid, threads, 0, st>>>(reinterpret_cast<const float4 *>(W), nb,
                                                            reinterpret_cast<uint16_t *>(codes), absmax);
    note_launch();
    return cudaGetLastError();
}

// ===========================================================================
// K2: partial sums for mu.  CTA c sums a[8192c, 8192(c+1)) as a perfect binary
// tree in binary64 (zero-padded): each thread folds its 32 consecutive leaves
// pairwise, a warp xor-butterfly adds lane pairs level by level (addition is
// commutative, so both lanes of a pair hold the same node), and the 8 warp
// roots are folded pairwise.  The result is exactly the aligned subtree of
// the whole-tensor tree.
// ===========================================================================
constexpr int kMeanLeavesPerThread = 32;
constexpr int kMeanThreads = 256;
constexpr int kMeanChunk = kMeanLeavesPerThread * kMeanThreads;  // 8192

__global__ void __launch_bounds__(kMeanThreads) dq_partial_kernel(const float *__restrict__ a, int64_t nb,
                                                                  double *__restrict__ partial) {
    __shared__ double warp_root[kMeanThreads / 32];
    const int64_t base = (int64_t)blockIdx.x * kMeanChunk + (int64_t)threadIdx.x * kMeanLeavesPerThread;
    double v[kMeanLeavesPerThread];
    if (base + kMeanLeavesPerThread <= nb) {
        const float4 *p = reinterpret_cast<const float4 *>(a + base);
#pragma unroll
        for (int i = 0; i < kMeanLeavesPerThread / 4; ++i) {
            float4 f = __ldg(p + i);
            v[4 * i + 0] = (double)f.x;
            v[4 * i + 1] = (double)f.y;
            v[4 * i + 2] = (double)f.z;
            v[4 * i + 3] = (double)f.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < kMeanLeavesPerThread; ++i) v[i] = (base + i < nb) ? (double)a[base + i] : 0.0;
    }
#pragma unroll
    for (int len = kMeanLeavesPerThread; len > 1; len >>= 1) {
#pragma unroll
        for (int i = 0; i < len / 2; ++i) v[i] = __dadd_rn(v[2 * i], v[2 * i + 1]);
    }
    double s = v[0];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) s = __dadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
    if ((threadIdx.x & 31) == 0) warp_root[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double w[kMeanThreads / 32];
#pragma unroll
        for (int i = 0; i < kMeanThreads / 32; ++i) w[i] = warp_root[i];
#pragma unroll
        for (int len = kMeanThreads / 32; len > 1; len >>= 1) {
#pragma unroll
            for (int i = 0; i < len / 2; ++i) w[i] = __dadd_rn(w[2 * i], w[2 * i + 1]);
        }
        partial[blockIdx.x] = w[0];
    }
}

// ===========================================================================
// K3: every CTA first folds the K2 partials (zero-padded to a power of two)
// into S and mu = fp32(S / nb) -- cheap, and it saves a launch -- then each
// warp quantizes one group of 256 constants: d = fp32(a - mu),
// b = fp32(max|d| / 127), rhat = clamp(rint(fp32(d / b)), -127, 127).
// ===========================================================================
constexpr int kDqThreads = 256;
constexpr int kMaxPartials = 4096;  // nb <= 4096 * 8192 = 2^25 blocks

__global__ void __launch_bounds__(kDqThreads) dq_quant_kernel(const float *__restrict__ a, int64_t nb,
                                                              const double *__restrict__ partial, int np,
                                                              int np_pow2, int8_t *__restrict__ qabs,
                                                              float *__restrict__ scale, float *__restrict__ mu_out) {
    __shared__ double tree[kMaxPartials];
    __shared__ float mu_s;
    for (int i = threadIdx.x; i < np_pow2; i += blockDim.x) tree[i] = (i < np) ? partial[i] : 0.0;
    __syncthreads();
    for (int len = np_pow2; len > 1; len >>= 1) {
        double v[kMaxPartials / kDqThreads / 2 > 0 ? kMaxPartials / kDqThreads / 2 : 1];
        const int half = len >> 1;
        int cnt = 0;
        for (int i = threadIdx.x; i < half; i += blockDim.x) v[cnt++] = __dadd_rn(tree[2 * i], tree[2 * i + 1]);
        __syncthreads();
        cnt = 0;
        for (int i = threadIdx.x; i < half; i += blockDim.x) tree[i] = v[cnt++];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        float mu = __double2float_rn(__ddiv_rn(tree[0], (double)nb));
        mu_s = mu;
        if (blockIdx.x == 0) *mu_out = mu;
    }
    __syncthreads();
    const float mu = mu_s;

    const int lane = threadIdx.x & 31;
    const int64_t g = (int64_t)blockIdx.x * (kDqThreads / 32) + (threadIdx.x >> 5);
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    if (g >= ng) return;
    const int64_t j0 = g * kDqGroup + 4 * lane;        // first of 4 constants of v0
    const int64_t j1 = j0 + 128;                       // first of 4 constants of v1
    float e0[4], e1[4];
    bool ok0[4], ok1[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        ok0[i] = (j0 + i) < nb;
        ok1[i] = (j1 + i) < nb;
    }
    if (j0 + 4 <= nb) {
        float4 f = __ldg(reinterpret_cast<const float4 *>(a + j0));
        e0[0] = f.x; e0[1] = f.y; e0[2] = f.z; e0[3] = f.w;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) e0[i] = ok0[i] ? a[j0 + i] : 0.f;
    }
    if (j1 + 4 <= nb) {
        float4 f = __ldg(reinterpret_cast<const float4 *>(a + j1));
        e1[0] = f.x; e1[1] = f.y; e1[2] = f.z; e1[3] = f.w;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) e1[i] = ok1[i] ? a[j1 + i] : 0.f;
    }
    float d0[4], d1[4], m = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        d0[i] = __fsub_rn(e0[i], mu);
        d1[i] = __fsub_rn(e1[i], mu);
        if (ok0[i]) m = fmaxf(m, fabsf(d0[i]));
        if (ok1[i]) m = fmaxf(m, fabsf(d1[i]));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float b = __fdiv_rn(m, 127.0f);
    if (lane == 0) scale[g] = b;
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int r0 = 0, r1 = 0;
        if (b != 0.f) {
            float q0 = fminf(fmaxf(rintf(__fdiv_rn(d0[i], b)), -127.f), 127.f);
            float q1 = fminf(fmaxf(rintf(__fdiv_rn(d1[i], b)), -127.f), 127.f);
            r0 = (int)q0;
            r1 = (int)q1;
        }
        w0 |= ((uint32_t)(r0 & 0xff)) << (8 * i);
        w1 |= ((uint32_t)(r1 & 0xff)) << (8 * i);
    }
    if (j0 + 4 <= nb) {
        *reinterpret_cast<uint32_t *>(qabs + j0) = w0;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (ok0[i]) qabs[j0 + i] = (int8_t)((w0 >> (8 * i)) & 0xff);
    }
    if (j1 + 4 <= nb) {
        *reinterpret_cast<uint32_t *>(qabs + j1) = w1;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (ok1[i]) qabs[j1 + i] = (int8_t)((w1 >> (8 * i)) & 0xff);
    }
}

size_t dq_workspace_bytes(int64_t nb) {
    const int64_t np = (nb + kMeanChunk - 1) / kMeanChunk;
    return (size_t)(256 + ((np * 8 + 255) / 256) * 256);
}

int64_t dq_max_blocks() { return (int64_t)kMaxPartials * kMeanChunk; }

cudaError_t launch_nf4_double_quant(const float *absmax, int64_t nb, int8_t *qabs, float *scale, float *mu,
                                    void *ws, cudaStream_t st) {
    const int np = (int)((nb + kMeanChunk - 1) / kMeanChunk);
    int np2 = 1;
    while (np2 < np) np2 <<= 1;
    double *partial = reinterpret_cast<double *>(reinterpret_cast<char *>(ws) + 256);
    dq_partial_kernel<<<np, kMeanThreads, 0, st>>>(absmax, nb, partial);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    const int64_t grid = (ng + (kDqThreads / 32) - 1) / (kDqThreads / 32);
    dq_quant_kernel<<<(unsigned)grid, kDqThreads, 0, st>>>(absmax, nb, partial, np, np2, qabs, scale, mu);
    note_launch();
    return cudaGetLastError();
}

// ===========================================================================
// Allocation-free double quantization.  The only scratch K2/K3 need is the
// binary64 partial sums of mu, one per 8192 block constants.  This variant
// keeps them in a fixed, file-scope device array instead of a caller
// workspace, so a caller that cannot allocate device memory can still run the
// path.  The array is 8 KB (1024 partials), which caps nb at 1024 * 8192 =
// 8,388,608 blocks (536,870,912 weights); every GPU that loads the library
// holds it until the process exits.  Each call overwrites every partial it
// reads before reading it, so nothing has to be cleared between calls; two
// calls that overlap on the GPU (different streams, no ordering) share the
// array and race.
// ===========================================================================
constexpr int kStaticPartials = 1024;
static __device__ __align__(256) double g_dq_static_partials[kStaticPartials];
static std::atomic<double *> g_dq_static_ptr[64];

int64_t dq_static_max_blocks() { return (int64_t)kStaticPartials * kMeanChunk; }

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
    const int np = (int)((nb + kMeanChunk - 1) / kMeanChunk);
    int np2 = 1;
    while (np2 < np) np2 <<= 1;
    dq_partial_kernel<<<np, kMeanThreads, 0, st>>>(absmax, nb, partial);
    note_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t ng = (nb + kDqGroup - 1) / kDqGroup;
    const int64_t grid = (ng + (kDqThreads / 32) - 1) / (kDqThreads / 32);
    dq_quant_kernel<<<(unsigned)grid, kDqThreads, 0, st>>>(absmax, nb, partial, np, np2, qabs, scale, mu);
    note_launch();
    return cudaGetLastError();
}

// ===========================================================================
// K4: doubleDequant to BF16.  A warp streams 64 code words (512 weights,
// 8 blocks) per step: lane l decodes words 2l and 2l+1 (16 weights of block
// l/4) with the register-only table decode and stores 32 contiguous bytes.
// w' = bf16_RN(fp32(ahat * c[q])).
// ===========================================================================
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint2 *__restrict__ codes64,
                                                          const float *__restrict__ absmax,
                                                          const int8_t *__restrict__ qabs,
                                                          const float *__restrict__ scale,
                                                          const float *__restrict__ mu_p, int64_t npairs,
                                                          uint4 *__restrict__ out) {
    const float mu = qabs ? __ldg(mu_p) : 0.f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < npairs; i += stride) {
        const int64_t j = i >> 2;  // 4 pairs of words (64 codes) per block
        float ah;
        if (qabs) ah = dq_restore(__ldg(qabs + j), __ldg(scale + (j >> 8)), mu);
        else ah = __ldg(absmax + j);
        const uint2 cw = __ldcs(codes64 + i);
        const NF4Table t = nf4_table(ah);
        __stcs(out + 2 * i, nf4_decode8(cw.x, t));
        __stcs(out + 2 * i + 1, nf4_decode8(cw.y, t));
    }
}

cudaError_t launch_nf4_dequant(const qln_nf4_weight *w, uint16_t *out, cudaStream_t st, int num_sms) {
    const int64_t numel = w->rows * w->cols;
    const int64_t npairs = numel / 16;
    int64_t grid = (npairs + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    nf4_dequant_kernel<<<(unsigned)grid, 256, 0, st>>>(reinterpret_cast<const uint2 *>(w->codes), w->absmax,
                                                      w->qabs, w->dq_scale, w->dq_mean, npairs,
                                                      reinterpret_cast<uint4 *>(out));
    note_launch();
    return cudaGetLastError();
}

}  // namespace qln
