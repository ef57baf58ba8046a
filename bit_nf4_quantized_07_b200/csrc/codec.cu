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
// xor-shuffles; x = w / absmax is the IEEE fp32 quotient, in [-1, 1].
// Snap without a 15-way compare and (almost always) without a division: the
// top 12 bits of x (sign, exponent, three mantissa bits) name an interval of
// fp32 values that contains at most one snap threshold (the narrowest gap between thresholds, 0.08, is wider than
// any such interval below 1 in magnitude).  A per-CTA table gives, for each
// key, the code of the interval's smallest value and that one threshold (or
// +inf), so  q = base[key] + (x > thr[key])  -- exactly #{k : x > t_k}.
// ===========================================================================
constexpr int kSnapKeys = 4096;

// Only keys of |x| <= 1.125 are ever looked up (|x| <= 1 up to a few ulps of
// the reciprocal product), i.e. keys 0x000..0x3F8 and 0x800..0xBF8.
__device__ void build_snap_lut(uint2 *lut) {
    float t[15];
#pragma unroll
    for (int k = 0; k < 15; ++k) t[k] = nf4_threshold(k);
    for (int i = threadIdx.x; i < 2 * 1024; i += blockDim.x) {
        const int key = (i & 1023) | ((i >> 10) << 11);
        if ((key & 0x3FF) > 0x3F8) continue;
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

// Codes of the 4 weights of v (block absmax a > 0, inv = the hardware
// reciprocal of a, relative error <= 2^-23), packed as two bytes, first weight
// in the high nibble of the first byte.  The product y = RN(w * inv) differs
// from the real quotient w/a by at most |w/a| (2^-23 + 2^-24) < 1.8e-7, and
// x = RN(w/a) is within 2^-25 of it, so y and x fall on the same side of a
// threshold t unless |y - t| < 2.2e-7 < 2^-21.  Only then is the exact quotient
// formed (IEEE division) and used instead: the code is always that of x.  The
// test looks only at the threshold of y's own key interval; that is enough
// because every threshold lies more than 15,000 ulps inside its key interval,
// so no threshold of a neighbouring interval is that close to y.  When a or
// 1/a is subnormal (a < 2^-126 or a >= 2^126) the bound does not hold and the
// group takes the exact path outright.
__device__ __forceinline__ uint32_t snap4(float4 v, float a, float inv, const uint2 *lut) {
    const float w[4] = {v.x, v.y, v.z, v.w};
    float y[4];
    {   // both products of a pair from one paired multiply (each rounded to nearest)
        uint64_t inv2, p01, p23;
        asm("mov.b64 %0, {%1, %1};" : "=l"(inv2) : "f"(inv));
        asm("{\n\t.reg .b64 a;\n\tmov.b64 a, {%1, %2};\n\tmul.rn.f32x2 %0, a, %3;\n\t}" : "=l"(p01) : "f"(w[0]), "f"(w[1]), "l"(inv2));
        asm("{\n\t.reg .b64 a;\n\tmov.b64 a, {%1, %2};\n\tmul.rn.f32x2 %0, a, %3;\n\t}" : "=l"(p23) : "f"(w[2]), "f"(w[3]), "l"(inv2));
        asm("mov.b64 {%0, %1}, %2;" : "=f"(y[0]), "=f"(y[1]) : "l"(p01));
        asm("mov.b64 {%0, %1}, %2;" : "=f"(y[2]), "=f"(y[3]) : "l"(p23));
    }
    uint32_t q[4];
    float dmin = 1.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint2 e = lut[__float_as_uint(y[i]) >> 20];
        const float d = __fsub_rn(y[i], __uint_as_float(e.x));
        q[i] = e.y + (d > 0.f ? 1u : 0u);
        dmin = fminf(dmin, fabsf(d));
    }
    const bool near = dmin < 4.76837158203125e-07f;  // some |y - t| < 2^-21
    if (near || !(a >= 0x1p-126f && a < 0x1p126f)) {  // rare: redo the group exactly (also for a or 1/a subnormal)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float x = __fdiv_rn(w[i], a);
            const uint2 e = lut[__float_as_uint(x) >> 20];
            q[i] = e.y + ((x > __uint_as_float(e.x)) ? 1u : 0u);
        }
    }
    if (!(a > 0.f)) return 0x7777u;  // all-zero block: the exact zero
    return (q[0] << 4) | q[1] | (q[2] << 12) | (q[3] << 8);
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

    // Two 256-weight chunks per iteration: four 16-byte loads in flight per lane.
    for (int64_t c0 = warp; c0 < nchunks; c0 += 2 * nwarps) {
        float4 v[2][2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t c = c0 + u * nwarps;
            const int64_t b0 = 4 * c + (lane >> 4);
            const float4 *src = W + 64 * c + lane;
            v[u][0] = (c < nchunks && b0 < nb) ? __ldcs(src) : make_float4(0.f, 0.f, 0.f, 0.f);
            v[u][1] = (c < nchunks && b0 + 2 < nb) ? __ldcs(src + 32) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // block absmax: |w| >= 0, so the bit patterns order like the values and a
        // 16-lane integer max reduction (one per half-warp, each with its own mask) is exact
        const unsigned half_mask = (lane < 16) ? 0x0000ffffu : 0xffff0000u;
        float m[2][2];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                m[u][h] = __uint_as_float(__reduce_max_sync(half_mask, __float_as_uint(absmax4(v[u][h]))));
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t c = c0 + u * nwarps;
            if (c >= nchunks) break;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t b = 4 * c + (lane >> 4) + 2 * h;  // block of v[u][h]
                if (b < nb) {
                    const float a = m[u][h];
                    float inv = 0.f;
                    if (a > 0.f) asm("rcp.approx.f32 %0, %1;" : "=f"(inv) : "f"(a));
                    __stcs(codes16 + 64 * c + 32 * h + lane, (uint16_t)snap4(v[u][h], a, inv, lut));
                    if ((lane & 15) == 0) absmax[b] = a;
                }
            }
        }
    }
}

cudaError_t launch_nf4_quantize(const float *W, int64_t numel, uint8_t *codes, float *absmax,
                                cudaStream_t st, int num_sms) {
    const int64_t nb = numel / kBlock;
    const int64_t nchunks = (nb + 3) / 4;
    const int threads = 256;
    int64_t grid = (nchunks + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 4;  // the table is built once per CTA
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
                                                          uint4 *__restrict__ out) {
    __shared__ __align__(16) uint4 stage[8][128];  // per warp 2 KB
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
        const float ah = qabs ? dq_restore(d0.q, d0.v, mu) : d0.v;
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
                                        uint4 *__restrict__ out) {
    const int64_t k = threadIdx.x;
    if (k >= ng) return;
    const int64_t i = g0 + k, j = i >> 1;
    const float ah = qabs ? dq_restore(__ldg(qabs + j), __ldg(scale + (j >> 8)), __ldg(mu_p)) : __ldg(absmax + j);
    const NF4Table t = nf4_table(ah);
    const uint4 cw = __ldg(codes128 + i);
    out[4 * i + 0] = nf4_decode8(cw.x, t);
    out[4 * i + 1] = nf4_decode8(cw.y, t);
    out[4 * i + 2] = nf4_decode8(cw.z, t);
    out[4 * i + 3] = nf4_decode8(cw.w, t);
}

cudaError_t launch_nf4_dequant(const qln_nf4_weight *w, uint16_t *out, cudaStream_t st, int num_sms) {
    const int64_t numel = w->rows * w->cols;
    const int64_t nchunks = numel / 1024;  // weights come in whole 64-blocks; chunks of 1024 + a tail below
    const int64_t tail = numel - nchunks * 1024;
    int64_t grid = (nchunks + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 6;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    if (nchunks > 0) {
        nf4_dequant_kernel<<<(unsigned)grid, 256, 0, st>>>(reinterpret_cast<const uint4 *>(w->codes), w->absmax,
                                                          w->qabs, w->dq_scale, w->dq_mean, nchunks,
                                                          reinterpret_cast<uint4 *>(out));
        note_launch();
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (tail > 0) {  // fewer than 1024 weights left: whole blocks, one 32-weight group per thread
        const int64_t g0 = nchunks * 32, ng = tail / 32;
        nf4_dequant_tail_kernel<<<1, 64, 0, st>>>(reinterpret_cast<const uint4 *>(w->codes), w->absmax, w->qabs,
                                                   w->dq_scale, w->dq_mean, g0, ng, reinterpret_cast<uint4 *>(out));
        note_launch();
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace qln
