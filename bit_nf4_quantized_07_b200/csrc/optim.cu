// The AdamW update of the LoRA factors, with the optimizer states optionally
// in unified (managed) memory -- the paged optimizer of the QLoRA recipe.
//
// Pages: deck "3 QLoRA Finetuning" card 5 (paged optimizers: optimizer states
// in NVIDIA unified memory, paged out to CPU RAM when the GPU runs short and
// paged back for the update); "LoRA 与 QLoRA" QLoRA usage notes
// (paged_adamw_32bit: 32-bit AdamW states, for the LoRA parameters only).
// The update is the published AdamW (Loshchilov & Hutter, "Decoupled Weight
// Decay Regularization", ICLR 2019), decay applied to the weight before the
// adaptive step:
//   m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) g^2;  p = p (1 - lr wd);
//   p = p - (lr / (1 - b1^t)) m / (sqrt(v / (1 - b2^t)) + eps)
// An HBM-bound elementwise pass: 16 B read and 12 B (+2 B BF16) written per
// element, four elements per thread per step, a grid-stride loop over
// whole-SM waves.
#include "qln_common.cuh"
#include "qln_internal.h"

namespace qln {

struct AdamWArgs {
    float *p;
    const float *g;
    float *m;
    float *v;
    uint16_t *p_bf16;  // may be null
    int64_t n;
    float lr, b1, b2, eps, wd;
    const int64_t *step;  // device: the step being taken, t >= 1
};

__device__ __forceinline__ void adamw_elem(float &p, float g, float &m, float &v, const AdamWArgs &a, float step_size,
                                           float inv_sqrt_bc2) {
    m = __fadd_rn(__fmul_rn(a.b1, m), __fmul_rn(1.0f - a.b1, g));
    v = __fadd_rn(__fmul_rn(a.b2, v), __fmul_rn(1.0f - a.b2, __fmul_rn(g, g)));
    p = __fmul_rn(p, 1.0f - a.lr * a.wd);
    const float denom = __fadd_rn(__fmul_rn(__fsqrt_rn(v), inv_sqrt_bc2), a.eps);
    p = __fsub_rn(p, __fmul_rn(step_size, __fdiv_rn(m, denom)));
}

__global__ void __launch_bounds__(256) adamw_kernel(const AdamWArgs a) {
    pdl_wait();
    // bias corrections of step t, in binary64 once per thread
    const int64_t tv = *a.step;
    const double t = (double)(tv < 1 ? 1 : tv);  // a step below 1 is taken as the first
    const double bc1 = 1.0 - pow((double)a.b1, t), bc2 = 1.0 - pow((double)a.b2, t);
    const float step_size = (float)((double)a.lr / bc1);
    const float inv_sqrt_bc2 = (float)(1.0 / sqrt(bc2));
    const int64_t n4 = a.n / 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        float4 p = reinterpret_cast<const float4 *>(a.p)[i];
        const float4 g = __ldcs(reinterpret_cast<const float4 *>(a.g) + i);
        float4 m = reinterpret_cast<const float4 *>(a.m)[i];
        float4 v = reinterpret_cast<const float4 *>(a.v)[i];
        adamw_elem(p.x, g.x, m.x, v.x, a, step_size, inv_sqrt_bc2);
        adamw_elem(p.y, g.y, m.y, v.y, a, step_size, inv_sqrt_bc2);
        adamw_elem(p.z, g.z, m.z, v.z, a, step_size, inv_sqrt_bc2);
        adamw_elem(p.w, g.w, m.w, v.w, a, step_size, inv_sqrt_bc2);
        reinterpret_cast<float4 *>(a.p)[i] = p;
        reinterpret_cast<float4 *>(a.m)[i] = m;
        reinterpret_cast<float4 *>(a.v)[i] = v;
        if (a.p_bf16)
            reinterpret_cast<uint2 *>(a.p_bf16)[i] = make_uint2(pack_bf16x2(p.x, p.y), pack_bf16x2(p.z, p.w));
    }
    // the n mod 4 tail
    const int64_t j = 4 * n4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j < a.n) {
        float p = a.p[j], m = a.m[j], v = a.v[j];
        adamw_elem(p, a.g[j], m, v, a, step_size, inv_sqrt_bc2);
        a.p[j] = p;
        a.m[j] = m;
        a.v[j] = v;
        if (a.p_bf16) {
            const __nv_bfloat16 b = __float2bfloat16_rn(p);
            a.p_bf16[j] = *reinterpret_cast<const uint16_t *>(&b);
        }
    }
}

// Managed-memory pages of [ptr, ptr + bytes) to `device` (cudaCpuDeviceId for
// host RAM), queued on the stream; nothing for memory of any other kind.
static cudaError_t page_to(const void *ptr, size_t bytes, int device, cudaStream_t st) {
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, ptr);
    if (e != cudaSuccess) {
        cudaGetLastError();  // an unregistered host pointer is not an error here
        return cudaSuccess;
    }
    if (at.type != cudaMemoryTypeManaged) return cudaSuccess;
    return cudaMemPrefetchAsync(ptr, bytes, device, st);
}

cudaError_t launch_adamw(float *p, const float *g, float *m, float *v, uint16_t *p_bf16, int64_t n, float lr,
                         float b1, float b2, float eps, float wd, const int64_t *step, int flags, cudaStream_t st,
                         int num_sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const size_t bytes = (size_t)n * sizeof(float);
    if (flags & QLN_ADAMW_PAGE_IN) {  // page the operands back in before the update
        const void *ops[4] = {p, g, m, v};
        for (const void *q : ops)
            if ((e = page_to(q, bytes, dev, st)) != cudaSuccess) return e;
    }
    AdamWArgs a{p, g, m, v, p_bf16, n, lr, b1, b2, eps, wd, step};
    int64_t grid = (n / 4 + 255) / 256;
    if (grid > (int64_t)num_sms * 8) grid = (int64_t)num_sms * 8;
    if (grid < 1) grid = 1;
    e = launch_pdl(adamw_kernel, dim3((unsigned)grid), dim3(256), 0, st, a);
    if (e != cudaSuccess) return e;
    if (flags & QLN_ADAMW_PAGE_OUT) {  // states back to host RAM until the next update
        if ((e = page_to(m, bytes, cudaCpuDeviceId, st)) != cudaSuccess) return e;
        if ((e = page_to(v, bytes, cudaCpuDeviceId, st)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace qln
