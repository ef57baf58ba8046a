// C ABI of libqlora_nf4: argument checks, workspace layout, kernel dispatch.
// Every entry point validates synchronously, then only enqueues work on the
// caller's stream: no device-memory allocation, no synchronisation, no
// host-device copies, no streams or events of its own.
#include <string.h>

#include <atomic>
#include <vector>

#include "qln_common.cuh"
#include "qln_internal.h"

namespace qln {
static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace qln

namespace {
using qln::note_launch;

constexpr int kMaxDevices = 64;
constexpr int32_t kMaxBatchJobs = 1 << 20;  // jobs per nf4_quantize_dq_batch call
int g_arch_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 not sm_100
int g_num_sms[kMaxDevices];

qln_status check_device(int *num_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QLN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return QLN_ERR_CUDA;
    if (g_arch_ok[dev] == 0) {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return QLN_ERR_CUDA;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return QLN_ERR_CUDA;
        g_num_sms[dev] = sms;
        g_arch_ok[dev] = (major == 10) ? 1 : -1;
    }
    if (g_arch_ok[dev] < 0) return QLN_ERR_ARCH;
    *num_sms = g_num_sms[dev];
    return QLN_OK;
}

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Split-K plans are made for this SM count (B200) on every device, so the
// workspace size never depends on the device queried.
constexpr int kSplitTargetSms = 148;

// Workspace layout of the linear calls (all offsets 256-byte aligned):
//   [0, 256)        header: int32 device status word (0 = QLN_OK) at 0
//   fwd: sU [n][r] bf16, U [n][r] bf16 (used when U_out is NULL),
//        split-K partials of U (fp32); the decode-sized forward uses only the
//        header
//   bwd: G [n][r] bf16, sG [n][r] bf16, U [n][r] bf16, split-K partials of
//        G / U (fp32, reused), dA partials, dB partials
// Split counts are planned for a fixed SM count so that the workspace size
// does not depend on the device queried.
struct FwdWs {
    size_t sU, U, pU, total;
};
struct BwdWs {
    size_t G, sG, U, pGU, pA, pB, total;
    int splitA, splitB;
};

FwdWs fwd_layout(int64_t rows, int64_t cols, int64_t n, int r) {
    FwdWs L;
    const size_t nr = round256((size_t)n * r * 2);
    (void)rows;
    L.sU = qln::kWsHeaderBytes;
    L.U = L.sU + nr;
    L.pU = L.U + nr;
    L.total = L.pU + round256(qln::lora_down_partial_bytes(n, cols, r, kSplitTargetSms));
    return L;
}

BwdWs bwd_layout(int64_t rows, int64_t cols, int64_t n, int r) {
    BwdWs L;
    const size_t nr = round256((size_t)n * r * 2);
    L.G = qln::kWsHeaderBytes;
    L.sG = L.G + nr;
    L.U = L.sG + nr;
    L.pGU = L.U + nr;
    const size_t pg = qln::lora_down_partial_bytes(n, rows, r, kSplitTargetSms);
    const size_t pu = qln::lora_down_partial_bytes(n, cols, r, kSplitTargetSms);
    L.splitA = qln::tn_skinny_splits(n, cols, r, kSplitTargetSms);
    L.splitB = qln::tn_skinny_splits(n, rows, r, kSplitTargetSms);
    L.pA = L.pGU + round256(pg > pu ? pg : pu);
    L.pB = L.pA + round256(qln::tn_skinny_partials_bytes(cols, r, L.splitA));
    L.total = L.pB + round256(qln::tn_skinny_partials_bytes(rows, r, L.splitB));
    return L;
}

qln_status check_weight(const qln_nf4_weight *w) {
    if (!w || !w->codes) return QLN_ERR_NULL;
    if (w->qabs) {
        if (!w->dq_scale || !w->dq_mean) return QLN_ERR_NULL;
    } else if (!w->absmax) {
        return QLN_ERR_NULL;
    }
    if (w->rows <= 0 || w->cols <= 0 || (w->cols % 64) != 0) return QLN_ERR_SHAPE;
    if (w->dq_format != QLN_DQ_INT8 && w->dq_format != QLN_DQ_E4M3) return QLN_ERR_SHAPE;
    if (!aligned(w->codes, 16)) return QLN_ERR_ALIGN;
    if (w->absmax && !aligned(w->absmax, 4)) return QLN_ERR_ALIGN;
    if (w->dq_scale && !aligned(w->dq_scale, 4)) return QLN_ERR_ALIGN;
    if (w->dq_mean && !aligned(w->dq_mean, 4)) return QLN_ERR_ALIGN;
    return QLN_OK;
}

qln_status check_linear(const qln_nf4_weight *w, const uint16_t *X, int64_t n, const uint16_t *A,
                        const uint16_t *B, int32_t r) {
    qln_status s = check_weight(w);
    if (s != QLN_OK) return s;
    if (!X || !A || !B) return QLN_ERR_NULL;
    if (n < 1 || r < 8 || r > 128 || (r % 8) != 0) return QLN_ERR_SHAPE;
    if ((w->rows % 64) != 0) return QLN_ERR_SHAPE;
    if (!aligned(X, 16) || !aligned(A, 16) || !aligned(B, 16)) return QLN_ERR_ALIGN;
    return QLN_OK;
}

qln_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QLN_OK : QLN_ERR_CUDA; }

// The fused weight GEMM: tcgen05 where the shape fills its tiles, otherwise
// the register-level path.
cudaError_t fused_gemm(const qln_nf4_weight *w, bool trans, const uint16_t *act, int64_t n, const uint16_t *lact,
                       const uint16_t *lw, int r, uint16_t *out, int *status, cudaStream_t st, int num_sms) {
    if (qln::nf4_tc_gemm_supported(w, trans, n, r))
        return qln::launch_nf4_tc_gemm(w, trans, act, n, lact, lw, r, out, status, st, num_sms);
    return qln::launch_nf4_mma_gemm(w, trans, act, n, lact, lw, r, out, status, st, num_sms);
}

// dA and dB beside the dX GEMM: when the GEMM leaves at least this many SMs
// idle (one wave of fewer CTAs than SMs), one persistent launch of as many
// CTAs as idle SMs computes both on those SMs.  It is the GEMM's programmatic
// dependent, so it starts only once every GEMM CTA is resident and can never
// hold an SM the GEMM needs.
constexpr int64_t kSideMinCtas = 8;

}  // namespace

extern "C" {

qln_status nf4_quantize(const float *W, int64_t numel, uint8_t *codes, float *absmax, void *stream) {
    if (!W || !codes || !absmax) return QLN_ERR_NULL;
    if (numel <= 0 || (numel % 64) != 0) return QLN_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(absmax, 4)) return QLN_ERR_ALIGN;
    int sms = 0;
    qln_status s = check_device(&sms);
    if (s != QLN_OK) return s;
    return from_cuda(qln::launch_nf4_quantize(W, QLN_DTYPE_F32, numel, codes, absmax, (cudaStream_t)stream, sms));
}

qln_status nf4_quantize_ex(const void *W, int32_t dtype, int64_t numel, uint8_t *codes, float *absmax,
                           void *stream) {
    if (!W || !codes || !absmax) return QLN_ERR_NULL;
    if (numel <= 0) return QLN_ERR_SHAPE;
    if (dtype != QLN_DTYPE_F32 && dtype != QLN_DTYPE_BF16 && dtype != QLN_DTYPE_F16) return QLN_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(absmax, 4)) return QLN_ERR_ALIGN;
    int sms = 0;
    qln_status s = check_device(&sms);
    if (s != QLN_OK) return s;
    return from_cuda(qln::launch_nf4_quantize(W, dtype, numel, codes, absmax, (cudaStream_t)stream, sms));
}

qln_status nf4_double_quant_ex(const float *absmax, int64_t nb, int32_t dq_format, void *qabs_v, float *dq_scale,
                               float *dq_mean, void *ws, size_t ws_bytes, void *stream) {
    int8_t *qabs = static_cast<int8_t *>(qabs_v);
    if (dq_format != QLN_DQ_INT8 && dq_format != QLN_DQ_E4M3) return QLN_ERR_SHAPE;
    if (!absmax || !qabs || !dq_scale || !dq_mean || !ws) return QLN_ERR_NULL;
    if (nb <= 0 || nb > qln::dq_max_blocks()) return QLN_ERR_SHAPE;
    if (!aligned(absmax, 16) || !aligned(qabs, 4) || !aligned(dq_scale, 4) || !aligned(dq_mean, 4))
        return QLN_ERR_ALIGN;
    if (!aligned(ws, 256)) return QLN_ERR_ALIGN;
    if (ws_bytes < qln::dq_workspace_bytes(nb)) return QLN_ERR_WORKSPACE;
    int sms = 0;
    qln_status s = check_device(&sms);
    if (s != QLN_OK) return s;
    return from_cuda(qln::launch_nf4_double_quant(absmax, nb, qabs, dq_scale, dq_mean, ws, dq_format == QLN_DQ_E4M3,
                                                     (cudaStream_t)stream, sms));
}

qln_status nf4_quantize_dq(const void *W, int32_t dtype, int64_t numel, int32_t dq_format, uint8_t *codes,
                           float *absmax, void *qabs_v, float *dq_scale, float *dq_mean, void *ws, size_t ws_bytes,
                           void *stream) {
    int8_t *qabs = static_cast<int8_t *>(qabs_v);
    if (!W || !codes || !absmax || !qabs || !dq_scale || !dq_mean || !ws) return QLN_ERR_NULL;
    if (numel <= 0 || (numel + 63) / 64 > qln::dq_max_blocks()) return QLN_ERR_SHAPE;
    if (dtype != QLN_DTYPE_F32 && dtype != QLN_DTYPE_BF16 && dtype != QLN_DTYPE_F16) return QLN_ERR_SHAPE;
    if (dq_format != QLN_DQ_INT8 && dq_format != QLN_DQ_E4M3) return QLN_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(absmax, 16) || !aligned(qabs, 4) ||
        !aligned(dq_scale, 4) || !aligned(dq_mean, 4) || !aligned(ws, 256))
        return QLN_ERR_ALIGN;
    if (ws_bytes < qln::dq_workspace_bytes((numel + 63) / 64)) return QLN_ERR_WORKSPACE;
    int sms = 0;
    qln_status s = check_device(&sms);
    if (s != QLN_OK) return s;
    return from_cuda(qln::launch_nf4_quantize_dq(W, dtype, numel, codes, absmax, qabs, dq_scale, dq_mean, ws,
                                                    dq_format == QLN_DQ_E4M3, (cudaStream_t)stream, sms));
}

static qln_status check_quant_job(const qln_quant_job &j) {
    if (!j.W || !j.codes || !j.absmax || !j.qabs || !j.dq_scale || !j.dq_mean) return QLN_ERR_NULL;
    if (j.numel <= 0 || (j.numel + 63) / 64 > qln::dq_max_blocks()) return QLN_ERR_SHAPE;
    if (j.dtype != QLN_DTYPE_F32 && j.dtype != QLN_DTYPE_BF16 && j.dtype != QLN_DTYPE_F16) return QLN_ERR_SHAPE;
    if (j.dq_format != QLN_DQ_INT8 && j.dq_format != QLN_DQ_E4M3) return QLN_ERR_SHAPE;
    if (!aligned(j.W, 16) || !aligned(j.codes, 16) || !aligned(j.absmax, 16) || !aligned(j.qabs, 4) ||
        !aligned(j.dq_scale, 4) || !aligned(j.dq_mean, 4))
        return QLN_ERR_ALIGN;
    return QLN_OK;
}

qln_status nf4_quantize_dq_batch(const qln_quant_job *jobs, int32_t njobs, void *ws, size_t ws_bytes, void *stream) {
    if (!jobs || !ws) return QLN_ERR_NULL;
    if (njobs < 1 || njobs > kMaxBatchJobs) return QLN_ERR_SHAPE;
    if (!aligned(ws, 256)) return QLN_ERR_ALIGN;
    for (int32_t i = 0; i < njobs; ++i) {
        const qln_status s = check_quant_job(jobs[i]);
        if (s != QLN_OK) return s;
    }
    if (ws_bytes < qln::kDqBatchScratchBytes * (size_t)njobs) return QLN_ERR_WORKSPACE;
    int sms = 0;
    qln_status s = check_device(&sms);
    if (s != QLN_OK) return s;
    std::vector<qln::QuantJob> q((size_t)njobs);
    for (int32_t i = 0; i < njobs; ++i) {
        const qln_quant_job &j = jobs[i];
        q[(size_t)i] = qln::QuantJob{j.W, j.dtype, j.numel, j.codes, j.absmax, static_cast<int8_t *>(j.qabs),
                                     j.dq_scale, j.dq_mean, j.dq_format == QLN_DQ_E4M3};
    }
    return from_cuda(qln::launch_nf4_quantize_dq_batch(q.data(), njobs, ws, (cudaStream_t)stream, sms));
}

qln_status nf4_double_quant(const float *absmax, int64_t nb, int8_t *qabs, float *dq_scale, float *dq_mean,
                            void *ws, size_t ws_bytes, void *stream) {
    return nf4_double_quant_ex(absmax, nb, QLN_DQ_INT8, qabs, dq_scale, dq_mean, ws, ws_bytes, stream);
}

qln_status nf4_double_quant_noalloc(const float *absmax, int64_t nb, int8_t *qabs, float *dq_scale,
                                    float *dq_mean, void *stream) {
    if (!absmax || !qabs || !dq_scale || !dq_mean) return QLN_ERR_NULL;
    if (nb <= 0 || nb > qln::dq_static_max_blocks()) return QLN_ERR_SHAPE;
    if (!aligned(absmax, 16) || !aligned(qabs, 4) || !aligned(dq_scale, 4) || !aligned(dq_mean, 4))
        return QLN_ERR_ALIGN;
    int sms = 0;
    qln_status s = check_device(&sms);
    if (s != QLN_OK) return s;
    return from_cuda(qln::launch_nf4_double_quant_static(absmax, nb, qabs, dq_scale, dq_mean, (cudaStream_t)stream, sms));
}

qln_status nf4_dequant(const qln_nf4_weight *w, uint16_t *out, void *stream) {
    qln_status s = check_weight(w);
    if (s != QLN_OK) return s;
    if (!out) return QLN_ERR_NULL;
    if (!aligned(out, 16)) return QLN_ERR_ALIGN;
    int sms = 0;
    s = check_device(&sms);
    if (s != QLN_OK) return s;
    return from_cuda(qln::launch_nf4_dequant(w, out, (cudaStream_t)stream, sms));
}

qln_status qln_adamw_step(float *param, const float *grad, float *m, float *v, uint16_t *param_bf16, int64_t n,
                          const qln_adamw_config *cfg, const int64_t *step, int32_t flags, void *stream) {
    if (!param || !grad || !m || !v || !cfg || !step) return QLN_ERR_NULL;
    if (n <= 0) return QLN_ERR_SHAPE;
    if (!aligned(param, 16) || !aligned(grad, 16) || !aligned(m, 16) || !aligned(v, 16)) return QLN_ERR_ALIGN;
    if (param_bf16 && !aligned(param_bf16, 8)) return QLN_ERR_ALIGN;
    int sms = 0;
    qln_status s = check_device(&sms);
    if (s != QLN_OK) return s;
    return from_cuda(qln::launch_adamw(param, grad, m, v, param_bf16, n, cfg->lr, cfg->beta1, cfg->beta2, cfg->eps,
                                       cfg->weight_decay, step, flags, (cudaStream_t)stream, sms));
}

qln_status nf4_dequant_flat(const qln_nf4_weight *w, int64_t numel, uint16_t *out, void *stream) {
    if (!w || !w->codes || !out) return QLN_ERR_NULL;
    if (w->qabs) {
        if (!w->dq_scale || !w->dq_mean) return QLN_ERR_NULL;
    } else if (!w->absmax) {
        return QLN_ERR_NULL;
    }
    if (numel <= 0) return QLN_ERR_SHAPE;
    if (w->dq_format != QLN_DQ_INT8 && w->dq_format != QLN_DQ_E4M3) return QLN_ERR_SHAPE;
    if (!aligned(w->codes, 16) || !aligned(out, 16)) return QLN_ERR_ALIGN;
    if (w->absmax && !aligned(w->absmax, 4)) return QLN_ERR_ALIGN;
    if (w->dq_scale && !aligned(w->dq_scale, 4)) return QLN_ERR_ALIGN;
    if (w->dq_mean && !aligned(w->dq_mean, 4)) return QLN_ERR_ALIGN;
    int sms = 0;
    qln_status s = check_device(&sms);
    if (s != QLN_OK) return s;
    return from_cuda(qln::launch_nf4_dequant_flat(w, numel, out, (cudaStream_t)stream, sms));
}

qln_status qlora_linear_fwd(const qln_nf4_weight *w, const uint16_t *X, int64_t n, const uint16_t *A,
                            const uint16_t *B, int32_t r, float s, uint16_t *Y, uint16_t *U_out, void *ws,
                            size_t ws_bytes, void *stream) {
    qln_status st = check_linear(w, X, n, A, B, r);
    if (st != QLN_OK) return st;
    if (!Y || !ws) return QLN_ERR_NULL;
    if (!aligned(Y, 16) || (U_out && !aligned(U_out, 16)) || !aligned(ws, 256)) return QLN_ERR_ALIGN;
    const FwdWs L = fwd_layout(w->rows, w->cols, n, r);
    if (ws_bytes < L.total) return QLN_ERR_WORKSPACE;
    int sms = 0;
    st = check_device(&sms);
    if (st != QLN_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    char *wsb = reinterpret_cast<char *>(ws);
    int *status = reinterpret_cast<int *>(wsb);
    uint16_t *sU = reinterpret_cast<uint16_t *>(wsb + L.sU);
    uint16_t *U = U_out ? U_out : reinterpret_cast<uint16_t *>(wsb + L.U);
    float *pU = reinterpret_cast<float *>(wsb + L.pU);
    if (qln::nf4_decode_fwd_supported(w, n, r)) {
        // decode-sized n: one launch forms U and the whole forward; it clears
        // the status word itself, so no memset precedes it
        return from_cuda(qln::launch_nf4_decode_fwd(w, X, n, A, B, r, s, Y, U_out, status, cs));
    }
    // U = X A^T (and s*U for the adapter MMA; its first kernel also clears the
    // status word), then the fused weight GEMM.  No memset between kernels:
    // the launches chain by programmatic dependent launch.
    cudaError_t e = qln::launch_lora_down(X, n, w->cols, A, false, r, s, U, sU, pU, cs, kSplitTargetSms, status);
    if (e != cudaSuccess) return QLN_ERR_CUDA;
    e = fused_gemm(w, false, X, n, sU, B, r, Y, status, cs, sms);
    return from_cuda(e);
}

qln_status qlora_linear_bwd(const qln_nf4_weight *w, const uint16_t *X, int64_t n, const uint16_t *A,
                            const uint16_t *B, int32_t r, float s, const uint16_t *dY, const uint16_t *U,
                            uint16_t *dX, float *dA, float *dB, void *ws, size_t ws_bytes, void *stream) {
    qln_status st = check_linear(w, X, n, A, B, r);
    if (st != QLN_OK) return st;
    if (!dY || !dX || !dA || !dB || !ws) return QLN_ERR_NULL;
    if (!aligned(dY, 16) || !aligned(dX, 16) || !aligned(dA, 16) || !aligned(dB, 16) || !aligned(ws, 256) ||
        (U && !aligned(U, 16)))
        return QLN_ERR_ALIGN;
    const BwdWs L = bwd_layout(w->rows, w->cols, n, r);
    if (ws_bytes < L.total) return QLN_ERR_WORKSPACE;
    int sms = 0;
    st = check_device(&sms);
    if (st != QLN_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    char *wsb = reinterpret_cast<char *>(ws);
    int *status = reinterpret_cast<int *>(wsb);
    uint16_t *G = reinterpret_cast<uint16_t *>(wsb + L.G);
    uint16_t *sG = reinterpret_cast<uint16_t *>(wsb + L.sG);
    float *pGU = reinterpret_cast<float *>(wsb + L.pGU);
    float *pA = reinterpret_cast<float *>(wsb + L.pA);
    float *pB = reinterpret_cast<float *>(wsb + L.pB);
    cudaError_t e;
    int *reset = status;  // the call's first kernel clears the status word
    if (!U) {
        uint16_t *Uw = reinterpret_cast<uint16_t *>(wsb + L.U);
        e = qln::launch_lora_down(X, n, w->cols, A, false, r, s, Uw, nullptr, pGU, cs, kSplitTargetSms, reset);
        if (e != cudaSuccess) return QLN_ERR_CUDA;
        U = Uw;
        reset = nullptr;
    }
    // G = dY B (and s*G; B read as stored, [dout][r]), dX = dY W' + (s G) A,
    // dA = s G^T X (the transpose of s X^T G), dB = s dY^T U.
    e = qln::launch_lora_down(dY, n, w->rows, B, true, r, s, G, sG, pGU, cs, kSplitTargetSms, reset);
    if (e != cudaSuccess) return QLN_ERR_CUDA;
    const int64_t gemm_ctas = qln::nf4_tc_gemm_ctas(w, true, n, r, sms);
    const int64_t idle = gemm_ctas > 0 && gemm_ctas < sms ? sms - gemm_ctas : 0;
    if (idle >= kSideMinCtas) {
        // the GEMM, then dA and dB on the SMs it leaves idle: launched on the
        // same stream as the GEMM's programmatic dependent, so the two overlap
        e = fused_gemm(w, true, dY, n, sG, A, r, dX, status, cs, sms);
        if (e != cudaSuccess) return QLN_ERR_CUDA;
        return from_cuda(qln::launch_tn_skinny_side(dY, U, w->rows, X, G, w->cols, n, r, s, dA, dB, (int)idle, cs));
    }
    e = fused_gemm(w, true, dY, n, sG, A, r, dX, status, cs, sms);
    if (e != cudaSuccess) return QLN_ERR_CUDA;
    e = qln::launch_tn_skinny(X, G, n, w->cols, r, s, true, dA, pA, L.splitA, cs);
    if (e != cudaSuccess) return QLN_ERR_CUDA;
    e = qln::launch_tn_skinny(dY, U, n, w->rows, r, s, false, dB, pB, L.splitB, cs);
    return from_cuda(e);
}

size_t qln_workspace_bytes(int32_t op, int64_t rows, int64_t cols, int64_t n, int32_t r) {
    switch (op) {
        case QLN_OP_DOUBLE_QUANT:
            return rows > 0 ? qln::dq_workspace_bytes(rows) : 0;
        case QLN_OP_LINEAR_FWD:
            return (rows > 0 && cols > 0 && n > 0 && r > 0) ? fwd_layout(rows, cols, n, r).total : 0;
        case QLN_OP_LINEAR_BWD:
            return (rows > 0 && cols > 0 && n > 0 && r > 0) ? bwd_layout(rows, cols, n, r).total : 0;
        case QLN_OP_QUANTIZE_DQ_BATCH:
            return (rows > 0 && rows <= kMaxBatchJobs) ? qln::kDqBatchScratchBytes * (size_t)rows : 0;
        default:
            return 0;
    }
}

void qln_codebook(float out16[16]) {
    for (int i = 0; i < 16; ++i) {
        uint32_t b = qln::nf4_bits(i);
        memcpy(&out16[i], &b, 4);
    }
}

const char *qln_status_str(qln_status st) {
    switch (st) {
        case QLN_OK: return "QLN_OK";
        case QLN_ERR_NULL: return "QLN_ERR_NULL";
        case QLN_ERR_SHAPE: return "QLN_ERR_SHAPE";
        case QLN_ERR_ALIGN: return "QLN_ERR_ALIGN";
        case QLN_ERR_WORKSPACE: return "QLN_ERR_WORKSPACE";
        case QLN_ERR_ARCH: return "QLN_ERR_ARCH";
        case QLN_ERR_CUDA: return "QLN_ERR_CUDA";
        case QLN_ERR_TIMEOUT: return "QLN_ERR_TIMEOUT";
        case QLN_ERR_INTERNAL: return "QLN_ERR_INTERNAL";
        default: return "QLN_ERR_UNKNOWN";
    }
}

int32_t qln_version(void) { return (1 << 16) | 0; }

uint64_t qln_launch_count(void) { return qln::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
