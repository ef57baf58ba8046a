// Internal launchers of libqlora_nf4 (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/qlora_nf4.h"

namespace qln {

// Host-side count of kernels enqueued by this library (qln_launch_count).
void note_launch();

// Launch `kernel` with the programmatic stream-serialization attribute (the
// kernel must call pdl_wait() before touching global memory that earlier
// kernels on the stream read or write).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    note_launch();
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// codec.cu
cudaError_t launch_nf4_quantize(const void *W, int dtype, int64_t numel, uint8_t *codes, float *absmax,
                                cudaStream_t st, int num_sms);
cudaError_t launch_nf4_double_quant(const float *absmax, int64_t nb, int8_t *qabs, float *scale, float *mu,
                                    void *ws, bool e4m3, cudaStream_t st, int num_sms);
cudaError_t launch_nf4_quantize_dq(const void *W, int dtype, int64_t numel, uint8_t *codes, float *absmax,
                                   int8_t *qabs, float *scale, float *mu, void *ws, bool e4m3, cudaStream_t st,
                                   int num_sms);
// One weight of a quantize + double quantization batch (validated by the caller).
struct QuantJob {
    const void *W;
    int dtype;
    int64_t numel;
    uint8_t *codes;
    float *absmax;
    int8_t *qabs;
    float *scale;
    float *mu;
    bool e4m3;
};
cudaError_t launch_nf4_quantize_dq_batch(const QuantJob *jobs, int njobs, void *ws, cudaStream_t st, int num_sms);
constexpr size_t kDqBatchScratchBytes = 256;  // per job
cudaError_t launch_nf4_dequant(const qln_nf4_weight *w, uint16_t *out, cudaStream_t st, int num_sms);
cudaError_t launch_adamw(float *p, const float *g, float *m, float *v, uint16_t *p_bf16, int64_t n, float lr,
                         float b1, float b2, float eps, float wd, const int64_t *step, int flags, cudaStream_t st,
                         int num_sms);
cudaError_t launch_nf4_dequant_flat(const qln_nf4_weight *w, int64_t numel, uint16_t *out, cudaStream_t st,
                                    int num_sms);
size_t dq_workspace_bytes(int64_t nb);
// allocation-free variant: scratch in a file-scope device array (codec.cu)
cudaError_t launch_nf4_double_quant_static(const float *absmax, int64_t nb, int8_t *qabs, float *scale, float *mu,
                                           cudaStream_t st, int num_sms);
int64_t dq_static_max_blocks();
int64_t dq_max_blocks();

// lora_small.cu: skinny products around the adapters.
//   out[t][j] = bf16(sum_k in[t][k] * wt[j][k]) and, if out_scaled != NULL,
//   out_scaled[t][j] = bf16(scale * that sum); wt is [r][K] row-major.
//   `partial` is fp32 scratch of lora_down_partial_bytes(n, K, r, num_sms).
//   wt_kmajor: wt is stored [K][r] instead (out[t][j] = sum_k in[t][k] * wt[k][j]).
cudaError_t launch_lora_down(const uint16_t *in, int64_t n, int64_t K, const uint16_t *wt, bool wt_kmajor, int r,
                             float scale, uint16_t *out, uint16_t *out_scaled, float *partial, cudaStream_t st,
                             int num_sms, int *status_reset = nullptr);
size_t lora_down_partial_bytes(int64_t n, int64_t K, int r, int num_sms);
//   C = scale * P^T Q with Q [n][R] narrow (R <= 128): C[m][j], or C[j][m] with
//   `transpose`; fp32 partials of tn_skinny_partials_bytes(M, R, splits).
cudaError_t launch_tn_skinny(const uint16_t *P, const uint16_t *Q, int64_t n, int64_t M, int R, float scale,
                             bool transpose, float *C, float *partials, int splits, cudaStream_t st);
size_t tn_skinny_partials_bytes(int64_t M, int R, int splits);
// dA and dB as one persistent launch of `nside` CTAs (for SMs a concurrent
// kernel leaves idle); no partials.
cudaError_t launch_tn_skinny_side(const uint16_t *dY, const uint16_t *U, int64_t dout, const uint16_t *X,
                                  const uint16_t *G, int64_t din, int64_t n, int R, float scale, float *dA, float *dB,
                                  int nside, cudaStream_t st);
// CTAs the tcgen05 GEMM launches for this call (0 when it does not take the call).
int64_t nf4_tc_gemm_ctas(const qln_nf4_weight *w, bool trans, int64_t n, int r, int num_sms);
int tn_skinny_splits(int64_t n, int64_t M, int R, int num_sms);

// nf4_gemm_sm80.cu: fused NF4 decode + legacy mma.sync GEMM (small n).
//   trans = false: out[t][m] = bf16(sum_k act[t][k] W'[m][k] + sum_j lact[t][j] lw[m][j])   (forward)
//   trans = true : out[t][m] = bf16(sum_k act[t][k] W'[k][m] + sum_j lact[t][j] lw[j][m])   (dX)
cudaError_t launch_nf4_mma_gemm(const qln_nf4_weight *w, bool trans, const uint16_t *act, int64_t n,
                                const uint16_t *lact, const uint16_t *lw, int r, uint16_t *out,
                                int *status, cudaStream_t st, int num_sms);

// 2D tiled TMA descriptor over a row-major [outer][inner] array (nf4_gemm_sm100.cu).
bool make_tensor_map_2d(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, uint64_t inner,
                        uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);

// Workspace header of the linear calls: the int32 device status word at byte 0.
constexpr int kWsHeaderBytes = 256;

// nf4_decode.cu: the whole forward for decode-sized n (<= 32) in one launch of
// thread-block clusters: U = X A^T, Y = bf16(X W'^T + bf16(s U) B^T),
// U_out = bf16(U) (if not null).  Needs no workspace beyond the status word.
bool nf4_decode_fwd_supported(const qln_nf4_weight *w, int64_t n, int r);
cudaError_t launch_nf4_decode_fwd(const qln_nf4_weight *w, const uint16_t *X, int64_t n, const uint16_t *A,
                                  const uint16_t *B, int r, float s, uint16_t *Y, uint16_t *U_out, int *status,
                                  cudaStream_t st);

// nf4_gemm_sm100.cu: fused NF4 decode + tcgen05 GEMM (TMA, TMEM accumulators).
cudaError_t launch_nf4_tc_gemm(const qln_nf4_weight *w, bool trans, const uint16_t *act, int64_t n,
                               const uint16_t *lact, const uint16_t *lw, int r, uint16_t *out,
                               int *status, cudaStream_t st, int num_sms);
bool nf4_tc_gemm_supported(const qln_nf4_weight *w, bool trans, int64_t n, int r);

}  // namespace qln
