// Kernel launchers of libspectra (internal).
#pragma once

#include <cuda_runtime.h>

#include "spectra_internal.h"

namespace spectra {

// Launch with programmatic stream serialisation (see pdl_wait in
// device_common.cuh); if the attribute is refused, launch plainly.
template <typename... Args>
cudaError_t launch_dependent(void (*kern)(Args...), dim3 grid, dim3 block, int smem, cudaStream_t st, Args... args) {
  static bool pdl_ok = true;
  if (pdl_ok) {
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e == cudaSuccess) return e;
    (void)cudaGetLastError();
    pdl_ok = false;
  }
  kern<<<grid, block, smem, st>>>(args...);
  return cudaGetLastError();
}

// As launch_dependent, in thread-block clusters of `cluster` CTAs; returns the
// launch error (the caller falls back to a launch without clusters).
template <typename... Args>
cudaError_t launch_dependent_cluster(void (*kern)(Args...), dim3 grid, dim3 block, int smem, cudaStream_t st,
                                     dim3 cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster.x;
  attr[0].val.clusterDim.y = cluster.y;
  attr[0].val.clusterDim.z = cluster.z;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e == cudaSuccess) return e;
  (void)cudaGetLastError();
  cfg.numAttrs = 1;  // without programmatic serialisation
  e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) (void)cudaGetLastError();
  return e;
}

// encode_kernels.cu
cudaError_t launch_project_gemv(const CodecDev& h, const uint16_t* wt, const uint16_t* H, int T,
                                float* C, int64_t ldc, cudaStream_t st);
cudaError_t launch_append_plan(const int32_t* seq_ids, int T, const spectra_cache& cache, int P,
                               int32_t* pos, int32_t* ok_flag, int32_t* err, cudaStream_t st);
cudaError_t launch_quantize_append(const CodecDev& h, const CodecDev* d, const float* C, int64_t ldc,
                                   const int32_t* seq_ids, const int32_t* pos, const int32_t* ok_flag,
                                   int T, const spectra_cache& cache, cudaStream_t st);

// Fused encode for decode steps: projection (split over d_model chunks),
// quantisation and packing in one kernel; a group's partial sums meet in one
// CTA, which packs the group; the last CTA to hold its positions advances the
// lengths.
constexpr int kFusedMaxT = 16;
// Decode-step encode plan: kept groups; d_model chunks of 256 * batch columns,
// cpc consecutive chunks per CTA, n_part CTAs per group; token count rounded up
// to a power of two.
struct EncodeFusedPlan {
  int n_groups, n_chunks, batch, cpc, n_part, tp;
  int staged, smem_bytes;  // chunks after a CTA's first staged in shared memory (bytes per CTA)
  int cluster;             // the n_part CTAs of a group form one thread-block cluster
};
constexpr int kMaxFusedGroups = kMaxKV * 2 * kMaxGroups;
// What the fused encode reads of the codec, passed by value so that its first
// W_down loads depend on no global load.
struct EncodeFusedArgs {
  const uint16_t* wt_down;
  const int32_t* col_groups;  // per kept group {width, block offset, record offset, side}
  int32_t* err;
  int64_t page_bytes;
  unsigned long long wait_ns;  // limit of the wait for staged W_down copies
  int d_model, n_eff, P;
  int staged;      // chunks after a CTA's first are bulk-copied into shared memory
  int cluster;     // the CTAs of a group form one cluster and add their partial sums in shared memory
  int drop_stage;  // test hook: CTA (0, 0) never issues its first staged copy (its wait then gives up)
};
EncodeFusedPlan encode_fused_plan(const CodecDev& h, int T);
// Workspace bytes of the fused encode's partial sums for T tokens.
size_t encode_fused_partial_bytes(const CodecDev& h, int T);
// counters: int32 [1 + kMaxFusedGroups], zero between calls; part: partial sums.
cudaError_t launch_encode_fused(const CodecDev& h, const CodecDev* d, const uint16_t* H, const int32_t* seq_ids,
                                int T, const spectra_cache& cache, float* latents_out, int32_t* counters,
                                float* part, cudaStream_t st);

// reconstruct_kernels.cu: k^ = (code s + z) W_up^K, v^ likewise, for tokens
// [t0, t0 + n) of sequence b; out of range or bad page ids -> device error INVALID
cudaError_t launch_reconstruct(const CodecDev& h, const CodecDev* d, const spectra_cache& cache, int b, int64_t t0,
                               int64_t n, float* K_out, float* V_out, cudaStream_t st);

// Reconstruct-then-attend decode (keys rebuilt per tile, optional rotary
// position embedding, V summed in the latent space and lifted once per head).
constexpr int kRtMaxDHead = 128;
struct RtPlan {
  int n_split;      // context splits per (KV head, sequence)
  int part_stride;  // floats per partial record
  int smem_bytes;   // dynamic shared memory of the split kernel
  size_t ws_bytes;  // workspace: the partial records
};
// upper_bound: size for any call on any device (the workspace query)
RtPlan make_rt_plan(const CodecDev& h, int batch, int max_pages_per_seq, bool upper_bound = false);
bool rt_supported(const CodecDev& h, std::string* why);
cudaError_t launch_decode_reconstruct(const CodecDev& h, const CodecDev* d, const spectra_cache& cache,
                                      const float* q, double theta, float* out, void* ws, const RtPlan& plan,
                                      cudaStream_t st);

// decode_kernels.cu
// Raises `kern`'s dynamic shared-memory limit on the current device to at least
// `bytes` (one record per kernel and device; the limit never shrinks).
cudaError_t ensure_dynamic_smem(const void* kern, int bytes);
struct DecodePlan {
  int n_split;       // context splits per (sequence, KV head)
  int cl;            // CTAs per thread-block cluster (1: no clusters)
  int slice_k;       // K coordinates folded per CTA
  int slice_v;       // V coordinates lifted by the last CTA
  int wv_staged;     // the last CTA bulk-copies W_up^V into its stage ring
  int stages;        // page stages of the CTA's ring
  int stage_bytes;   // bytes per stage (largest head section, rounded to 16)
  int off_stages;    // shared-memory offset of the ring
  int smem_bytes;    // dynamic shared memory per CTA
  int rec_stride;    // floats per cluster record of one q head
  size_t cnt_off, rec_off, ws_bytes;  // workspace: arrival counters (zero between calls), split records
};
DecodePlan make_decode_plan(const CodecDev& h, int batch, int max_pages_per_seq);
cudaError_t launch_decode(const CodecDev& h, const CodecDev* d, const spectra_cache& cache,
                          const float* q, float* out, void* ws, const DecodePlan& plan,
                          cudaStream_t st);

// gemm_sm100.cu (tcgen05)
// Prefill encode: projection GEMM with quantise/pack/append in its epilogue;
// positions and the plan's flag from launch_append_plan (launched before it).
cudaError_t launch_encode_gemm(const CodecDev& h, const CodecDev* d, const uint16_t* H, int T,
                               const int32_t* seq_ids, const int32_t* pos, const int32_t* ok_flag,
                               const spectra_cache& cache, cudaStream_t st);
cudaError_t launch_project_tcgen05(const CodecDev& h, const uint16_t* wt, const uint16_t* H, int T,
                                   float* C, int64_t ldc, cudaStream_t st);
cudaError_t launch_gram_tcgen05(const uint16_t* H, int64_t n_tokens, int d_model, float* G,
                                cudaStream_t st);

// calib_kernels.cu
cudaError_t launch_gram_f32(const float* H, int64_t n_tokens, int d_model, float* G, cudaStream_t st);
// C[M][N] = sum_k A[k][m] * B[k][n] (A^T B), A and B row-major with leading dims lda, ldb;
// `a_bf16`/`b_bf16` select bf16 inputs (else fp32).  fp32 accumulate.
cudaError_t launch_gemm_tn_f32(const void* A, bool a_bf16, int64_t lda, const void* B, bool b_bf16,
                               int64_t ldb, float* C, int64_t ldc, int M, int N, int K,
                               cudaStream_t st);
// C[M][N] = A[M][K] B[K][N], row-major, fp32 (A, B may be bf16).
cudaError_t launch_gemm_nn_f32(const void* A, bool a_bf16, int64_t lda, const void* B, bool b_bf16,
                               int64_t ldb, float* C, int64_t ldc, int M, int N, int K,
                               cudaStream_t st);
cudaError_t launch_causal_attention(const float* Q, const float* K, const float* V, float* O,
                                    int n, int dk, int dv, int64_t ldq, int64_t ldk, int64_t ldv,
                                    int64_t ldo, cudaStream_t st);
cudaError_t launch_check_finite(const void* X, bool bf16, int64_t n, int32_t* flag, cudaStream_t st);

}  // namespace spectra
