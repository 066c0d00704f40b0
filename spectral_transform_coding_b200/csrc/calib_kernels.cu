// Calibration-side kernels of libspectra (once per layer, off the hot path):
// fp32 GEMMs for W^T G W and W V_r ("SPECTRA pipeline", stage 1), an fp32 Gram
// for fp32 inputs, causal attention for the W_O refinement, a finiteness check.
#include <cuda_bf16.h>
#include <math_constants.h>

#include <algorithm>

#include "device_common.cuh"
#include "kernels.h"

namespace spectra {

namespace {

template <bool BF16>
__device__ __forceinline__ float ld(const void* p, int64_t i) {
  if (BF16) return __uint_as_float((uint32_t)(reinterpret_cast<const uint16_t*>(p)[i]) << 16);
  return reinterpret_cast<const float*>(p)[i];
}

constexpr int BM = 64, BN = 64, BK = 16;

// C[M][N] = sum_k opA(k, m) * B[k][n]; opA = A[k][m] (TRANS) or A[m][k].
// 256 threads, 4x4 outputs each, fp32 accumulate.
template <bool TRANS_A, bool A_BF16, bool B_BF16>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const void* __restrict__ A, int64_t lda,
                                                       const void* __restrict__ B, int64_t ldb,
                                                       float* __restrict__ C, int64_t ldc, int M,
                                                       int N, int K) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int e = threadIdx.x; e < BK * BM; e += 256) {
      const int kk = e / BM, mm = e % BM;
      const int gk = k0 + kk, gm = m0 + mm;
      float v = 0.f;
      if (gk < K && gm < M) v = TRANS_A ? ld<A_BF16>(A, (int64_t)gk * lda + gm) : ld<A_BF16>(A, (int64_t)gm * lda + gk);
      As[kk][mm] = v;
    }
    for (int e = threadIdx.x; e < BK * BN; e += 256) {
      const int kk = e / BN, nn = e % BN;
      const int gk = k0 + kk, gn = n0 + nn;
      Bs[kk][nn] = (gk < K && gn < N) ? ld<B_BF16>(B, (int64_t)gk * ldb + gn) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i) b[i] = Bs[kk][tx * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gm = m0 + ty * 4 + i, gn = n0 + tx * 4 + j;
      if (gm < M && gn < N) C[(int64_t)gm * ldc + gn] = acc[i][j];
    }
}

template <bool TRANS_A>
cudaError_t gemm_dispatch(const void* A, bool a_bf16, int64_t lda, const void* B, bool b_bf16,
                          int64_t ldb, float* C, int64_t ldc, int M, int N, int K, cudaStream_t st) {
  const dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  if (a_bf16 && b_bf16)
    gemm_f32_kernel<TRANS_A, true, true><<<grid, 256, 0, st>>>(A, lda, B, ldb, C, ldc, M, N, K);
  else if (a_bf16)
    gemm_f32_kernel<TRANS_A, true, false><<<grid, 256, 0, st>>>(A, lda, B, ldb, C, ldc, M, N, K);
  else if (b_bf16)
    gemm_f32_kernel<TRANS_A, false, true><<<grid, 256, 0, st>>>(A, lda, B, ldb, C, ldc, M, N, K);
  else
    gemm_f32_kernel<TRANS_A, false, false><<<grid, 256, 0, st>>>(A, lda, B, ldb, C, ldc, M, N, K);
  return cudaGetLastError();
}

// One block per query row: scores against keys 0..i (width dk), softmax,
// weighted values (width dv).
__global__ void __launch_bounds__(256) causal_attention_kernel(const float* __restrict__ Q,
                                                               const float* __restrict__ K,
                                                               const float* __restrict__ V,
                                                               float* __restrict__ O, int n, int dk,
                                                               int dv, int64_t ldq, int64_t ldk,
                                                               int64_t ldv, int64_t ldo) {
  extern __shared__ float sh[];
  float* q = sh;          // [dk]
  float* s = sh + dk;     // [n]
  __shared__ float red[32];
  const int i = blockIdx.x;
  for (int e = threadIdx.x; e < dk; e += blockDim.x) q[e] = Q[(int64_t)i * ldq + e];
  __syncthreads();
  const float scale = rsqrtf((float)dk);
  float mx = -CUDART_INF_F;
  for (int j = threadIdx.x; j <= i; j += blockDim.x) {
    float acc = 0.f;
    for (int e = 0; e < dk; ++e) acc = fmaf(q[e], K[(int64_t)j * ldk + e], acc);
    s[j] = acc * scale;
    mx = fmaxf(mx, s[j]);
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = -CUDART_INF_F;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
    red[31] = m;
  }
  __syncthreads();
  const float m = red[31];
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j <= i; j += blockDim.x) {
    s[j] = expf(s[j] - m);
    sum += s[j];
  }
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    red[30] = t;
  }
  __syncthreads();
  const float inv = 1.f / red[30];
  for (int e = threadIdx.x; e < dv; e += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j <= i; ++j) acc = fmaf(s[j], V[(int64_t)j * ldv + e], acc);
    O[(int64_t)i * ldo + e] = acc * inv;
  }
}

template <bool BF16>
__global__ void check_finite_kernel(const void* __restrict__ X, int64_t n, int32_t* flag) {
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    bad |= !isfinite(ld<BF16>(X, i));
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicExch(flag, 1);
}

}  // namespace

cudaError_t launch_gemm_tn_f32(const void* A, bool a_bf16, int64_t lda, const void* B, bool b_bf16,
                               int64_t ldb, float* C, int64_t ldc, int M, int N, int K,
                               cudaStream_t st) {
  return gemm_dispatch<true>(A, a_bf16, lda, B, b_bf16, ldb, C, ldc, M, N, K, st);
}

cudaError_t launch_gemm_nn_f32(const void* A, bool a_bf16, int64_t lda, const void* B, bool b_bf16,
                               int64_t ldb, float* C, int64_t ldc, int M, int N, int K,
                               cudaStream_t st) {
  return gemm_dispatch<false>(A, a_bf16, lda, B, b_bf16, ldb, C, ldc, M, N, K, st);
}

cudaError_t launch_gram_f32(const float* H, int64_t n_tokens, int d_model, float* G, cudaStream_t st) {
  return gemm_dispatch<true>(H, false, d_model, H, false, d_model, G, d_model, d_model, d_model,
                             (int)n_tokens, st);
}

cudaError_t launch_causal_attention(const float* Q, const float* K, const float* V, float* O, int n,
                                    int dk, int dv, int64_t ldq, int64_t ldk, int64_t ldv, int64_t ldo,
                                    cudaStream_t st) {
  const int smem = (dk + n) * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(causal_attention_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  causal_attention_kernel<<<n, 256, smem, st>>>(Q, K, V, O, n, dk, dv, ldq, ldk, ldv, ldo);
  return cudaGetLastError();
}

cudaError_t launch_check_finite(const void* X, bool bf16, int64_t n, int32_t* flag, cudaStream_t st) {
  const int blocks = (int)std::min<int64_t>(1024, (n + 255) / 256 + 1);
  if (bf16) check_finite_kernel<true><<<blocks, 256, 0, st>>>(X, n, flag);
  else check_finite_kernel<false><<<blocks, 256, 0, st>>>(X, n, flag);
  return cudaGetLastError();
}

}  // namespace spectra
