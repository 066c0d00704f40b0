// tcgen05 (5th-generation tensor core) GEMM of libspectra:
//   C[M][N] (fp32) = A[M][K] . B[N][K]^T,  A and B bf16, both K-major.
// Used for the encode projection latents = H W_down ("SPECTRA pipeline",
// stage 3: tokens are projected down; A = H, B = W_down^T) and for the
// calibration Gram G = H^T H (stage 1, observation 3; A = B = H^T).
//
// Per CTA one 128 x BN output tile: warp 0 streams A/B k-blocks of 64 with TMA
// (128-byte swizzle, no multicast) into a ring of shared-memory stages; warp 1
// (one elected thread) issues tcgen05.mma kind::f16 into a TMEM accumulator and
// frees each stage with tcgen05.commit; then all four warps drain TMEM with
// tcgen05.ld and store fp32 rows.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "device_common.cuh"
#include "kernels.h"

namespace spectra {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;                   // one 128-byte swizzle atom of bf16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;     // 16 KB
constexpr int B_BYTES = BN * BK * 2;     // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint64_t kLimitNs = 2000ull * 1000ull * 1000ull;  // 2 s per wait

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor (tcgen05): K-major tile, 128-byte swizzle,
// rows of 128 bytes, 8-row core groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* p) {
  const uint32_t addr = smem_u32(p);
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);          // start address
  d |= (uint64_t)(16 >> 4) << 16;                  // leading byte offset (unused with swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset: 8 rows x 128 B
  d |= (uint64_t)1 << 46;                          // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                          // swizzle mode: 128B
  return d;
}

// Instruction descriptor: kind::f16, A = B = bf16, D = f32, K-major, M = 128, N = BN.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(kIdesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld_32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(128, 1) gemm_tcgen05_kernel(const __grid_constant__ CUtensorMap map_a,
                                                              const __grid_constant__ CUtensorMap map_b,
                                                              float* __restrict__ C, int64_t ldc, int M,
                                                              int N, int K, int32_t* __restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* done = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int kblocks = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // producer
    for (int kb = 0; kb < kblocks; ++kb) {
      const int s = kb % STAGES;
      if (kb >= STAGES) {
        if (!mbar_wait_bounded(&empty[s], (uint32_t)(((kb / STAGES) - 1) & 1), kLimitNs)) {
          device_error(err, SPECTRA_ERR_TIMEOUT);
          atomicExch(&abort_flag, 1);
          break;
        }
      }
      if (*(volatile int*)&abort_flag) break;
      uint8_t* sa = smem + s * STAGE_BYTES;
      uint8_t* sb = sa + A_BYTES;
      mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
      tma_load_2d(sa, &map_a, kb * BK, m0, &full[s]);
      tma_load_2d(sb, &map_b, kb * BK, n0, &full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    for (int kb = 0; kb < kblocks; ++kb) {
      const int s = kb % STAGES;
      if (!mbar_wait_bounded(&full[s], (uint32_t)((kb / STAGES) & 1), kLimitNs)) {
        device_error(err, SPECTRA_ERR_TIMEOUT);
        atomicExch(&abort_flag, 1);
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint8_t* sa = smem + s * STAGE_BYTES;
      const uint8_t* sb = sa + A_BYTES;
      const uint64_t da = smem_desc_sw128(sa), db = smem_desc_sw128(sb);
#pragma unroll
      for (int k = 0; k < BK / 16; ++k)  // +32 bytes per K step inside the swizzle atom
        umma_f16(tmem, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), (kb > 0 || k > 0) ? 1u : 0u);
      umma_commit(&empty[s]);
    }
    umma_commit(done);  // arrives once every issued MMA has completed
  }
  __syncwarp();

  // epilogue: TMEM lanes [32w, 32w+32) hold rows m0 + 32w + lane
  const bool have = __all_sync(0xffffffffu, mbar_wait_bounded(done, 0, kLimitNs));
  if (!have && lane == 0) device_error(err, SPECTRA_ERR_TIMEOUT);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const int row = m0 + warp * 32 + lane;
  if (have && !*(volatile int*)&abort_flag) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t r[32];
      tmem_ld_32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, r);
      if (row < M) {
        float* dst = C + (int64_t)row * ldc + n0 + c;
        if (n0 + c + 32 <= N && (((uintptr_t)dst) & 15) == 0) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + i) =
                make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                            __uint_as_float(r[i + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (n0 + c + i < N) dst[i] = __uint_as_float(r[i]);
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
}

// H[n][d] (bf16) -> Ht[d][ldt] (bf16), zero-padded to ldt columns.
__global__ void transpose_bf16_kernel(const uint16_t* __restrict__ H, int64_t n, int d, uint16_t* __restrict__ Ht,
                                      int64_t ldt) {
  __shared__ uint16_t tile[32][33];
  const int64_t t0 = (int64_t)blockIdx.x * 32;
  const int d0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int64_t t = t0 + i;
    const int dd = d0 + threadIdx.x;
    tile[i][threadIdx.x] = (t < n && dd < d) ? H[t * d + dd] : (uint16_t)0;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int dd = d0 + i;
    const int64_t t = t0 + threadIdx.x;
    if (dd < d && t < ldt) Ht[(int64_t)dd * ldt + t] = tile[threadIdx.x][i];
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows][cols] (cols contiguous, row pitch ld elements), box
// {64 cols, box_rows rows}, 128-byte swizzle, out-of-range reads return zero.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t gemm_tn(const uint16_t* A, int64_t lda, const uint16_t* B, int64_t ldb, float* C, int64_t ldc, int M,
                    int N, int K, int32_t* err, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0) return cudaSuccess;
  if ((lda * 2) % 16 || (ldb * 2) % 16 || ((uintptr_t)A) % 16 || ((uintptr_t)B) % 16) return cudaErrorNotSupported;
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, M, K, lda, BM) || !make_map(&mb, B, N, K, ldb, BN)) return cudaErrorNotSupported;
  {
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(gemm_tcgen05_kernel), SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  gemm_tcgen05_kernel<<<grid, 128, SMEM_BYTES, st>>>(ma, mb, C, ldc, M, N, K, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_project_tcgen05(const CodecDev& h, const uint16_t* wt, const uint16_t* H, int T, float* C,
                                   int64_t ldc, cudaStream_t st) {
  // rows of W_down^T beyond n_eff are zero padding; only n_eff columns are stored
  return gemm_tn(H, h.d_model, wt, h.d_model, C, ldc, T, h.n_eff, h.d_model, h.err, st);
}

cudaError_t launch_gram_tcgen05(const uint16_t* H, int64_t n_tokens, int d_model, float* G, cudaStream_t st) {
  // G = (H^T)(H^T)^T with H^T [d_model][n_pad] K-major
  const int64_t n_pad = (n_tokens + 7) / 8 * 8;
  if (n_pad > ((int64_t)1 << 31)) return cudaErrorNotSupported;
  uint16_t* Ht = nullptr;
  cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&Ht), (size_t)d_model * n_pad * 2, st);
  if (e != cudaSuccess) return e;
  const dim3 tgrid((unsigned)((n_pad + 31) / 32), (unsigned)((d_model + 31) / 32));
  transpose_bf16_kernel<<<tgrid, dim3(32, 8), 0, st>>>(H, n_tokens, d_model, Ht, n_pad);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = gemm_tn(Ht, n_pad, Ht, n_pad, G, d_model, d_model, d_model, (int)n_pad, nullptr, st);
  cudaError_t e2 = cudaFreeAsync(Ht, st);
  return e != cudaSuccess ? e : e2;
}

}  // namespace spectra
