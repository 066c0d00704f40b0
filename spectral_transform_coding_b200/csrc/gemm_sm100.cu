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
//
// encode_gemm_kernel is the same product for the prefill encode with the
// quantiser in its epilogue (the latents never reach memory); see its comment.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "device_common.cuh"
#include "kernels.h"
#include "pack_device.cuh"

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

// ---------------------------------------------------------------------------
// Prefill encode: latents = H W_down on the tensor cores with the quantiser and
// page writer in the epilogue ("SPECTRA pipeline" stage 3: tokens are projected
// down, quantised per token and appended).  No fp32 latents reach memory.
//
// Persistent CTAs (at most one per SM) walk the 128-token x 256-column output
// tiles, the column tile fastest, so the CTAs working at one time share each
// 128-token block of H in L2 (W_down stays resident there).  12 warps:
//   warp 0 (one lane): TMA producer of A/B k-blocks into a 4-stage ring;
//   warp 1 (one lane): tcgen05.mma issuer into one of two TMEM accumulators of
//     256 columns, so that the epilogue of tile i overlaps the main loop of
//     tile i + 1;
//   warps 4-11: epilogue.  Warp w reads TMEM lanes 32 (w % 4) .. + 31 (its
//     token rows) and column half (w - 4) / 4, one group of G columns at a time
//     (tcgen05.ld 32x32b: each thread holds one token's group), quantises it in
//     registers and writes codes and scale/zero record into the token's page.
//     A block of 256/G tokens that the lane set covers whole goes through a
//     256-byte shared buffer in fragment order, from which lanes assemble the
//     block's words and store them with 16-byte stores; partial blocks merge
//     their bits into the page with atomics (other tiles or calls may share
//     them).
// Groups never straddle a column tile: every head side's columns start at a
// multiple of G and BN is a multiple of G.  The accumulators are produced by
// the same MMA sequence as gemm_tcgen05_kernel's (same tile shape and k order),
// so the codes equal those of the projection followed by the quantise kernel.
// Positions come from the append plan, which runs first: if it rejected the
// append (flag 0) nothing is written.  Every wait is bounded; on a timeout the
// kernel records SPECTRA_ERR_TIMEOUT, stops issuing, waits for its copies and
// MMAs in flight and frees its TMEM.
// ---------------------------------------------------------------------------
constexpr int kEpiWarps = 8;
constexpr int kEncThreads = 32 * (4 + kEpiWarps);
constexpr uint32_t kEncTmemCols = 2 * BN;
constexpr int kWbufWords = kEpiWarps * 2 * 64;  // one 256-byte buffer per lane set (half-warp)
constexpr int ENC_SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/ + kWbufWords * 4;

__device__ __forceinline__ void mbar_arrive_one(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int G>
__device__ __forceinline__ void tmem_ld_group(uint32_t taddr, uint32_t (&r)[G]);

template <>
__device__ __forceinline__ void tmem_ld_group<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <>
__device__ __forceinline__ void tmem_ld_group<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <int G>
__global__ void __launch_bounds__(kEncThreads, 1) encode_gemm_kernel(
    const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
    const CodecDev* __restrict__ cd, int T, int n_eff, int K, const int32_t* __restrict__ seq_ids,
    const int32_t* __restrict__ pos, const int32_t* __restrict__ ok_flag, uint8_t* __restrict__ pool,
    const int32_t* __restrict__ page_table, int max_pages, int32_t* __restrict__ err) {
  constexpr int TB = 256 / G;  // tokens per packed block (16 or 32)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* fin = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* wbuf = reinterpret_cast<uint32_t*>(smem + STAGES * STAGE_BYTES + 256);
  __shared__ int abort_flag;

  // No early trigger: a decode launched next copies pages before its own
  // dependency wait, so it may start only once these writes are done.
  pdl_wait();  // H, seq_ids, the positions and the plan's flag come from earlier kernels
  if (*ok_flag == 0) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = (n_eff + BN - 1) / BN;
  const int n_tiles = nt * ((T + BM - 1) / BM);
  const int kblocks = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kEpiWarps);
    }
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kEncTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // producer
      uint32_t kc = 0;  // k-blocks issued by this CTA
      bool stop = false;
      for (int t = blockIdx.x; t < n_tiles && !stop; t += gridDim.x) {
        const int m0 = (t / nt) * BM, n0 = (t % nt) * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          const int s = (int)(kc % STAGES);
          if (kc >= (uint32_t)STAGES &&
              !mbar_wait_bounded(&empty[s], (kc / STAGES - 1) & 1u, kLimitNs)) {
            device_error(err, SPECTRA_ERR_TIMEOUT);
            atomicExch(&abort_flag, 1);
          }
          if (*(volatile int*)&abort_flag) {
            stop = true;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(sa, &map_a, kb * BK, m0, &full[s]);
          tma_load_2d(sa + A_BYTES, &map_b, kb * BK, n0, &full[s]);
          ++kc;
        }
      }
      // the last copy issued into each stage has landed before the CTA exits
      for (uint32_t s = 0; s < (uint32_t)STAGES && s < kc; ++s) {
        const uint32_t last = ((kc - 1 - s) / STAGES) * STAGES + s;
        if (!mbar_wait_bounded(&full[s], (last / STAGES) & 1u, kLimitNs)) device_error(err, SPECTRA_ERR_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer
      uint32_t kc = 0;
      int i = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < n_tiles && !stop; t += gridDim.x, ++i) {
        const int a = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        if (use >= 1 && !mbar_wait_bounded(&acc_empty[a], (use - 1) & 1u, kLimitNs)) {
          device_error(err, SPECTRA_ERR_TIMEOUT);
          atomicExch(&abort_flag, 1);
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t d = tmem + (uint32_t)(a * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++kc) {
          const int s = (int)(kc % STAGES);
          if (*(volatile int*)&abort_flag || !mbar_wait_bounded(&full[s], (kc / STAGES) & 1u, kLimitNs)) {
            if (!*(volatile int*)&abort_flag) device_error(err, SPECTRA_ERR_TIMEOUT);
            atomicExch(&abort_flag, 1);
            stop = true;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint8_t* sa = smem + s * STAGE_BYTES;
          const uint64_t da = smem_desc_sw128(sa), db = smem_desc_sw128(sa + A_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_f16(d, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (!stop) umma_commit(&acc_full[a]);
      }
      umma_commit(fin);  // arrives once every MMA issued has completed
      if (!mbar_wait_bounded(fin, 0, kLimitNs)) device_error(err, SPECTRA_ERR_TIMEOUT);
    }
  } else if (warp >= 4) {
    // epilogue
    const int q = warp & 3, ew = warp - 4, half = ew >> 2;
    const int P = cd->P;
    const int64_t pbytes = cd->page_bytes;
    const int32_t* __restrict__ colg = cd->col_groups;
    uint32_t* wb = wbuf + (ew * 2 + (lane / TB)) * 64;
    const int sub = lane % TB;
    const unsigned hm = TB == 16 ? (0xFFFFu << (16 * (lane >> 4))) : 0xFFFFFFFFu;
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int a = i & 1;
      const uint32_t use = (uint32_t)(i >> 1);
      const int m0 = (t / nt) * BM, n0 = (t % nt) * BN;
      // this thread's token (read before the accumulator is ready)
      const int r = m0 + 32 * q + lane;
      const bool valid = r < T;
      int tau = 0;
      uint8_t* page = pool;
      if (valid) {
        const int p = pos[r];
        const int pid = page_table[(size_t)seq_ids[r] * max_pages + p / P];
        page = pool + (size_t)pid * (size_t)pbytes;
        tau = p % P;
      }
      const int blk = tau / TB, tb = tau % TB;
      // the TB rows of this lane set fill one whole block: all present, one
      // sequence (so consecutive positions), the first at a block boundary
      const int i0 = m0 + 32 * q + (lane / TB) * TB;
      const bool whole = i0 + TB <= T && seq_ids[i0] == seq_ids[i0 + TB - 1] && pos[i0] % TB == 0;
      const bool ready = __all_sync(0xffffffffu, mbar_wait_bounded(&acc_full[a], use & 1u, kLimitNs));
      if (!ready) {
        if (lane == 0) device_error(err, SPECTRA_ERR_TIMEOUT);
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t tbase = tmem + (uint32_t)(a * BN + 128 * half) + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
      for (int j = 0; j < 128 / G; ++j) {
        const int c = n0 + 128 * half + G * j;
        if (c >= n_eff) break;
        __syncwarp();
        uint32_t rg[G];
        tmem_ld_group<G>(tbase + (uint32_t)(G * j), rg);
        const int4 gi = *reinterpret_cast<const int4*>(colg + 4 * (c / G));  // {b, plane_off, sz_off, side}
        const int b = gi.x;
        float x[G];
#pragma unroll
        for (int k = 0; k < G; ++k) x[k] = __uint_as_float(rg[k]);
        __half s_h, z_h;
        uint32_t code[G];
        pack::quantize_group<G>(x, b, s_h, z_h, code);
        uint32_t* blkw = reinterpret_cast<uint32_t*>(page + gi.y + blk * (32 * b));
        if (whole) {
          uint8_t* fb = reinterpret_cast<uint8_t*>(wb);
          pack::frag_bytes<G>(fb, gi.w, tb, code);
          __syncwarp(hm);
          if (sub < 2 * b) reinterpret_cast<uint4*>(blkw)[sub] = pack::block_words(fb, b, sub);
          __syncwarp(hm);  // before the next group reuses the buffer
        } else if (valid) {
          pack::put_codes<G, false>(blkw, gi.w, tb, b, code);
        }
        if (valid) pack::put_record(page + gi.z, P, tau, s_h, z_h);
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&acc_empty[a]);
    }
  }
  __syncwarp();  // the producer and MMA lanes rejoin their warps
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kEncTmemCols));
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

int sm_count_cached() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 1;
  }
  return n;
}

}  // namespace

cudaError_t launch_encode_gemm(const CodecDev& h, const CodecDev* d, const uint16_t* H, int T,
                               const int32_t* seq_ids, const int32_t* pos, const int32_t* ok_flag,
                               const spectra_cache& cache, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  if (((uintptr_t)H) % 16 || (h.d_model * 2) % 16 || (h.group != 8 && h.group != 16)) return cudaErrorNotSupported;
  CUtensorMap ma, mb;
  if (!make_map(&ma, H, T, h.d_model, h.d_model, BM) || !make_map(&mb, h.wt_down, h.n_eff, h.d_model, h.d_model, BN))
    return cudaErrorNotSupported;
  const auto kern = h.group == 16 ? encode_gemm_kernel<16> : encode_gemm_kernel<8>;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), ENC_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long tiles = (long)((h.n_eff + BN - 1) / BN) * ((T + BM - 1) / BM);
  const int grid = (int)std::min<long>(tiles, sm_count_cached());
  return launch_dependent(kern, dim3(grid), dim3(kEncThreads), ENC_SMEM_BYTES, st, ma, mb, d, T, h.n_eff, h.d_model,
                          seq_ids, pos, ok_flag, static_cast<uint8_t*>(cache.pool), cache.page_table,
                          (int)cache.max_pages_per_seq, h.err);
}

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
