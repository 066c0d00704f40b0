// Encode side of libspectra: "tokens are projected down, quantised per token and
// appended to the latent cache" (SPECTRA technical summary, "SPECTRA pipeline",
// stage 3), with groups of adjacent latent coordinates sharing one width (stage 2,
// "grouping").
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device_common.cuh"
#include "kernels.h"

namespace spectra {

// ---------------------------------------------------------------------------
// latents[t][n] = sum_k H[t][k] * W_down[k][n]   for small T (decode steps).
// W_down is stored transposed (wt[n][k], bf16).  A warp owns CPW columns and
// streams their rows with 16-byte loads, KC/256 per column and lane in flight;
// each KC-wide slice of up to ROWS H rows is staged once per CTA in shared
// memory (loaded after the warp's W loads are issued, so the two overlap).
// bf16 x bf16 products are exact in fp32; accumulation is fp32.
// ---------------------------------------------------------------------------
namespace {

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float f[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
}  // namespace

template <int CPW, int ROWS, int KC>
__global__ void __launch_bounds__(256) project_gemv_kernel(const uint16_t* __restrict__ wt,
                                                           const uint16_t* __restrict__ H, int T,
                                                           int d_model, int n_eff,
                                                           float* __restrict__ C, int64_t ldc) {
  constexpr int BATCH = KC / 256;  // 16-byte chunks per column and lane per slice
  __shared__ __align__(16) uint16_t h_s[ROWS * KC];
  const int tid = threadIdx.x;
  const int warp = (blockIdx.x * blockDim.x + tid) >> 5;
  const int lane = tid & 31;
  const int n0 = warp * CPW;
  const bool active = n0 < n_eff;  // every warp stages H and meets the barriers
  pdl_launch_dependents();
  for (int t0 = 0; t0 < T; t0 += ROWS) {
    const int nr = min(ROWS, T - t0);
    float acc[CPW][ROWS];
#pragma unroll
    for (int c = 0; c < CPW; ++c)
#pragma unroll
      for (int r = 0; r < ROWS; ++r) acc[c][r] = 0.f;
    for (int kc0 = 0; kc0 < d_model; kc0 += KC) {
      uint4 wv[CPW][BATCH];
#pragma unroll
      for (int i = 0; i < BATCH; ++i)
#pragma unroll
        for (int c = 0; c < CPW; ++c) {
          const int k = kc0 + lane * 8 + 256 * i;
          const int n = min(n0 + c, n_eff - 1);
          wv[c][i] = (active && k < d_model)
                         ? __ldg(reinterpret_cast<const uint4*>(wt + (size_t)n * d_model + k))
                         : make_uint4(0u, 0u, 0u, 0u);
        }
      pdl_wait();       // H may come from the previous kernel; W_down is read-only codec data
      __syncthreads();  // the previous slice's readers are done
      for (int e = tid; e < ROWS * KC / 8; e += blockDim.x) {
        const int r = e / (KC / 8), col = (e % (KC / 8)) * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < nr && kc0 + col < d_model)
          v = __ldg(reinterpret_cast<const uint4*>(H + (size_t)(t0 + r) * d_model + kc0 + col));
        *reinterpret_cast<uint4*>(h_s + r * KC + col) = v;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < BATCH; ++i) {
        const int kl = lane * 8 + 256 * i;
        float w[CPW][8];
#pragma unroll
        for (int c = 0; c < CPW; ++c) bf16x8_to_f32(wv[c][i], w[c]);
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
          if (r < nr) {
            float h[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(h_s + r * KC + kl), h);
#pragma unroll
            for (int c = 0; c < CPW; ++c)
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[c][r] = fmaf(w[c][e], h[e], acc[c][r]);
          }
        }
      }
    }
#pragma unroll
    for (int c = 0; c < CPW; ++c)
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        float v = acc[c][r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && active && n0 + c < n_eff && r < nr) C[(size_t)(t0 + r) * ldc + n0 + c] = v;
      }
  }
}

// ---------------------------------------------------------------------------
// Append planner (one block): checks seq_ids are non-decreasing and in range,
// gives every token its cache position lengths[s] + (i - first index of s),
// checks capacity and page ids, and only if everything fits writes the positions,
// advances lengths and raises ok_flag.  Otherwise nothing is written and the
// codec's error word records SPECTRA_ERR_ORDER or SPECTRA_ERR_CAPACITY.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) append_plan_kernel(
    const int32_t* __restrict__ seq_ids, int T, int batch, int32_t* __restrict__ lengths,
    const int32_t* __restrict__ page_table, int max_pages, int64_t n_pool_pages, int P,
    int32_t* __restrict__ pos_out, int32_t* __restrict__ ok_flag, int32_t* __restrict__ err) {
  pdl_launch_dependents();
  pdl_wait();  // lengths, page table and seq_ids may come from earlier kernels
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < T; i += blockDim.x) {
    const int s = seq_ids[i];
    if (s < 0 || s >= batch || (i > 0 && seq_ids[i - 1] > s)) atomicMax(&bad, (int)SPECTRA_ERR_ORDER);
  }
  __syncthreads();
  if (bad == 0) {
    for (int i = threadIdx.x; i < T; i += blockDim.x) {
      const int s = seq_ids[i];
      int lo = 0, hi = i;  // first index with seq_ids[idx] == s (array is sorted)
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (seq_ids[mid] < s) lo = mid + 1;
        else hi = mid;
      }
      const int64_t pos = (int64_t)lengths[s] + (i - lo);
      if (pos < 0 || pos >= (int64_t)max_pages * P) {
        atomicMax(&bad, (int)SPECTRA_ERR_CAPACITY);
      } else {
        const int pid = page_table[(size_t)s * max_pages + pos / P];
        if (pid < 0 || pid >= n_pool_pages) atomicMax(&bad, (int)SPECTRA_ERR_CAPACITY);
      }
      pos_out[i] = (int32_t)pos;
    }
  }
  __syncthreads();
  if (bad == 0) {
    for (int i = threadIdx.x; i < T; i += blockDim.x)
      if (i == T - 1 || seq_ids[i + 1] != seq_ids[i]) lengths[seq_ids[i]] = pos_out[i] + 1;
  }
  if (threadIdx.x == 0) {
    *ok_flag = bad ? 0 : 1;
    if (bad) device_error(err, bad);
  }
}

// ---------------------------------------------------------------------------
// Quantise + pack + append.  Block (4 warps) = one chunk of 256/G input tokens
// for one (head, side); warps take the kept groups in turn.  For G = 16 a warp
// quantises two groups at once (lanes 0-15 and 16-31, one token per lane); for
// G = 8 one group with one token per lane.
//
// Per token and group (every step one IEEE fp32 operation, no contraction):
//   s = fp16(sat((max - min) / (2^b - 1))), z = fp16(sat(min)),
//   code = clamp(rint((x - z) / s), 0, 2^b - 1), s == 0 -> 0.
// Code bits go to the group's block at the canonical (word, bit) addresses of
// the page layout (fragment position of the entry, then the width rule); the
// token's bits are cleared then set with atomics, so tokens of one block written
// by different blocks of this grid (or by different calls) never race.
// ---------------------------------------------------------------------------
namespace {

__device__ __forceinline__ float sat16(float x) { return fminf(fmaxf(x, -65504.f), 65504.f); }

// Fragment position (gid, t4, slot) of entry (token tb of the block, coordinate k).
template <int G>
__device__ __forceinline__ void k_side_pos(int tb, int k, int* gid, int* t4, int* slot) {
  if (G == 16) {
    const int row = (tb & 1) ? 8 + (tb >> 1) : (tb >> 1);
    *slot = (row >> 3) + 2 * (k >> 3) + 4 * (k & 1);
    *gid = row & 7;
    *t4 = (k & 7) >> 1;
  } else {
    const int mi = tb >> 4, tl = tb & 15;
    const int row = (tl & 1) ? 8 + (tl >> 1) : (tl >> 1);
    *slot = (row >> 3) + 2 * mi + 4 * (k & 1);
    *gid = row & 7;
    *t4 = k >> 1;
  }
}

template <int G>
__device__ __forceinline__ void v_side_pos(int tb, int k, int* gid, int* t4, int* slot) {
  if (G == 16) {
    *slot = (k >> 3) + 2 * (tb >> 3) + 4 * (tb & 1);
    *gid = k & 7;
    *t4 = (tb & 7) >> 1;
  } else {
    const int mi = tb >> 4, tl = tb & 15;
    *slot = mi + 2 * (tl >> 3) + 4 * (tl & 1);
    *gid = k;
    *t4 = (tl & 7) >> 1;
  }
}

// Pending bits of one block word: consecutive entries that land in the same word
// are merged and written with one atomicAnd/atomicOr pair.
struct WordBits {
  int w;
  uint32_t mask, val;
};

__device__ __forceinline__ void flush_word(uint32_t* blk, WordBits& a) {
  if (a.w >= 0) {
    atomicAnd(blk + a.w, ~a.mask);
    atomicOr(blk + a.w, a.val);
  }
  a.w = -1;
  a.mask = a.val = 0u;
}

__device__ __forceinline__ void put_bits(uint32_t* blk, WordBits& a, int w, int shift, uint32_t width_mask,
                                         uint32_t v) {
  if (w != a.w) {
    flush_word(blk, a);
    a.w = w;
  }
  a.mask |= width_mask << shift;
  a.val |= (v & width_mask) << shift;
}

// Writes one code (width b) of fragment position (gid, t4, slot) into a block:
//   b = 4: word 4 gid + t4, nibble `slot`;
//   b = 2: word 2 gid + t4/2, bits 4 slot + 2 (t4 % 2) + {0, 1};
//   b = 1: word gid, bit 4 slot + t4;
//   b = 3: bits 0-1 as b = 2, bit 2 as b = 1 in words 16 + gid (second pending word);
//   b = 8: word 2 (4 gid + t4) + (slot / 2) % 2, byte (slot % 2) + 2 (slot / 4).
__device__ __forceinline__ void put_code(uint32_t* blk, WordBits& a, WordBits& a1, int b, int gid, int t4,
                                         int slot, uint32_t code) {
  switch (b) {
    case 4: put_bits(blk, a, 4 * gid + t4, 4 * slot, 0xFu, code); break;
    case 2: put_bits(blk, a, 2 * gid + (t4 >> 1), 4 * slot + 2 * (t4 & 1), 0x3u, code); break;
    case 1: put_bits(blk, a, gid, 4 * slot + t4, 0x1u, code); break;
    case 3:
      put_bits(blk, a, 2 * gid + (t4 >> 1), 4 * slot + 2 * (t4 & 1), 0x3u, code);
      put_bits(blk, a1, 16 + gid, 4 * slot + t4, 0x1u, code >> 2);
      break;
    default:
      put_bits(blk, a, 2 * (4 * gid + t4) + ((slot >> 1) & 1), 8 * ((slot & 1) + 2 * (slot >> 2)), 0xFFu, code);
      break;
  }
}

}  // namespace

template <int G>
__global__ void __launch_bounds__(128) quantize_append_kernel(
    const CodecDev* __restrict__ cd, const float* __restrict__ C, int64_t ldc,
    const int32_t* __restrict__ seq_ids, const int32_t* __restrict__ pos,
    const int32_t* __restrict__ ok_flag, int T, uint8_t* __restrict__ pool,
    const int32_t* __restrict__ page_table, int max_pages) {
  constexpr int TB = 256 / G;               // tokens per 256-bit block
  constexpr int LANES_PER_TOKENSET = TB;    // 16 or 32
  constexpr int GROUPS_PER_WARP = 32 / LANES_PER_TOKENSET;
  pdl_launch_dependents();
  pdl_wait();  // latents and the append plan come from the preceding kernels
  if (*ok_flag == 0) return;
  const int a = blockIdx.y >> 1, side = blockIdx.y & 1;
  const SideDev& sd = cd->head[a].side[side];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * TB + (lane % TB);
  if (i >= T) return;
  const int P = cd->P;
  const int p_tok = pos[i];
  const int seq = seq_ids[i];
  const int pid = page_table[(size_t)seq * max_pages + p_tok / P];
  uint8_t* page = pool + (size_t)pid * (size_t)cd->page_bytes;
  const int tau = p_tok % P;
  const int blk = tau / TB, tb = tau % TB;
  const float* crow = C + (size_t)i * ldc + sd.c_col0;
  const int n_groups = sd.n_groups;
  for (int j = warp * GROUPS_PER_WARP + lane / LANES_PER_TOKENSET; j < n_groups;
       j += 4 * GROUPS_PER_WARP) {
    const GroupDev gd = sd.grp[j];
    const int b = gd.b;
    float x[G];
#pragma unroll
    for (int q = 0; q < G / 4; ++q) {
      const float4 v = *reinterpret_cast<const float4*>(crow + gd.col + 4 * q);
      x[4 * q] = v.x;
      x[4 * q + 1] = v.y;
      x[4 * q + 2] = v.z;
      x[4 * q + 3] = v.w;
    }
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int k = 1; k < G; ++k) {
      mn = fminf(mn, x[k]);
      mx = fmaxf(mx, x[k]);
    }
    const float levels = (float)((1 << b) - 1);
    const __half s_h = __float2half_rn(sat16(__fdiv_rn(__fsub_rn(mx, mn), levels)));
    const __half z_h = __float2half_rn(sat16(mn));
    const float sf = __half2float(s_h), zf = __half2float(z_h);
    uint32_t code[G];
#pragma unroll
    for (int k = 0; k < G; ++k) {
      float c = 0.f;
      if (sf > 0.f) {
        const float t = __fdiv_rn(__fsub_rn(x[k], zf), sf);
        c = fminf(fmaxf(rintf(t), 0.f), levels);
      }
      code[k] = (uint32_t)c;
    }
    uint32_t* blkw = reinterpret_cast<uint32_t*>(page + gd.plane_off + blk * (32 * b));
    WordBits acc{-1, 0u, 0u}, acc1{-1, 0u, 0u};
#pragma unroll
    for (int k = 0; k < G; ++k) {
      int gid, t4, slot;
      if (side == 0) k_side_pos<G>(tb, k, &gid, &t4, &slot);
      else v_side_pos<G>(tb, k, &gid, &t4, &slot);
      put_code(blkw, acc, acc1, b, gid, t4, slot, code[k]);
    }
    flush_word(blkw, acc);
    flush_word(blkw, acc1);
    // record of the token pair u = tau/2: index (u % 8) * (P/16) + u / 8
    const int u = tau >> 1;
    __half* rec = reinterpret_cast<__half*>(page + gd.sz_off + 8 * ((u & 7) * (P >> 4) + (u >> 3)));
    rec[tau & 1] = s_h;
    rec[2 + (tau & 1)] = z_h;
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_project_gemv(const CodecDev& h, const uint16_t* wt, const uint16_t* H, int T,
                                float* C, int64_t ldc, cudaStream_t st) {
  // one column per warp for single-token steps (a whole 4096-wide row in flight
  // per warp); two columns per warp and 16 H rows per pass for larger batches
  if (T <= 1) {
    const int blocks = (h.n_eff * 32 + 255) / 256;
    return launch_dependent(project_gemv_kernel<1, 1, 4096>, dim3(blocks), dim3(256), 0, st, wt, H, T, h.d_model,
                            h.n_eff, C, ldc);
  } else {
    const int warps = (h.n_eff + 1) / 2;
    const int blocks = (warps * 32 + 255) / 256;
    return launch_dependent(project_gemv_kernel<2, 16, 1024>, dim3(blocks), dim3(256), 0, st, wt, H, T,
                            h.d_model, h.n_eff, C, ldc);
  }
}

cudaError_t launch_append_plan(const int32_t* seq_ids, int T, const spectra_cache& cache, int P,
                               int32_t* pos, int32_t* ok_flag, int32_t* err, cudaStream_t st) {
  return launch_dependent(append_plan_kernel, dim3(1), dim3(1024), 0, st, seq_ids, T, (int)cache.batch,
                          cache.lengths, cache.page_table, (int)cache.max_pages_per_seq, (int64_t)cache.n_pages, P,
                          pos, ok_flag, err);
}

cudaError_t launch_quantize_append(const CodecDev& h, const CodecDev* d, const float* C, int64_t ldc,
                                   const int32_t* seq_ids, const int32_t* pos, const int32_t* ok_flag,
                                   int T, const spectra_cache& cache, cudaStream_t st) {
  const int tb = 256 / h.group;
  dim3 grid((T + tb - 1) / tb, h.n_kv * 2);
  if (h.group == 16)
    return launch_dependent(quantize_append_kernel<16>, grid, dim3(128), 0, st, d, C, ldc, seq_ids, pos,
                            (const int32_t*)ok_flag, T, (uint8_t*)cache.pool, cache.page_table,
                            (int)cache.max_pages_per_seq);
  return launch_dependent(quantize_append_kernel<8>, grid, dim3(128), 0, st, d, C, ldc, seq_ids, pos,
                          (const int32_t*)ok_flag, T, (uint8_t*)cache.pool, cache.page_table,
                          (int)cache.max_pages_per_seq);
}

}  // namespace spectra
