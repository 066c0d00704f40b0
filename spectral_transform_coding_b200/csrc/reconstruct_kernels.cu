// Reconstruction of cached keys and values: "SPECTRA: Pushing the KV Cache
// Beyond the 2-Bit Cliff via Spectral Transform Coding", technical summary,
// "SPECTRA pipeline" stage 3 (the latents are dequantised and lifted back with
// W_up to keys and values for standard attention).
//
//   c^ = code * s + z   (per token and kept group; zero-width groups are 0)
//   k^ = c^_K W_up^K,   v^ = c^_V W_up^V
//
// One CTA per (16 tokens, KV head, side): the codes are read from the page's
// code blocks through the canonical (word, bit) addresses, dequantised in fp32
// into shared memory, then multiplied by W_up (fp32 accumulation).
#include <cuda_fp16.h>

#include "device_common.cuh"
#include "kernels.h"

namespace spectra {

namespace {

constexpr int kRecTokens = 16;
constexpr int kMaxKeptRec = kMaxDHead;  // kept coordinates per side <= rank <= d_head

// Fragment position of entry (token tb of the block, coordinate k); the same
// rule the encoder packs with (see the page layout in include/spectra.h).
__device__ __forceinline__ void frag_pos(int G, int side, int tb, int k, int* gid, int* t4, int* slot) {
  if (G == 16) {
    int row, col;
    if (side == 0) {
      row = (tb & 1) ? 8 + (tb >> 1) : (tb >> 1);
      col = k;
    } else {
      row = k;
      col = tb;
    }
    *gid = row & 7;
    *t4 = (col & 7) >> 1;
    *slot = (row >> 3) + 2 * (col >> 3) + 4 * (col & 1);
  } else {
    const int mi = tb >> 4, tl = tb & 15;
    if (side == 0) {
      const int row = (tl & 1) ? 8 + (tl >> 1) : (tl >> 1);
      *gid = row & 7;
      *t4 = k >> 1;
      *slot = (row >> 3) + 2 * mi + 4 * (k & 1);
    } else {
      *gid = k;
      *t4 = (tl & 7) >> 1;
      *slot = mi + 2 * (tl >> 3) + 4 * (tl & 1);
    }
  }
}

// Code of fragment position (gid, t4, slot) in a block of width b.
__device__ __forceinline__ uint32_t read_code(const uint32_t* __restrict__ blk, int b, int gid, int t4, int slot) {
  switch (b) {
    case 4: return (blk[4 * gid + t4] >> (4 * slot)) & 0xFu;
    case 2: return (blk[2 * gid + (t4 >> 1)] >> (4 * slot + 2 * (t4 & 1))) & 0x3u;
    case 1: return (blk[gid] >> (4 * slot + t4)) & 0x1u;
    case 3:
      return ((blk[2 * gid + (t4 >> 1)] >> (4 * slot + 2 * (t4 & 1))) & 0x3u) |
             (((blk[16 + gid] >> (4 * slot + t4)) & 0x1u) << 2);
    default:
      return (blk[2 * (4 * gid + t4) + ((slot >> 1) & 1)] >> (8 * ((slot & 1) + 2 * (slot >> 2)))) & 0xFFu;
  }
}

__global__ void __launch_bounds__(128) reconstruct_kernel(const CodecDev* __restrict__ cd, const uint8_t* __restrict__ pool,
                                                          const int32_t* __restrict__ page_table,
                                                          const int32_t* __restrict__ lengths, int64_t n_pool_pages,
                                                          int max_pages, int b, int64_t t0, int64_t n,
                                                          float* __restrict__ K_out, float* __restrict__ V_out) {
  __shared__ float lat[kRecTokens][kMaxKeptRec];
  const int a = blockIdx.y, side = blockIdx.z;
  const int64_t tok0 = t0 + (int64_t)blockIdx.x * kRecTokens;
  const int64_t left = t0 + n - tok0;
  const int nt = left < kRecTokens ? (int)left : kRecTokens;
  const SideDev& sd = cd->head[a].side[side];
  const int G = cd->group, P = cd->P, d_h = cd->d_h, nk = sd.n_kept, n_kv = cd->n_kv;
  const int TB = 256 / G;
  const int len = lengths[b];
  // range and page checks (the same verdict in every CTA)
  bool bad = t0 < 0 || t0 + n > len;
  for (int t = 0; t < nt && !bad; ++t) {
    const int64_t pos = tok0 + t;
    const int pid = page_table[(size_t)b * max_pages + pos / P];
    bad = pid < 0 || (int64_t)pid >= n_pool_pages;
  }
  float* out = side == 0 ? K_out : V_out;
  if (bad) {
    if (threadIdx.x == 0) device_error(cd->err, SPECTRA_ERR_INVALID);
    return;
  }
  // dequantised latents of this CTA's tokens
  for (int e = threadIdx.x; e < nt * nk; e += blockDim.x) {
    const int t = e / nk, c = e % nk;
    const int j = c / G, k = c % G;
    const GroupDev gd = sd.grp[j];
    const int64_t pos = tok0 + t;
    const int pid = page_table[(size_t)b * max_pages + pos / P];
    const uint8_t* page = pool + (size_t)pid * (size_t)cd->page_bytes;
    const int tau = (int)(pos % P);
    int gid, t4, slot;
    frag_pos(G, side, tau % TB, k, &gid, &t4, &slot);
    const uint32_t* blk = reinterpret_cast<const uint32_t*>(page + gd.plane_off + (tau / TB) * (32 * gd.b));
    const uint32_t code = read_code(blk, gd.b, gid, t4, slot);
    const int u = tau >> 1;
    const __half* rec = reinterpret_cast<const __half*>(page + gd.sz_off + 8 * ((u & 7) * (P >> 4) + (u >> 3)));
    const float s = __half2float(rec[tau & 1]), z = __half2float(rec[2 + (tau & 1)]);
    lat[t][c] = fmaf((float)code, s, z);
  }
  __syncthreads();
  // lift with W_up (V side rows [n_kept][d_h], K side transposed [d_h][n_kept])
  const float* w = cd->w_up + sd.wup_off;
  for (int e = threadIdx.x; e < nt * d_h; e += blockDim.x) {
    const int t = e / d_h, d = e % d_h;
    float acc = 0.f;
    for (int c = 0; c < nk; ++c) acc = fmaf(lat[t][c], side == 0 ? w[(size_t)d * nk + c] : w[(size_t)c * d_h + d], acc);
    out[((size_t)(tok0 - t0 + t) * n_kv + a) * d_h + d] = acc;
  }
}

}  // namespace

cudaError_t launch_reconstruct(const CodecDev& h, const CodecDev* d, const spectra_cache& cache, int b, int64_t t0,
                               int64_t n, float* K_out, float* V_out, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((n + kRecTokens - 1) / kRecTokens), h.n_kv, 2);
  reconstruct_kernel<<<grid, 128, 0, st>>>(d, static_cast<const uint8_t*>(cache.pool), cache.page_table,
                                           cache.lengths, cache.n_pages, cache.max_pages_per_seq, b, t0, n, K_out,
                                           V_out);
  return cudaGetLastError();
}

}  // namespace spectra
