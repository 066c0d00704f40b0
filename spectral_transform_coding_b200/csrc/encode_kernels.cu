// Encode side of libspectra: "tokens are projected down, quantised per token and
// appended to the latent cache" (SPECTRA technical summary, "SPECTRA pipeline",
// stage 3), with groups of adjacent latent coordinates sharing one width (stage 2,
// "grouping").
#include <cuda_bf16.h>
#include <algorithm>
#include <cstdlib>
#include <cuda_fp16.h>

#include "device_common.cuh"
#include "kernels.h"
#include "pack_device.cuh"

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
using namespace pack;

template <int G>
__global__ void __launch_bounds__(128) quantize_append_kernel(
    const CodecDev* __restrict__ cd, const float* __restrict__ C, int64_t ldc,
    const int32_t* __restrict__ seq_ids, const int32_t* __restrict__ pos,
    const int32_t* __restrict__ ok_flag, int T, uint8_t* __restrict__ pool,
    const int32_t* __restrict__ page_table, int max_pages) {
  constexpr int TB = 256 / G;               // tokens per 256-bit block
  constexpr int LANES_PER_TOKENSET = TB;    // 16 or 32
  constexpr int GROUPS_PER_WARP = 32 / LANES_PER_TOKENSET;
  // No early trigger: a decode launched next copies pages before its own
  // dependency wait, so its kernels may start only once these writes are done
  // (the implicit trigger at this grid's completion).
  pdl_wait();  // latents and the append plan come from the preceding kernels
  if (*ok_flag == 0) return;
  const int a = blockIdx.y >> 1, side = blockIdx.y & 1;
  const SideDev& sd = cd->head[a].side[side];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // This CTA's TB input tokens fill one whole block when they exist, belong to
  // one sequence and start at a block boundary (positions of one sequence are
  // consecutive): then each group's block is assembled in shared memory and
  // stored whole; otherwise tokens merge their bits into the page with atomics.
  const int i0 = blockIdx.x * TB;
  const bool full = i0 + TB <= T && seq_ids[i0] == seq_ids[i0 + TB - 1] && pos[i0] % TB == 0;
  __shared__ __align__(16) uint32_t wbuf[4][GROUPS_PER_WARP][64];
  const int i = i0 + (lane % TB);
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
    __half s_h, z_h;
    uint32_t code[G];
    quantize_group<G>(x, b, s_h, z_h, code);
    uint32_t* blkw = reinterpret_cast<uint32_t*>(page + gd.plane_off + blk * (32 * b));
    if (full) {
      // the TB lanes holding this group (one half-warp for G = 16) own the block
      const unsigned hm = GROUPS_PER_WARP == 2 ? (0xFFFFu << (16 * (lane >> 4))) : 0xFFFFFFFFu;
      const int sub = lane % LANES_PER_TOKENSET;
      uint32_t* wb = wbuf[warp][lane / LANES_PER_TOKENSET];
      for (int w = sub; w < 8 * b; w += LANES_PER_TOKENSET) wb[w] = 0u;
      __syncwarp(hm);
      put_codes<G, true>(wb, side, tb, b, code);
      __syncwarp(hm);
      for (int w4 = sub; w4 < 2 * b; w4 += LANES_PER_TOKENSET)
        reinterpret_cast<uint4*>(blkw)[w4] = reinterpret_cast<const uint4*>(wb)[w4];
      __syncwarp(hm);  // before the next group reuses the buffer
    } else {
      put_codes<G, false>(blkw, side, tb, b, code);
    }
    put_record(page + gd.sz_off, P, tau, s_h, z_h);
  }
}

// ---------------------------------------------------------------------------
// Fused small-batch encode (decode steps, T <= kFusedMaxT tokens).  The
// projection of the step's tokens is split over CTAs (kept group, consecutive
// d_model chunks of KCH columns of H): each CTA has all of its group's G rows
// of W_down over its chunks in flight before the dependency wait (the first
// chunk in registers, later ones staged in shared memory by bulk copies),
// multiplies them with the tokens' H (read after the wait) and reduces across
// the warp.  A group split over several CTAs adds their partial sums in CTA
// order: in rank 0's shared memory when the CTAs form a cluster, else through
// the workspace and the group's last CTA to arrive (a counter per group).
// That CTA quantises and packs the group for the step's tokens, one half warp
// per token.  Every CTA computes and validates the positions the same way from
// the current lengths, so a failed check writes nothing anywhere; the last CTA
// to hold its positions (a second counter) advances the lengths at once.  All
// counters are left at zero.
// ---------------------------------------------------------------------------
namespace {

// Cache position of token t of an append (seq_ids non-decreasing) and the page
// id it lands in, or an error.
__device__ __forceinline__ int append_position(const int32_t* __restrict__ seq_ids, int t,
                                               const spectra_cache& c, int P, int64_t* pos, int* page = nullptr) {
  const int s = seq_ids[t];
  if (s < 0 || s >= c.batch || (t > 0 && seq_ids[t - 1] > s)) return SPECTRA_ERR_ORDER;
  int first = t;
  while (first > 0 && seq_ids[first - 1] == s) --first;
  const int64_t p = (int64_t)c.lengths[s] + (t - first);
  if (p < 0 || p >= (int64_t)c.max_pages_per_seq * P) return SPECTRA_ERR_CAPACITY;
  const int pid = c.page_table[(size_t)s * c.max_pages_per_seq + p / P];
  if (pid < 0 || (int64_t)pid >= c.n_pages) return SPECTRA_ERR_CAPACITY;
  *pos = p;
  if (page) *page = pid;
  return 0;
}

}  // namespace

namespace {

// Sum of vals[v] over the 32 lanes of a warp for V values per lane (V a power
// of two <= 32), by recursive halving: lane l ends with the total of value
// l >> (5 - log2 V).
template <int V>
__device__ __forceinline__ float warp_transpose_sum(float (&vals)[V], int lane) {
  int len = V;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (len > 1) {
      const int half = len / 2;
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < half) {
          const float send = upper ? vals[i] : vals[i + half];
          const float keep = upper ? vals[i + half] : vals[i];
          vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      len = half;
    } else {
      vals[0] += __shfl_xor_sync(0xffffffffu, vals[0], o);
    }
  }
  return vals[0];
}

__host__ __device__ constexpr int log2_int(int v) { return v <= 1 ? 0 : 1 + log2_int(v / 2); }

constexpr int kMaxChunks = 16;  // d_model chunks per group (the plan keeps to it)
constexpr int kFusedMaxStageBytes = 96 * 1024;  // staged W_down per CTA
constexpr unsigned long long kFusedWaitLimitNs = 200ull * 1000ull * 1000ull;  // bounded wait for staged copies

}  // namespace

template <int G, int TP, int BATCH>
__global__ void __launch_bounds__(256) encode_fused_kernel(const EncodeFusedArgs A, const uint16_t* __restrict__ H,
                                                           int T, const int32_t* __restrict__ seq_ids,
                                                           const spectra_cache cache,
                                                           float* __restrict__ latents_out,
                                                           int32_t* __restrict__ counters,
                                                           float* __restrict__ part, int n_chunks, int cpc) {
  constexpr int CPW = G / 8;        // columns per warp (8 warps cover the group)
  constexpr int KCH = 256 * BATCH;  // d_model columns of H per chunk
  constexpr int V = CPW * TP;       // partial sums per lane
  extern __shared__ __align__(128) uint8_t w_s[];  // staged chunks: [chunk - ch0 - 1][G][KCH] bf16
  __shared__ float x_s[TP][G];
  __shared__ float red_s[kMaxChunks * TP * G];  // cluster rank 0: the group's partial sums [rank][TP][G]
  __shared__ int64_t pos_s[TP];
  __shared__ int pid_s[TP];
  __shared__ __align__(8) uint64_t w_bar;
  __shared__ int worst;
  __shared__ int flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_launch_dependents();
  // this CTA's kept group gi (numbered head-major, K side then V side: latent
  // columns gi G .. gi G + G - 1) and its chunks [ch0, ch1) of d_model
  const int gi = blockIdx.x, n_part = gridDim.y;
  const int ch0 = blockIdx.y * cpc;
  int ch1 = min(n_chunks, ch0 + cpc);
  const int d_model = A.d_model;
  const int n0 = gi * G + warp * CPW;  // latent columns of this warp
  // W_down rows of the group (read-only codec data) all go out before the
  // wait: the first chunk into registers, this warp's columns; with `staged`
  // the later chunks by bulk copies into shared memory, else into registers
  // after the wait
  const bool staged = A.staged && ch1 - ch0 > 1;
  if (staged && tid == 0) {
    mbar_init(&w_bar, 1);
    fence_mbar_init();
    uint32_t bytes = 0;
    for (int ch = ch0 + 1; ch < ch1; ++ch) bytes += (uint32_t)(G * 2 * min(KCH, d_model - ch * KCH));
    mbar_arrive_expect_tx(&w_bar, bytes);
    for (int ch = ch0 + 1; ch < ch1; ++ch) {
      const int len = min(KCH, d_model - ch * KCH);
      for (int r = 0; r < G; ++r) {
        if (A.drop_stage && gi == 0 && blockIdx.y == 0 && ch == ch0 + 1 && r == 0) continue;  // test hook
        bulk_copy_g2s(w_s + ((size_t)(ch - ch0 - 1) * G + r) * (KCH * 2),
                      A.wt_down + (size_t)(gi * G + r) * d_model + (size_t)ch * KCH, (uint32_t)len * 2u, &w_bar);
      }
    }
  }
  uint4 wv[CPW][BATCH];
  auto load_w = [&](int ch) {
#pragma unroll
    for (int i = 0; i < BATCH; ++i)
#pragma unroll
      for (int c = 0; c < CPW; ++c) {
        const int k = ch * KCH + lane * 8 + 256 * i;
        wv[c][i] = k < d_model ? __ldg(reinterpret_cast<const uint4*>(A.wt_down + (size_t)(n0 + c) * d_model + k))
                               : make_uint4(0u, 0u, 0u, 0u);
      }
  };
  auto stage_w = [&](int ch) {
    const uint8_t* src = w_s + (size_t)(ch - ch0 - 1) * G * (KCH * 2);
#pragma unroll
    for (int i = 0; i < BATCH; ++i)
#pragma unroll
      for (int c = 0; c < CPW; ++c) {
        const int kl = lane * 8 + 256 * i;
        wv[c][i] = ch * KCH + kl < d_model
                       ? *reinterpret_cast<const uint4*>(src + ((size_t)(warp * CPW + c) * KCH + kl) * 2)
                       : make_uint4(0u, 0u, 0u, 0u);
      }
  };
  load_w(ch0);
  const int4 cg = __ldg(reinterpret_cast<const int4*>(A.col_groups) + gi);  // {width, block off, record off, side}
  pdl_wait();  // H, lengths and the page table may come from earlier kernels
  // positions of the step's tokens (their loads overlap the projection); every
  // CTA that finishes a group reaches the same verdict from them
  if (warp == 0) {  // T <= 16
    int e = 0;
    int64_t pos = 0;
    if (lane < T) {
      int pid = 0;
      e = append_position(seq_ids, lane, cache, A.P, &pos, &pid);
      pos_s[lane] = pos;
      pid_s[lane] = pid;
    }
    e = __reduce_max_sync(0xffffffffu, e);  // also orders the lanes' reads before the arrival
    // Every CTA arrives once it holds its positions; the last to arrive advances
    // the lengths at once (no CTA of this grid reads them afterwards) and leaves
    // the counter at zero for the next call.  The lengths thus run ahead of this
    // grid's page writes by at most T tokens per sequence until it completes; a
    // decode that starts early copies only pages full kFusedMaxT tokens below
    // its length hint before its own dependency wait.
    int last = 0;
    if (lane == 0) {
      worst = e;
      last = atom_add_acq_rel(counters, 1) == (int)(gridDim.x * gridDim.y) - 1;
      if (last) counters[0] = 0;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last && !e && lane < T && (lane == T - 1 || seq_ids[lane + 1] != seq_ids[lane]))
      cache.lengths[seq_ids[lane]] = (int32_t)(pos + 1);
  }
  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;
  if (staged) {
    __syncthreads();  // the barrier is initialised
    // bounded: a copy that never lands ends in a status (no writes; the
    // arrivals below still happen), not a hang
    if (!__syncthreads_and(mbar_wait_bounded(&w_bar, 0, A.wait_ns))) {
      if (tid == 0) {
        device_error(A.err, SPECTRA_ERR_TIMEOUT);
        atomicMax(&worst, SPECTRA_ERR_TIMEOUT);
      }
      ch1 = ch0 + 1;
    }
  }
  for (int ch = ch0; ch < ch1; ++ch) {
    if (ch > ch0) {
      if (staged) stage_w(ch);
      else load_w(ch);
    }
#pragma unroll
    for (int r = 0; r < TP; ++r) {
      if (r < T) {
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const int k = ch * KCH + lane * 8 + 256 * i;
          float h[8];
          bf16x8_to_f32(k < d_model ? __ldg(reinterpret_cast<const uint4*>(H + (size_t)r * d_model + k))
                                    : make_uint4(0u, 0u, 0u, 0u), h);
#pragma unroll
          for (int c = 0; c < CPW; ++c) {
            float w[8];
            bf16x8_to_f32(wv[c][i], w);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[c * TP + r] = fmaf(w[e], h[e], acc[c * TP + r]);
          }
        }
      }
    }
  }
  {
    const float tot = warp_transpose_sum<V>(acc, lane);
    constexpr int SH = 5 - log2_int(V);
    const int v = lane >> SH, c = v / TP, r = v % TP;
    if ((lane & ((1 << SH) - 1)) == 0 && r < T) {
      if (n_part == 1) x_s[r][warp * CPW + c] = tot;
      else if (A.cluster)
        st_shared_cluster_f32(mapa_shared(smem_u32(&red_s[(blockIdx.y * TP + r) * G + warp * CPW + c]), 0), tot);
      else part[((size_t)(gi * n_part + blockIdx.y) * TP + r) * G + warp * CPW + c] = tot;
    }
  }
  if (n_part > 1 && A.cluster) {
    // the group's CTAs are one cluster (rank = blockIdx.y): rank 0 adds the
    // partial sums that every rank stored into its shared memory, in rank order
    cluster_sync_all();
    if (blockIdx.y != 0) return;
    if (tid < T * G) {
      const int r = tid / G, c = tid % G;
      float x = 0.f;
      for (int k = 0; k < n_part; ++k) x += red_s[(k * TP + r) * G + c];
      x_s[r][c] = x;
    }
  } else if (n_part > 1) {
    // the last CTA of this group to arrive adds the CTAs' partial sums in order
    // (barrier, then one thread's fence releases the partials before the
    // arrival; the last CTA's thread fences again to acquire the others')
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const int t = atomicAdd(counters + 1 + gi, 1);
      flag = t == n_part - 1;
      if (flag) __threadfence();
    }
    __syncthreads();
    if (!flag) return;
    if (tid < T * G) {
      const int r = tid / G, c = tid % G;
      const float* pp = part + ((size_t)gi * n_part * TP + r) * G + c;
      float v[kMaxChunks];
#pragma unroll
      for (int k = 0; k < kMaxChunks; ++k) v[k] = k < n_part ? __ldcg(pp + (size_t)k * TP * G) : 0.f;
      float x = 0.f;
#pragma unroll
      for (int k = 0; k < kMaxChunks; ++k) x += v[k];  // CTA order; absent ones add zero
      x_s[r][c] = x;
    }
  }
  __syncthreads();
  const int bad = worst;
  if (bad && gi == 0 && tid == 0) device_error(A.err, bad);
  // quantise and pack: half warp t takes token t, lane k of the half latent k
  {
    const int t = tid >> 4, k = tid & 15;
    if (!bad && t < T) {
      const float x = x_s[t][k < G ? k : 0];
      if (latents_out && k < G) latents_out[(size_t)t * A.n_eff + gi * G + k] = x;
      const int P = A.P, TB = 256 / G;
      const int64_t pos = pos_s[t];
      uint8_t* page = static_cast<uint8_t*>(cache.pool) + (size_t)pid_s[t] * (size_t)A.page_bytes;
      const int tau = (int)(pos % P), b = cg.x;
      __half s_h, z_h;
      const uint32_t code = quantize_half_warp(x, b, s_h, z_h);
      if (k < G) {
        int g8, t4, slot;
        if (cg.w == 0) k_side_pos<G>(tau % TB, k, &g8, &t4, &slot);
        else v_side_pos<G>(tau % TB, k, &g8, &t4, &slot);
        const CodeBits cb = code_bits(b, g8, t4, slot, code);
        uint32_t* blkw = reinterpret_cast<uint32_t*>(page + cg.y + (tau / TB) * (32 * b));
        // other lanes' and tokens' bits share these words: clear and set only ours
        atomicAnd(blkw + cb.w0, ~cb.m0);
        atomicOr(blkw + cb.w0, cb.v0);
        if (cb.w1 >= 0) {
          atomicAnd(blkw + cb.w1, ~cb.m1);
          atomicOr(blkw + cb.w1, cb.v1);
        }
      }
      if (k == 0) put_record(page + cg.z, P, tau, s_h, z_h);
    }
  }
  // every CTA of this group has arrived: its counter is free for the next call,
  // which starts after this grid
  if (n_part > 1 && !A.cluster && tid == 0) counters[1 + gi] = 0;
}

// Advances the lengths of an append that writes no codes (a codec that keeps
// no group at all), with the checks of the fused encode.
__global__ void __launch_bounds__(32) length_advance_kernel(const int32_t* __restrict__ seq_ids, int T,
                                                            const spectra_cache cache, int P, int32_t* err) {
  pdl_wait();
  const int t = threadIdx.x;
  int64_t pos = 0;
  const int e = t < T ? append_position(seq_ids, t, cache, P, &pos) : 0;
  const int bad = __reduce_max_sync(0xffffffffu, e);
  if (bad) {
    if (t == 0) device_error(err, bad);
    return;
  }
  if (t < T && (t == T - 1 || seq_ids[t + 1] != seq_ids[t])) cache.lengths[seq_ids[t]] = (int32_t)(pos + 1);
}

cudaError_t launch_length_advance(const int32_t* seq_ids, int T, const spectra_cache& cache, int P, cudaStream_t st,
                                  int32_t* err = nullptr);

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

cudaError_t launch_length_advance(const int32_t* seq_ids, int T, const spectra_cache& cache, int P, cudaStream_t st,
                                  int32_t* err) {
  return launch_dependent(length_advance_kernel, dim3(1), dim3(32), 0, st, seq_ids, T, cache, P, err);
}

EncodeFusedPlan encode_fused_plan(const CodecDev& h, int T) {
  EncodeFusedPlan p{};
  for (int a = 0; a < h.n_kv; ++a) p.n_groups += h.head[a].side[0].n_groups + h.head[a].side[1].n_groups;
  p.tp = 1;
  while (p.tp < T) p.tp *= 2;
  static int sm_of_dev[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (sm_of_dev[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    sm_of_dev[dev] = n;
  }
  const int sms = sm_of_dev[dev];
  // CTAs to aim for.  A step of a few sequences leaves one decode CTA per SM
  // running beside this kernel, so one wave of CTAs that fits next to it starts
  // early and streams W_down before its dependency wait; with more sequences the
  // decode fills the SMs and this kernel runs after it, as wide as possible.
  const long target = T >= 4 ? 2L * sms : (long)sms;
  // chunks: the widest (fewest partial sums, at most 8 loads of 16 bytes per
  // column and lane) that gives the target, at most kMaxChunks
  p.batch = 8;
  for (int bt = 8; bt >= 1; bt /= 2) {
    const int nch = (h.d_model + 256 * bt - 1) / (256 * bt);
    if (nch > kMaxChunks) break;
    p.batch = bt;
    if ((long)p.n_groups * nch >= target) break;
  }
  p.n_chunks = (h.d_model + 256 * p.batch - 1) / (256 * p.batch);
  // consecutive chunks per CTA: one when the kernel runs after the decode (every
  // CTA's loads then start at once), else as many as keep to the target
  const long per_group = p.n_groups > 0 ? std::max(1L, target / p.n_groups) : 1L;
  p.cpc = T >= 4 ? 1 : (int)((p.n_chunks + per_group - 1) / per_group);
  p.n_part = (p.n_chunks + p.cpc - 1) / p.cpc;
  // the chunks after a CTA's first go to shared memory by bulk copies before the
  // wait when they fit beside a running decode CTA
  const int stage = (p.cpc - 1) * h.group * 256 * p.batch * 2;
  p.staged = p.cpc > 1 && stage <= kFusedMaxStageBytes && h.d_model % 8 == 0;
  p.smem_bytes = p.staged ? stage : 0;
  // the group's CTAs add their partial sums in a cluster's shared memory when
  // they run beside the decode (a few sequences); with more sequences the
  // decode fills the SMs and clusters wait for whole free groups of SMs, so the
  // partial sums go through global memory (measured: slower by 6-7 us per layer
  // at batch 16 with clusters of 8 or 16)
  p.cluster = T < 4 && p.n_part > 1 && p.n_part <= 8;
  return p;
}

size_t encode_fused_partial_bytes(const CodecDev& h, int T) {
  const EncodeFusedPlan p = encode_fused_plan(h, T);
  return (size_t)p.n_groups * p.n_part * p.tp * h.group * 4;
}

namespace {
template <int G, int TP>
cudaError_t launch_fused_tp(const EncodeFusedPlan& p, const EncodeFusedArgs& args, const uint16_t* H, int T,
                            const int32_t* seq_ids, const spectra_cache& cache, float* latents_out,
                            int32_t* counters, float* part, cudaStream_t st) {
  const dim3 grid(p.n_groups, p.n_part), block(256);
  auto go = [&](auto kern) -> cudaError_t {
    if (p.smem_bytes > 0) {
      const cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), p.smem_bytes);
      if (e != cudaSuccess) return e;
    }
    if (p.cluster) {
      // the group's CTAs as one cluster (at most 8: a portable size); if the
      // launch is refused, the partial sums go through global memory
      EncodeFusedArgs ca = args;
      ca.cluster = 1;
      if (launch_dependent_cluster(kern, grid, block, p.smem_bytes, st, dim3(1, p.n_part, 1), ca, H, T, seq_ids,
                                   cache, latents_out, counters, part, p.n_chunks, p.cpc) == cudaSuccess)
        return cudaSuccess;
    }
    return launch_dependent(kern, grid, block, p.smem_bytes, st, args, H, T, seq_ids, cache, latents_out, counters,
                            part, p.n_chunks, p.cpc);
  };
  switch (p.batch) {
    case 8: return go(encode_fused_kernel<G, TP, 8>);
    case 4: return go(encode_fused_kernel<G, TP, 4>);
    case 2: return go(encode_fused_kernel<G, TP, 2>);
    default: return go(encode_fused_kernel<G, TP, 1>);
  }
}

template <int G>
cudaError_t launch_fused_g(const EncodeFusedPlan& p, const EncodeFusedArgs& d, const uint16_t* H, int T,
                           const int32_t* seq_ids, const spectra_cache& cache, float* latents_out,
                           int32_t* counters, float* part, cudaStream_t st) {
  switch (p.tp) {
    case 1: return launch_fused_tp<G, 1>(p, d, H, T, seq_ids, cache, latents_out, counters, part, st);
    case 2: return launch_fused_tp<G, 2>(p, d, H, T, seq_ids, cache, latents_out, counters, part, st);
    case 4: return launch_fused_tp<G, 4>(p, d, H, T, seq_ids, cache, latents_out, counters, part, st);
    case 8: return launch_fused_tp<G, 8>(p, d, H, T, seq_ids, cache, latents_out, counters, part, st);
    default: return launch_fused_tp<G, 16>(p, d, H, T, seq_ids, cache, latents_out, counters, part, st);
  }
}
}  // namespace

cudaError_t launch_encode_fused(const CodecDev& h, const CodecDev* d, const uint16_t* H, const int32_t* seq_ids,
                                int T, const spectra_cache& cache, float* latents_out, int32_t* counters,
                                float* part, cudaStream_t st) {
  const EncodeFusedPlan p = encode_fused_plan(h, T);
  if (p.n_groups == 0) return launch_length_advance(seq_ids, T, cache, h.P, st, h.err);
  if (T > kFusedMaxT || p.n_groups > kMaxFusedGroups || p.n_part > kMaxChunks) return cudaErrorNotSupported;
  (void)d;
  EncodeFusedArgs args;
  args.wt_down = h.wt_down;
  args.col_groups = h.col_groups;
  args.err = h.err;
  args.page_bytes = h.page_bytes;
  // test hooks for the bounded wait on the staged copies:
  // SPECTRA_ENCODE_TEST_DROP_STAGE makes the first CTA skip its first staged
  // copy (its wait then gives up and the call reports SPECTRA_ERR_TIMEOUT), and
  // SPECTRA_ENCODE_TEST_WAIT_NS shortens the wait's limit
  const char* ds = std::getenv("SPECTRA_ENCODE_TEST_DROP_STAGE");
  const char* wn = std::getenv("SPECTRA_ENCODE_TEST_WAIT_NS");
  const long long wait = wn ? std::atoll(wn) : 0;
  args.drop_stage = ds ? 1 : 0;
  args.wait_ns = wait > 0 ? (unsigned long long)wait : kFusedWaitLimitNs;
  args.d_model = h.d_model;
  args.n_eff = h.n_eff;
  args.P = h.P;
  args.staged = p.staged;
  args.cluster = 0;
  if (h.group == 16) return launch_fused_g<16>(p, args, H, T, seq_ids, cache, latents_out, counters, part, st);
  return launch_fused_g<8>(p, args, H, T, seq_ids, cache, latents_out, counters, part, st);
}

}  // namespace spectra
