// Decode side of libspectra: attention over the packed latent cache, computed in
// the latent space ("SPECTRA: Pushing the KV Cache Beyond the 2-Bit Cliff via
// Spectral Transform Coding", "Significance and claims": the latent structure
// allows attention directly in latent space; "SPECTRA pipeline" stage 3: the
// rebuilt keys/values feed standard softmax attention).
//
// For q head h of KV head a, with per-group dequantised latents c = code*s + z:
//   q . k      = q_lat . c_K,                 q_lat = q W_up^K^T
//   q_lat . c_K = sum_j [ s_j (q_lat,j . code_j) + z_j (sum_{k in j} q_lat,k) ]
//   sum_t p_t c_V,t = sum_t (p_t s_t,j) code_t,j + sum_t p_t z_t,j   (per group j)
//   out = (sum_t p_t c_V,t / sum_t p_t) W_up^V.
// Integer codes enter mma.sync as exact fp16 subnormals (code * 2^-24); q_lat is
// split into fp16 hi + lo columns so scores keep ~22 bits; the z terms are two
// more MMAs per 16-token tile.
//
// Three kernels per decode step, chained with programmatic dependent launch:
//   fold    one CTA per (sequence, KV head): q_lat and its group sums, written
//           as the split kernel's MMA B fragments;
//   split   one CTA per (context split, KV head, sequence): streams its pages
//           (bulk copies into per-warp shared-memory stages) while the fold
//           runs, then an online softmax over 64-token chunks; one partial
//           record (max, sum, latent accumulator) per q head;
//   combine one CTA per (q head, sequence): merges the splits, applies W_up^V
//           (bulk-copied into shared memory while the splits finish).
#include <cuda_fp16.h>
#include <math_constants.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "device_common.cuh"
#include "kernels.h"

namespace spectra {

namespace {

constexpr int kDecWarps = 4;
constexpr int kMaxG = 8;          // kept groups per side handled by the decode kernels
constexpr int kMaxKept = 128;     // kept coordinates per side
constexpr int kChunk = 4;         // 16-token tiles per softmax chunk
constexpr int kMaxSplit = 256;    // context splits per (sequence, KV head)
constexpr uint64_t kWaitLimitNs = 200ull * 1000ull * 1000ull;  // bounded mbarrier waits
constexpr float kPScaleLog2 = 8.f;   // p = 2^(s - m + 8): fp16 keeps small weights normal
constexpr float kTwo24 = 16777216.f; // undo the 2^-24 of subnormal codes
constexpr int kFragWords = (kMaxG * 2 + 2) * 32;  // uint2 per (sequence, KV head): bq[j][nt], bz[nt]

// split kernel shared-memory carve-up (bytes)
constexpr int kSmBars = 0;                                   // 4 warps x 8 mbarriers
constexpr int kSmBq = 512;                                   // fragments [kMaxG*2 + 2][32] uint2
constexpr int kSmGrp = kSmBq + kFragWords * 8;               // int4 {plane, rec, b, -} x (K 8, V 8)
constexpr int kSmMisc = kSmGrp + 2 * kMaxG * 16;             // 32 ints
constexpr int kSmAcc = kSmMisc + 128;                        // value accumulators [warp][kMaxG][32] float4
constexpr int kSmStages = kSmAcc + kDecWarps * kMaxG * 32 * 16;

struct DecodeArgs {
  const CodecDev* cd;
  const uint8_t* pool;
  const int32_t* page_table;
  const int32_t* lengths;
  const float* q;
  float* out;
  float* part;
  uint2* frag;
  int64_t n_pool_pages;
  int64_t page_bytes;
  int max_pages;
  int n_split;
  int stages;
  int stage_bytes;
  int part_stride;
  int n_q;
  int n_kv;
  float q_scale;
};

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// mma with a zero accumulator input (no register moves for C)
__device__ __forceinline__ void mma_m16n8k16_z(float d[4], const uint32_t a[4], const uint32_t b[2]) {
  const float z = 0.f;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(z));
}

__device__ __forceinline__ void mma_m16n8k8_z(float d[4], const uint32_t a[2], uint32_t b) {
  const float z = 0.f;
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%7,%7,%7};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(b), "f"(z));
}

// Codes of one group into 4-bit fields: rotating plane p's word right by
// (t4 - p mod 4) places this lane's 8 bits of the block at bits 4*slot + p mod 4;
// planes 0-3 fill `lo`, planes 4-7 fill `hi`.
template <int B>
__device__ __forceinline__ void gather_fixed(const uint8_t* pw, int stride, const uint32_t (&rot)[4],
                                             uint32_t& lo, uint32_t& hi) {
  lo = 0u;
  hi = 0u;
#pragma unroll
  for (int p = 0; p < B; ++p) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(pw + p * stride);
    const uint32_t r = __funnelshift_r(w, w, rot[p & 3]);
    if (p < 4) lo |= r & (0x11111111u << p);
    else hi |= r & (0x11111111u << (p - 4));
  }
}

// Element pair (slot i, slot i+4) as two 16-bit integers: as fp16 bit patterns
// these are the subnormals code * 2^-24.
__device__ __forceinline__ uint32_t slot_pair(uint32_t lo, uint32_t hi, int i, bool wide) {
  uint32_t v = (lo >> (4 * i)) & 0x000F000Fu;
  if (wide) v |= ((hi >> (4 * i)) & 0x000F000Fu) << 4;
  return v;
}

template <int G>
__device__ __forceinline__ void code_frag_k(uint32_t lo, uint32_t hi, bool wide, int mi, uint32_t (&av)[4]) {
  if (G == 16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) av[i] = slot_pair(lo, hi, i, wide);
  } else {  // m16n8k8: rows (gid, gid+8) of half mi
    av[0] = slot_pair(lo, hi, 2 * mi, wide);
    av[1] = slot_pair(lo, hi, 2 * mi + 1, wide);
  }
}

template <int G>
__device__ __forceinline__ void code_frag_v(uint32_t lo, uint32_t hi, bool wide, int mi, uint32_t (&av)[4]) {
  if (G == 16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) av[i] = slot_pair(lo, hi, i, wide);
  } else {  // m16n8k16 with coordinate rows 8..15 padded with zeros
    av[0] = slot_pair(lo, hi, mi, wide);
    av[1] = 0u;
    av[2] = slot_pair(lo, hi, mi + 2, wide);
    av[3] = 0u;
  }
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// ---------------------------------------------------------------------------
// fold: q_lat[h][c] = (q_h . W_up^K[c]) * log2(e)/sqrt(d_h) and group sums, as
// B fragments: bq[j][nt][lane] column n = lane/4 of n-tile nt is q head
// nt*4 + n/2, part n&1 (0: fp16(q_lat), 1: fp16(q_lat - fp16(q_lat))); rows
// k = 2*(lane%4) + {0,1} (+8).  bz[nt][lane] likewise over group sums.
// ---------------------------------------------------------------------------
template <int G, int NT>
__global__ void __launch_bounds__(256) fold_kernel(const DecodeArgs A) {
  const CodecDev* __restrict__ cd = A.cd;
  const int a = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  float* qlat_s = reinterpret_cast<float*>(smem + 128);            // [kMaxGQ][kMaxKept]
  float* qsum_s = qlat_s + kMaxGQ * kMaxKept;                      // [kMaxGQ][kMaxG]
  float* q_s = qsum_s + kMaxGQ * kMaxG;                            // [kMaxGQ][kMaxDHead]
  float* w_s = q_s + kMaxGQ * kMaxDHead;                           // [d_h][n_kept]
  const int gq = cd->gq, d_h = cd->d_h;
  const SideDev* sk = &cd->head[a].side[0];
  const int nk = sk->n_kept, nK = sk->n_groups;
  const uint32_t wbytes = (uint32_t)nk * d_h * 4;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    if (wbytes) {
      mbar_arrive_expect_tx(bar, wbytes);
      bulk_copy_g2s(w_s, cd->w_up + sk->wup_off, wbytes, bar);
    }
  }
  const float* qb = A.q + ((size_t)b * A.n_q + (size_t)a * gq) * d_h;
  for (int e = tid; e < gq * d_h; e += blockDim.x) q_s[(e / d_h) * kMaxDHead + e % d_h] = qb[e];
  __syncthreads();
  bool ok = true;
  if (wbytes) ok = mbar_wait_bounded(bar, 0, kWaitLimitNs);
  if (!ok && tid == 0) device_error(cd->err, SPECTRA_ERR_TIMEOUT);
  for (int idx = tid; idx < nk * gq; idx += blockDim.x) {
    const int c = idx % nk, h = idx / nk;
    float acc = 0.f;
    for (int d = 0; d < d_h; ++d) acc = fmaf(q_s[h * kMaxDHead + d], w_s[d * nk + c], acc);
    qlat_s[h * kMaxKept + c] = ok ? acc * A.q_scale : 0.f;
  }
  __syncthreads();
  if (tid < gq * kMaxG) {
    const int h = tid / kMaxG, j = tid % kMaxG;
    float s = 0.f;
    if (j < nK)
      for (int k = 0; k < G; ++k) s += qlat_s[h * kMaxKept + j * G + k];
    qsum_s[h * kMaxG + j] = s;
  }
  __syncthreads();
  uint2* out = A.frag + ((size_t)b * A.n_kv + a) * kFragWords;
  for (int idx = tid; idx < (kMaxG + 1) * NT * 32; idx += blockDim.x) {
    const int lane = idx % 32, row = idx / 32;  // row < kMaxG*NT: bq[j][nt]; then bz[nt]
    const int gid = lane >> 2, t4 = lane & 3;
    const bool is_bz = row >= kMaxG * NT;
    const int j = is_bz ? 0 : row / NT, nt = is_bz ? row - kMaxG * NT : row % NT;
    const int hl = nt * 4 + (gid >> 1);
    const int part = gid & 1;
    auto split_h = [&](float x) -> float {
      const float hi = __half2float(__float2half_rn(x));
      return part ? (x - hi) : hi;
    };
    uint2 v = make_uint2(0u, 0u);
    if (hl < gq) {
      if (is_bz) {
        const float* qs = qsum_s + hl * kMaxG;
        v.x = pack_half2(split_h(qs[2 * t4]), split_h(qs[2 * t4 + 1]));
      } else if (j < nK) {
        const float* base = qlat_s + hl * kMaxKept + j * G;
        v.x = pack_half2(split_h(base[2 * t4]), split_h(base[2 * t4 + 1]));
        if (G == 16) v.y = pack_half2(split_h(base[2 * t4 + 8]), split_h(base[2 * t4 + 9]));
      }
    }
    out[(is_bz ? kMaxG * 2 + nt : j * NT + nt) * 32 + lane] = v;
  }
}

// ---------------------------------------------------------------------------
// split: one context split of one (sequence, KV head)
// ---------------------------------------------------------------------------

// Keys of one group for the tiles of a chunk: s_j (q_lat,j . code_j) accumulated
// into acc[tt][nt][hi/lo of token 2gid, hi/lo of token 2gid+1].
template <int G, int NT, int B>
__device__ __forceinline__ void key_group(const uint8_t* __restrict__ pbase, const uint8_t* __restrict__ rbase,
                                          const uint2 (&bqj)[NT], int t0, int ntile, int plane_stride,
                                          const uint32_t (&rot)[4], float (&acc)[kChunk][NT][4]) {
#pragma unroll
  for (int tt = 0; tt < kChunk; ++tt) {
    if (tt < ntile) {
      const int t = t0 + tt;
      const int blk = (G == 16) ? t : (t >> 1);
      const int mi = (G == 16) ? 0 : (t & 1);
      uint32_t lo, hi;
      gather_fixed<B>(pbase + blk * 32, plane_stride, rot, lo, hi);
      const uint32_t s2 = *reinterpret_cast<const uint32_t*>(rbase + t * 64);
      const float sA = half_lo(s2), sB = half_hi(s2);
      uint32_t av[4];
      code_frag_k<G>(lo, hi, B > 4, mi, av);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float d[4];
        const uint32_t bb[2] = {bqj[nt].x, bqj[nt].y};
        if (G == 16) mma_m16n8k16_z(d, av, bb);
        else mma_m16n8k8_z(d, av, bb[0]);
        acc[tt][nt][0] = fmaf(sA, d[0], acc[tt][nt][0]);
        acc[tt][nt][1] = fmaf(sA, d[1], acc[tt][nt][1]);
        acc[tt][nt][2] = fmaf(sB, d[2], acc[tt][nt][2]);
        acc[tt][nt][3] = fmaf(sB, d[3], acc[tt][nt][3]);
      }
    }
  }
}

// Values of one group for the tiles of a chunk: va += code^T (p s) (codes as
// subnormals, so va carries a factor 2^-24).
template <int G, int B>
__device__ __forceinline__ void value_group(const uint8_t* __restrict__ pbase, const uint8_t* __restrict__ rbase,
                                            const uint32_t (&pb)[kChunk][2], const uint32_t (&msk)[kChunk][2],
                                            int t0, int ntile, int plane_stride, const uint32_t (&rot)[4],
                                            float (&va)[4]) {
#pragma unroll
  for (int tt = 0; tt < kChunk; ++tt) {
    if (tt < ntile) {
      const int t = t0 + tt;
      const int blk = (G == 16) ? t : (t >> 1);
      const int mi = (G == 16) ? 0 : (t & 1);
      uint32_t lo, hi;
      gather_fixed<B>(pbase + blk * 32, plane_stride, rot, lo, hi);
      const uint8_t* rb = rbase + t * 64;
      const uint32_t s0 = *reinterpret_cast<const uint32_t*>(rb) & msk[tt][0];
      const uint32_t s1 = *reinterpret_cast<const uint32_t*>(rb + 32) & msk[tt][1];
      const uint32_t bj[2] = {hmul2_u32(pb[tt][0], s0), hmul2_u32(pb[tt][1], s1)};
      uint32_t av[4];
      code_frag_v<G>(lo, hi, B > 4, mi, av);
      mma_m16n8k16(va, av, bj);
    }
  }
}

template <int G, int NT>
__global__ void __launch_bounds__(kDecWarps * 32) split_kernel(const DecodeArgs A) {
  const CodecDev* __restrict__ cd = A.cd;
  const int split = blockIdx.x, a = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, t4 = lane & 3;
  pdl_launch_dependents();
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmBars) + warp * 8;
  uint2* bq_s = reinterpret_cast<uint2*>(smem + kSmBq);              // [row][lane]
  int4* grp_s = reinterpret_cast<int4*>(smem + kSmGrp);              // [0..7] K, [8..15] V
  int* misc_s = reinterpret_cast<int*>(smem + kSmMisc);
  float4* vacc_s = reinterpret_cast<float4*>(smem + kSmAcc) + warp * kMaxG * 32;  // [j][lane]
  uint8_t* region = smem + kSmStages;
  uint8_t* my_stages = region + (size_t)warp * A.stages * A.stage_bytes;

  const int P = cd->P, gq = cd->gq;
  const HeadDev* hd = &cd->head[a];
  const int sec_off = hd->sec_off, sec_bytes = hd->sec_bytes;
  const int plane_stride = P * G / 8;
  // the cache (written by the preceding encode) is complete once this grid runs:
  // the fold it depends on started only after the encode finished
  const int len = A.lengths[b];
  const int n_pages = (len + P - 1) / P;
  const int per = (n_pages + A.n_split - 1) / A.n_split;
  const int p0 = min(split * per, n_pages), p1 = min(p0 + per, n_pages);
  const int count = (p1 - p0 > warp) ? (p1 - p0 - warp + kDecWarps - 1) / kDecWarps : 0;
  const SideDev* sk = &hd->side[0];
  const SideDev* sv = &hd->side[1];
  const int nK = sk->n_groups, nV = sv->n_groups;

  // ---- 1. page ids of this warp, then its first bulk copies -----------------
  bool bad = false;
  for (int i = lane; i < count; i += 32) {
    const int pid = A.page_table[(size_t)b * A.max_pages + p0 + warp + kDecWarps * i];
    bad |= (pid < 0 || (int64_t)pid >= A.n_pool_pages);
  }
  const bool warp_bad = __any_sync(0xffffffffu, bad);
  if (warp_bad && lane == 0) device_error(cd->err, SPECTRA_ERR_INVALID);
  const int my_count = warp_bad ? 0 : count;
  const int S = A.stages;
  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  auto issue = [&](int i) {
    const int pg = p0 + warp + kDecWarps * i;
    const int pid = A.page_table[(size_t)b * A.max_pages + pg];
    const uint8_t* src = A.pool + (size_t)pid * (size_t)A.page_bytes + sec_off;
    uint64_t* bar = &bars[i % S];
    mbar_arrive_expect_tx(bar, (uint32_t)sec_bytes);
    bulk_copy_g2s(my_stages + (size_t)(i % S) * A.stage_bytes, src, (uint32_t)sec_bytes, bar);
  };
  if (lane == 0)
    for (int i = 0; i < min(S, my_count); ++i) issue(i);

  if (tid < 2 * kMaxG) {
    const bool isv = tid >= kMaxG;
    const int j = tid & (kMaxG - 1);
    const SideDev* sd = isv ? sv : sk;
    int4 g = make_int4(0, 0, 0, 0);
    if (j < sd->n_groups) {
      const GroupDev gd = sd->grp[j];
      g = make_int4(gd.plane_off - sec_off, gd.plane_off - sec_off + gd.b * plane_stride, gd.b, 0);
    }
    grp_s[tid] = g;
  }
  for (int j = 0; j < kMaxG; ++j) vacc_s[j * 32 + lane] = make_float4(0.f, 0.f, 0.f, 0.f);

  // ---- 2. the folded query (written by the fold grid) -----------------------
  pdl_wait();
  {
    const uint2* src = A.frag + ((size_t)b * A.n_kv + a) * kFragWords;
    for (int e = tid; e < kFragWords; e += blockDim.x) bq_s[e] = src[e];
  }
  __syncthreads();
  if (tid < kMaxG) misc_s[tid] = (tid < nV) ? grp_s[kMaxG + tid].y : -1;  // V record offsets by group
  __syncthreads();
  uint32_t bz[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const uint2 v = bq_s[(kMaxG * 2 + nt) * 32 + lane];
    bz[nt][0] = v.x;
    bz[nt][1] = v.y;
  }
  uint32_t rot[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) rot[p] = (uint32_t)(t4 - p) & 31u;
  const int vrec_mine = misc_s[gid];  // record offset of V group `gid` (-1 if none)
  const int krecA = (2 * t4 < nK) ? grp_s[2 * t4].y : -1;          // K groups 2*t4, 2*t4+1
  const int krecB = (2 * t4 + 1 < nK) ? grp_s[2 * t4 + 1].y : -1;

  float m_run[NT], l_run[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt] = -CUDART_INF_F;
    l_run[nt] = 0.f;
  }
  float dz[4] = {0.f, 0.f, 0.f, 0.f};

  // ---- 3. stream this warp's pages in chunks of 64 tokens -------------------
  bool timed_out = false;
  int i = 0;
  for (; i < my_count; ++i) {
    const int s = i % S;
    const bool ok = mbar_wait_bounded(&bars[s], (uint32_t)((i / S) & 1), kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ok)) {
      timed_out = true;
      break;
    }
    const uint8_t* sec = my_stages + (size_t)s * A.stage_bytes;
    const int pg = p0 + warp + kDecWarps * i;
    const int n_valid = min(P, len - pg * P);
    const int n_tiles = (n_valid + 15) >> 4;
#pragma unroll 1
    for (int t0 = 0; t0 < n_tiles; t0 += kChunk) {
      const int ntile = min(kChunk, n_tiles - t0);
      // keys
      float acc[kChunk][NT][4];
#pragma unroll
      for (int tt = 0; tt < kChunk; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[tt][nt][r] = 0.f;
#pragma unroll 1
      for (int j = 0; j < nK; ++j) {
        const int4 g = grp_s[j];
        uint2 bqj[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) bqj[nt] = bq_s[(j * NT + nt) * 32 + lane];
        const uint8_t* pbase = sec + g.x + gid * 4;
        const uint8_t* rbase = sec + g.y + gid * 8;
        switch (g.z) {
          case 1: key_group<G, NT, 1>(pbase, rbase, bqj, t0, ntile, plane_stride, rot, acc); break;
          case 2: key_group<G, NT, 2>(pbase, rbase, bqj, t0, ntile, plane_stride, rot, acc); break;
          case 3: key_group<G, NT, 3>(pbase, rbase, bqj, t0, ntile, plane_stride, rot, acc); break;
          case 4: key_group<G, NT, 4>(pbase, rbase, bqj, t0, ntile, plane_stride, rot, acc); break;
          default: key_group<G, NT, 8>(pbase, rbase, bqj, t0, ntile, plane_stride, rot, acc); break;
        }
      }
      // z term of the keys (k = group index) and the scores
      float sc[kChunk][NT][2];
#pragma unroll
      for (int tt = 0; tt < kChunk; ++tt) {
        const int t = t0 + tt;
        const int nv = n_valid - t * 16;
        if (tt < ntile) {
          const uint32_t zA = krecA >= 0 ? *reinterpret_cast<const uint32_t*>(sec + krecA + (t * 8 + gid) * 8 + 4) : 0u;
          const uint32_t zB = krecB >= 0 ? *reinterpret_cast<const uint32_t*>(sec + krecB + (t * 8 + gid) * 8 + 4) : 0u;
          const uint32_t az[4] = {__byte_perm(zA, zB, 0x5410), __byte_perm(zA, zB, 0x7632), 0u, 0u};
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            float d[4];
            mma_m16n8k16_z(d, az, bz[nt]);
            sc[tt][nt][0] = fmaf(acc[tt][nt][0] + acc[tt][nt][1], kTwo24, d[0] + d[1]);
            sc[tt][nt][1] = fmaf(acc[tt][nt][2] + acc[tt][nt][3], kTwo24, d[2] + d[3]);
            if (2 * gid >= nv) sc[tt][nt][0] = -CUDART_INF_F;
            if (2 * gid + 1 >= nv) sc[tt][nt][1] = -CUDART_INF_F;
          }
        } else {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) sc[tt][nt][0] = sc[tt][nt][1] = -CUDART_INF_F;
        }
      }
      // online softmax (log2 units); rescale only when a running max grows
      float mt[NT];
      bool grow = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int tt = 0; tt < kChunk; ++tt) mx = fmaxf(mx, fmaxf(sc[tt][nt][0], sc[tt][nt][1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        mt[nt] = mx;
        grow |= mx > m_run[nt];
      }
      const bool grew = __any_sync(0xffffffffu, grow);
      float ae = 1.f, ao = 1.f;
      if (grew) {
        float alpha[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float m_new = fmaxf(m_run[nt], mt[nt]);
          alpha[nt] = exp2f(m_run[nt] - m_new);
          m_run[nt] = m_new;
          l_run[nt] *= alpha[nt];
        }
        // value accumulators hold heads 2*t4 and 2*t4+1
        ae = __shfl_sync(0xffffffffu, alpha[0], (2 * t4) & 3);
        ao = __shfl_sync(0xffffffffu, alpha[0], (2 * t4 + 1) & 3);
        if (NT == 2) {
          const float be = __shfl_sync(0xffffffffu, alpha[NT - 1], (2 * t4) & 3);
          const float bo = __shfl_sync(0xffffffffu, alpha[NT - 1], (2 * t4 + 1) & 3);
          if (t4 >= 2) {
            ae = be;
            ao = bo;
          }
        }
        dz[0] *= ae;
        dz[1] *= ao;
      }
      // p as the B operand (tokens x heads): lane (gid, t4) needs head gid,
      // tokens (2t4, 2t4+1) and (2t4+8, 2t4+9)
      uint32_t pb[kChunk][2];
      uint32_t msk[kChunk][2];
      const int src0 = (t4 << 2) | (gid & 3), src1 = ((t4 + 4) << 2) | (gid & 3);
#pragma unroll
      for (int tt = 0; tt < kChunk; ++tt) {
        uint32_t p01[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float pa = exp2f(sc[tt][nt][0] - m_run[nt] + kPScaleLog2);
          const float pv = exp2f(sc[tt][nt][1] - m_run[nt] + kPScaleLog2);
          l_run[nt] += pa + pv;
          p01[nt] = pack_half2(pa, pv);
        }
        pb[tt][0] = __shfl_sync(0xffffffffu, p01[0], src0);
        pb[tt][1] = __shfl_sync(0xffffffffu, p01[0], src1);
        if (NT == 2) {
          const uint32_t y0 = __shfl_sync(0xffffffffu, p01[NT - 1], src0);
          const uint32_t y1 = __shfl_sync(0xffffffffu, p01[NT - 1], src1);
          if (gid >= 4) {
            pb[tt][0] = y0;
            pb[tt][1] = y1;
          }
        }
        if (gid >= gq) pb[tt][0] = pb[tt][1] = 0u;
        // tokens past the end: their records may hold anything; zero their s and z
        const int nv = n_valid - (t0 + tt) * 16;
        msk[tt][0] = msk[tt][1] = 0xffffffffu;
        if (nv < 16) {
          msk[tt][0] = ((2 * t4 < nv) ? 0x0000ffffu : 0u) | ((2 * t4 + 1 < nv) ? 0xffff0000u : 0u);
          msk[tt][1] = ((2 * t4 + 8 < nv) ? 0x0000ffffu : 0u) | ((2 * t4 + 9 < nv) ? 0xffff0000u : 0u);
        }
      }
      // values: per group, sum_t (p_t s_t,j) code_t,j ...
#pragma unroll 1
      for (int j = 0; j < nV; ++j) {
        const int4 g = grp_s[kMaxG + j];
        const float4 v4 = vacc_s[j * 32 + lane];
        float va[4] = {v4.x * ae, v4.y * ao, v4.z * ae, v4.w * ao};
        const uint8_t* pbase = sec + g.x + gid * 4;
        const uint8_t* rbase = sec + g.y + t4 * 8;
        switch (g.z) {
          case 1: value_group<G, 1>(pbase, rbase, pb, msk, t0, ntile, plane_stride, rot, va); break;
          case 2: value_group<G, 2>(pbase, rbase, pb, msk, t0, ntile, plane_stride, rot, va); break;
          case 3: value_group<G, 3>(pbase, rbase, pb, msk, t0, ntile, plane_stride, rot, va); break;
          case 4: value_group<G, 4>(pbase, rbase, pb, msk, t0, ntile, plane_stride, rot, va); break;
          default: value_group<G, 8>(pbase, rbase, pb, msk, t0, ntile, plane_stride, rot, va); break;
        }
        vacc_s[j * 32 + lane] = make_float4(va[0], va[1], va[2], va[3]);
      }
      // ... plus sum_t p_t z_t,j for all groups (rows = groups)
#pragma unroll
      for (int tt = 0; tt < kChunk; ++tt) {
        if (tt < ntile) {
          uint32_t az[4] = {0u, 0u, 0u, 0u};
          if (vrec_mine >= 0) {
            const uint8_t* rb = sec + vrec_mine + (t0 + tt) * 64;
            az[0] = *reinterpret_cast<const uint32_t*>(rb + t4 * 8 + 4) & msk[tt][0];
            az[2] = *reinterpret_cast<const uint32_t*>(rb + (t4 + 4) * 8 + 4) & msk[tt][1];
          }
          mma_m16n8k16(dz, az, pb[tt]);
        }
      }
    }
    __syncwarp();
    if (lane == 0 && i + S < my_count) {
      fence_proxy_async_smem();
      issue(i + S);
    }
  }
  if (timed_out) {
    if (lane == 0) {
      device_error(cd->err, SPECTRA_ERR_TIMEOUT);
      for (int k = i; k < min(i + S, my_count); ++k)  // let copies still in flight land
        mbar_wait_bounded(&bars[k % S], (uint32_t)((k / S) & 1), kWaitLimitNs);
    }
    __syncwarp();
  }

  // sum of p over the 8 lanes that share a head
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float l = l_run[nt];
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    l_run[nt] = l;
  }

  // ---- 4. merge the warps of this CTA into one partial record per q head ----
  __syncthreads();
  const int nkv = sv->n_kept;
  const int rec = 2 + kMaxKept;
  float* wsm = reinterpret_cast<float*>(region);
  if (gid == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hl = nt * 4 + t4;
      if (hl < gq) {
        wsm[(warp * gq + hl) * rec + 0] = m_run[nt];
        wsm[(warp * gq + hl) * rec + 1] = l_run[nt];
      }
    }
  }
  for (int j = 0; j < nV; ++j) {
    const float4 v4 = vacc_s[j * 32 + lane];
    const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int hl = 2 * t4 + (c & 1);
      const int coord = j * G + gid + ((c >> 1) ? 8 : 0);
      if (hl < gq && (G == 16 || c < 2)) wsm[(warp * gq + hl) * rec + 2 + coord] = vv[c] * kTwo24;
    }
  }
  __syncwarp();
  if (gid < nV) {  // z term of group gid, heads 2*t4 and 2*t4+1
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int hl = 2 * t4 + c;
      if (hl < gq)
        for (int k = 0; k < G; ++k) wsm[(warp * gq + hl) * rec + 2 + gid * G + k] += dz[c];
    }
  }
  __syncthreads();
  float* part = A.part + ((size_t)(b * A.n_q + a * gq) * A.n_split + split) * A.part_stride;
  for (int idx = tid; idx < gq * (2 + nkv); idx += blockDim.x) {
    const int hl = idx / (2 + nkv), c = idx % (2 + nkv);
    float M = -CUDART_INF_F;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wsm[(w * gq + hl) * rec]);
    float v = 0.f;
    if (c == 0) {
      v = M;
    } else if (M != -CUDART_INF_F) {
      for (int w = 0; w < kDecWarps; ++w) {
        const float mw = wsm[(w * gq + hl) * rec];
        if (mw != -CUDART_INF_F) v += exp2f(mw - M) * wsm[(w * gq + hl) * rec + c];
      }
    }
    part[(size_t)hl * A.n_split * A.part_stride + c] = v;
  }
}

// ---------------------------------------------------------------------------
// combine: out = (sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s) W_up^V
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const DecodeArgs A) {
  const CodecDev* __restrict__ cd = A.cd;
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
  const int gq = cd->gq, d_h = cd->d_h;
  const int a = h / gq;
  const SideDev* sv = &cd->head[a].side[1];
  const int nkv = sv->n_kept, ns = A.n_split, stride = A.part_stride;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  float* red = reinterpret_cast<float*>(smem + 64);      // 32 floats
  float* olat = red + 32;                                // [kMaxKept]
  float* wgt = olat + kMaxKept;                          // [kMaxSplit]
  float* w_s = wgt + kMaxSplit;                          // [nkv][d_h]
  float* p_s = w_s + kMaxKept * kMaxDHead;               // [ns][stride]
  const uint32_t wbytes = (uint32_t)nkv * d_h * 4;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    if (wbytes) {
      mbar_arrive_expect_tx(bar, wbytes);
      bulk_copy_g2s(w_s, cd->w_up + sv->wup_off, wbytes, bar);
    }
  }
  pdl_wait();  // the split partials are complete from here on
  const float* pr = A.part + ((size_t)b * A.n_q + h) * ns * stride;
  for (int e = tid; e < ns * stride; e += blockDim.x) p_s[e] = pr[e];
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  float mloc = -CUDART_INF_F;
  for (int s = tid; s < ns; s += blockDim.x) mloc = fmaxf(mloc, p_s[s * stride]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
  if (lane == 0) red[warp] = mloc;
  __syncthreads();
  float M = -CUDART_INF_F;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) M = fmaxf(M, red[w]);
  __syncthreads();
  float lloc = 0.f;
  for (int s = tid; s < ns; s += blockDim.x) {
    const float ms = p_s[s * stride];
    const float w = (M == -CUDART_INF_F || ms == -CUDART_INF_F) ? 0.f : exp2f(ms - M);
    wgt[s] = w;
    lloc += w * p_s[s * stride + 1];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lloc += __shfl_xor_sync(0xffffffffu, lloc, o);
  if (lane == 0) red[warp] = lloc;
  __syncthreads();
  float L = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) L += red[w];
  const float invL = L > 0.f ? 1.f / L : 0.f;
  for (int c = tid; c < nkv; c += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < ns; ++s) acc = fmaf(wgt[s], p_s[s * stride + 2 + c], acc);
    olat[c] = acc * invL;
  }
  __syncthreads();
  bool ok = true;
  if (wbytes) ok = mbar_wait_bounded(bar, 0, kWaitLimitNs);
  if (!ok && tid == 0) device_error(cd->err, SPECTRA_ERR_TIMEOUT);
  float* orow = A.out + ((size_t)b * A.n_q + h) * d_h;
  for (int d = tid; d < d_h; d += blockDim.x) {
    float acc = 0.f;
    for (int c = 0; c < nkv; ++c) acc = fmaf(olat[c], w_s[c * d_h + d], acc);
    orow[d] = ok ? acc : 0.f;
  }
}

int fold_smem_bytes() { return 128 + (kMaxGQ * kMaxKept + kMaxGQ * kMaxG + kMaxGQ * kMaxDHead) * 4 + kMaxKept * kMaxDHead * 4; }
int combine_smem_bytes(int ns, int stride) {
  return 64 + (32 + kMaxKept + kMaxSplit + kMaxKept * kMaxDHead) * 4 + ns * stride * 4;
}

// Launch with programmatic stream serialisation (the kernel may start while the
// previous one in the stream finishes; it waits with griddepcontrol.wait).  If
// the attribute is refused, launch plainly: griddepcontrol.wait is then a no-op.
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

template <int G, int NT>
int split_occupancy(int smem) {
  int n = 0;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(split_kernel<G, NT>), smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, split_kernel<G, NT>, kDecWarps * 32, smem) != cudaSuccess ||
      n <= 0)
    n = 1;
  return n;
}

int split_ctas_per_sm(int group, bool two_tiles, int smem) {
  if (group == 16) return two_tiles ? split_occupancy<16, 2>(smem) : split_occupancy<16, 1>(smem);
  return two_tiles ? split_occupancy<8, 2>(smem) : split_occupancy<8, 1>(smem);
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

template <int G, int NT>
cudaError_t launch_all(const DecodeArgs& args, const DecodePlan& plan, int batch, int n_kv, int n_q, cudaStream_t st) {
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(fold_kernel<G, NT>), fold_smem_bytes());
  if (e != cudaSuccess) return e;
  e = ensure_dynamic_smem(reinterpret_cast<const void*>(split_kernel<G, NT>), plan.smem_bytes);
  if (e != cudaSuccess) return e;
  const int csm = combine_smem_bytes(args.n_split, args.part_stride);
  e = ensure_dynamic_smem(reinterpret_cast<const void*>(combine_kernel), csm);
  if (e != cudaSuccess) return e;
  fold_kernel<G, NT><<<dim3(n_kv, batch), 256, fold_smem_bytes(), st>>>(args);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_dependent(split_kernel<G, NT>, dim3(args.n_split, n_kv, batch), dim3(kDecWarps * 32), plan.smem_bytes,
                       st, args);
  if (e != cudaSuccess) return e;
  return launch_dependent(combine_kernel, dim3(n_q, batch), dim3(256), csm, st, args);
}

}  // namespace

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device.  One record per (kernel, device): the limit only ever grows,
// so a launch never meets a limit that another caller lowered.
cudaError_t ensure_dynamic_smem(const void* kern, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  int& cur = done[{kern, dev}];
  if (bytes <= cur) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) cur = bytes;
  return e;
}

DecodePlan make_decode_plan(const CodecDev& h, int batch, int max_pages_per_seq) {
  DecodePlan p{};
  p.stage_bytes = std::max(16, ((h.max_sec_bytes + 15) / 16) * 16);
  // 2 stages per warp (more when sections are small) keep > 40 KB in flight per SM
  const int budget = 64 * 1024;
  p.stages = std::max(2, std::min(4, budget / (kDecWarps * p.stage_bytes)));
  const int merge_bytes = kDecWarps * h.gq * (2 + kMaxKept) * 4;
  p.smem_bytes = kSmStages + std::max(kDecWarps * p.stages * p.stage_bytes, merge_bytes);
  // context splits: fill one wave of resident CTAs when that wastes < 15% of the
  // slots, else two waves; the count does not depend on the context length, so a
  // workspace sized once fits every call (the call clamps it to the cache's pages)
  const int units = std::max(1, batch * h.n_kv);
  const int slots = split_ctas_per_sm(h.group, h.gq > 4, p.smem_bytes) * sm_count();
  int ns = std::max(1, slots / units);
  if ((double)units * ns / slots < 0.85) {
    const int ns2 = std::max(1, 2 * slots / units);
    if ((double)units * ns2 / (2.0 * slots) > (double)units * ns / slots) ns = ns2;
  }
  ns = std::min(ns, kMaxSplit);
  (void)max_pages_per_seq;
  p.n_split = ns;
  p.part_stride = ((2 + h.max_kept_v) + 3) / 4 * 4;
  size_t off = 0;
  auto carve = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  };
  p.frag_off = carve((size_t)batch * h.n_kv * kFragWords * 8);
  p.part_off = carve((size_t)batch * h.n_q * ns * p.part_stride * 4);
  p.ws_bytes = off;
  return p;
}

cudaError_t launch_decode(const CodecDev& h, const CodecDev* d, const spectra_cache& cache, const float* q,
                          float* out, void* ws, const DecodePlan& plan, cudaStream_t st) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  DecodeArgs args;
  args.cd = d;
  args.pool = static_cast<const uint8_t*>(cache.pool);
  args.page_table = cache.page_table;
  args.lengths = cache.lengths;
  args.q = q;
  args.out = out;
  args.part = reinterpret_cast<float*>(w + plan.part_off);
  args.frag = reinterpret_cast<uint2*>(w + plan.frag_off);
  args.n_pool_pages = cache.n_pages;
  args.page_bytes = h.page_bytes;
  args.max_pages = cache.max_pages_per_seq;
  args.n_split = std::max(1, std::min(plan.n_split, cache.max_pages_per_seq));
  args.stages = plan.stages;
  args.stage_bytes = plan.stage_bytes;
  args.part_stride = plan.part_stride;
  args.n_q = h.n_q;
  args.n_kv = h.n_kv;
  args.q_scale = 1.4426950408889634f / sqrtf((float)h.d_h);
  const bool two = h.gq > 4;
  if (h.group == 16)
    return two ? launch_all<16, 2>(args, plan, cache.batch, h.n_kv, h.n_q, st)
               : launch_all<16, 1>(args, plan, cache.batch, h.n_kv, h.n_q, st);
  return two ? launch_all<8, 2>(args, plan, cache.batch, h.n_kv, h.n_q, st)
             : launch_all<8, 1>(args, plan, cache.batch, h.n_kv, h.n_q, st);
}

}  // namespace spectra
