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
//           (bulk copies into per-warp shared-memory stages, the first ones
//           issued while the fold runs) through an online softmax over
//           64-token chunks; one partial record (max, sum, latent accumulator)
//           per q head;
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
constexpr int kMaxSplit = 256;    // context splits per (sequence, KV head)
constexpr int kMaxSmemPerBlock = 227 * 1024;  // opt-in dynamic shared memory per CTA (sm_100)
constexpr uint64_t kWaitLimitNs = 200ull * 1000ull * 1000ull;  // bounded mbarrier waits
constexpr float kPScaleLog2 = 8.f;   // p = 2^(s - m + 8): fp16 keeps small weights normal
constexpr float kTwo24 = 16777216.f; // undo the 2^-24 of subnormal codes
constexpr float kTwo20 = 1048576.f;  // the same for codes held at nibble bits 4-7 (x16)
constexpr int kFragWords = (kMaxG * 2 + 2) * 32;  // uint2 per (sequence, KV head): bq[j][nt], bz[nt]

// split kernel shared-memory carve-up (bytes)
constexpr int kSmBars = 0;                                   // 4 warps x 8 mbarriers
constexpr int kSmBq = 512;                                   // fragments [kMaxG*2 + 2][32] uint2
constexpr int kSmGrp = kSmBq + kFragWords * 8;               // group tables (448 B)
constexpr int kSmAcc = kSmGrp + 512;                         // value accumulators [warp][kMaxG][32] float4
constexpr int kSmStages = kSmAcc + kDecWarps * kMaxG * 32 * 16;
constexpr int kMergeBytes = (kDecWarps * kMaxGQ * (2 + kMaxKept) + kMaxGQ * (kDecWarps + 2)) * 4;

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
  int max_kept_v;
  int d_h;
  float q_scale;
};


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

// 2^x for x <= 0 (and up to 2^8 for the scaled softmax weights); flushes
// results below 2^-126 to zero.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 16-byte asynchronous global -> shared copy (both addresses 16-byte aligned)
// and the wait for all of this thread's outstanding copies.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }


// ---------------------------------------------------------------------------
// fold: q_lat[h][c] = (q_h . W_up^K[c]) * log2(e)/sqrt(d_h) and group sums, as
// B fragments: bq[j][nt][lane] column n = lane/4 of n-tile nt is q head
// nt*4 + n/2, part n&1 (0: fp16(q_lat), 1: fp16(q_lat - fp16(q_lat))); rows
// k = 2*(lane%4) + {0,1} (+8).  bz[nt][lane] likewise over group sums.
// ---------------------------------------------------------------------------
//
// One CTA per (KV head, sequence, quarter z of the kept K coordinates): lane c
// of each warp owns coordinate 32 z + c, warp w heads w and w + 4.  A quarter
// holds whole groups (2 of 16 or 4 of 8), so the CTA writes every fragment of
// its groups, and the bz lanes whose rows (2 t4, 2 t4 + 1) are its groups.
// ---------------------------------------------------------------------------
constexpr int kFoldThreads = 128;

template <int G, int NT>
__global__ void __launch_bounds__(kFoldThreads) fold_kernel(const DecodeArgs A) {
  const CodecDev* __restrict__ cd = A.cd;
  const int a = blockIdx.x, b = blockIdx.y, z = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_launch_dependents();
  __shared__ float q_s[kMaxGQ * kMaxDHead];
  __shared__ float qlat_s[kMaxGQ][33];
  __shared__ __align__(16) float w_s[kMaxDHead * 32];  // this quarter's columns of W_up^K
  const int gq = cd->gq, d_h = cd->d_h;
  const SideDev* sk = &cd->head[a].side[0];
  const int nk = sk->n_kept, nK = sk->n_groups;
  const float* w = cd->w_up + sk->wup_off;  // [d_h][nk]; nk is a multiple of 8
  // all 16-byte pieces of the quarter in flight at once
  for (int e = tid; e < d_h * 8; e += kFoldThreads) {
    const int d = e >> 3, c4 = 32 * z + 4 * (e & 7);
    if (c4 < nk) cp_async16(w_s + d * 32 + 4 * (e & 7), w + (size_t)d * nk + c4);
  }
  const float* qb = A.q + ((size_t)b * A.n_q + (size_t)a * gq) * d_h;
  for (int e = tid; e < gq * d_h; e += kFoldThreads) q_s[e] = qb[e];
  cp_async_wait_all();
  __syncthreads();
  const int c = 32 * z + lane;
  float acc0 = 0.f, acc1 = 0.f;
  const int h0 = warp, h1 = warp + 4;
  if (c < nk) {
    const float* q0 = q_s + h0 * d_h;
    const float* q1 = q_s + (h1 < gq ? h1 : h0) * d_h;
#pragma unroll 8
    for (int d = 0; d < d_h; ++d) {
      const float wv = w_s[d * 32 + lane];
      acc0 = fmaf(q0[d], wv, acc0);
      acc1 = fmaf(q1[d], wv, acc1);
    }
  }
  qlat_s[h0][lane] = acc0 * A.q_scale;
  qlat_s[h1][lane] = acc1 * A.q_scale;
  __syncthreads();
  pdl_wait();  // the fragment buffer may still be read by an earlier decode's split kernel
  // fragments of this quarter's groups
  constexpr int kGroupsPerQ = 32 / G;
  uint2* out = A.frag + ((size_t)b * A.n_kv + a) * kFragWords;
  for (int idx = tid; idx < kGroupsPerQ * NT * 32; idx += kFoldThreads) {
    const int ln = idx % 32, r = idx / 32;
    const int jl = r / NT, nt = r % NT;
    const int j = z * kGroupsPerQ + jl;
    if (j >= kMaxG) continue;
    const int gid = ln >> 2, t4 = ln & 3;
    const int hl = nt * 4 + (gid >> 1), part = gid & 1;
    auto split_h = [&](float x) -> float {
      const float hi = __half2float(__float2half_rn(x));
      return part ? (x - hi) : hi;
    };
    uint2 v = make_uint2(0u, 0u);
    if (hl < gq && j < nK) {
      const float* base = &qlat_s[hl][jl * G];
      v.x = pack_half2(split_h(base[2 * t4]), split_h(base[2 * t4 + 1]));
      if (G == 16) v.y = pack_half2(split_h(base[2 * t4 + 8]), split_h(base[2 * t4 + 9]));
    }
    out[(j * NT + nt) * 32 + ln] = v;
  }
  // bz rows k = 2 t4, 2 t4 + 1 are groups; lanes whose groups lie in this quarter
  for (int idx = tid; idx < NT * 32; idx += kFoldThreads) {
    const int ln = idx % 32, nt = idx / 32;
    const int gid = ln >> 2, t4 = ln & 3;
    const int j0 = 2 * t4;
    if (j0 / kGroupsPerQ != z) continue;
    const int hl = nt * 4 + (gid >> 1), part = gid & 1;
    auto gsum = [&](int j) -> float {
      float s = 0.f;
      if (j < nK)
        for (int k = 0; k < G; ++k) s += qlat_s[hl][(j - z * kGroupsPerQ) * G + k];
      return s;
    };
    auto split_h = [&](float x) -> float {
      const float hi = __half2float(__float2half_rn(x));
      return part ? (x - hi) : hi;
    };
    uint2 v = make_uint2(0u, 0u);
    if (hl < gq) v.x = pack_half2(split_h(gsum(j0)), split_h(gsum(j0 + 1)));
    out[(kMaxG * 2 + nt) * 32 + ln] = v;
  }
}

// ---------------------------------------------------------------------------
// split: one context split of one (sequence, KV head)
// ---------------------------------------------------------------------------

// Fragment registers of one 256-entry block of a group with width B.  The
// block's bytes hold, for every MMA lane, its 8 codes (slots 0..7, see the page
// layout): B = 4: word `lane` holds them as nibbles; B = 2: word 2*gid + t4/2,
// bits 2*(t4%2) + {0,1} of each nibble; B = 1: word gid, bit t4 of each nibble;
// B = 3: a B = 2 part (16 words, code bits 0-1) then a B = 1 part (8 words,
// code bit 2); B = 8: words 2*lane, 2*lane+1 hold bytes [s0 s1 s4 s5] [s2 s3 s6 s7].
// A nibble-held code is used in place: as an fp16 bit pattern, bits 0-3 of a
// 16-bit lane are the subnormal code * 2^-24 and bits 4-7 are code * 16 * 2^-24.
// So registers a1, a3 (MMA rows gid+8) carry a factor 16 for B <= 4.
template <int B>
__device__ __forceinline__ uint32_t nibble_codes(const uint8_t* __restrict__ p, const uint8_t* __restrict__ p1,
                                                 uint32_t sh, uint32_t rot1) {
  if (B == 4) return *reinterpret_cast<const uint32_t*>(p);
  if (B == 2 || B == 1) return *reinterpret_cast<const uint32_t*>(p) >> sh;
  // B == 3: code bits 0-1 from the 2-bit part, bit 2 from the 1-bit part (rotated
  // from nibble bit t4 to nibble bit 2); bit 3 of each nibble is left as junk and
  // cleared by the fragment masks
  const uint32_t lo = *reinterpret_cast<const uint32_t*>(p) >> sh;
  const uint32_t w1 = *reinterpret_cast<const uint32_t*>(p1);
  const uint32_t hi = __funnelshift_r(w1, w1, rot1);
  return (lo & 0x33333333u) | (hi & 0xCCCCCCCCu);
}

template <int B>
__device__ __forceinline__ constexpr uint32_t frag_mask() {
  return B >= 4 ? 0x000F000Fu : (B == 3 ? 0x00070007u : (B == 2 ? 0x00030003u : 0x00010001u));
}

// K side, A = codes (rows: tokens, cols: coordinates).  G = 16: m16n8k16, four
// registers; G = 8: m16n8k8, two registers for half `mi` of a 32-token block.
template <int G, int B>
__device__ __forceinline__ void frag_k(const uint8_t* __restrict__ p, const uint8_t* __restrict__ p1, uint32_t sh,
                                       uint32_t rot1, int mi, uint32_t (&av)[4]) {
  if (B == 8) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    if (G == 16) {
      av[0] = w.x & 0x00FF00FFu;
      av[1] = (w.x >> 8) & 0x00FF00FFu;
      av[2] = w.y & 0x00FF00FFu;
      av[3] = (w.y >> 8) & 0x00FF00FFu;
    } else {
      const uint32_t x = mi ? w.y : w.x;
      av[0] = x & 0x00FF00FFu;
      av[1] = (x >> 8) & 0x00FF00FFu;
    }
  } else {
    constexpr uint32_t M = frag_mask<B>();
    const uint32_t x = nibble_codes<B>(p, p1, sh, rot1);
    if (G == 16) {
      const uint32_t y = x >> 8;
      av[0] = x & M;
      av[1] = x & (M << 4);
      av[2] = y & M;
      av[3] = y & (M << 4);
    } else {
      const uint32_t y = mi ? (x >> 8) : x;
      av[0] = y & M;
      av[1] = y & (M << 4);
    }
  }
}

// V side, A = codes transposed (rows: coordinates, cols: tokens), m16n8k16.
// G = 8: rows 8..15 are zero; no factor 16 (shifts instead).
template <int G, int B>
__device__ __forceinline__ void frag_v(const uint8_t* __restrict__ p, const uint8_t* __restrict__ p1, uint32_t sh,
                                       uint32_t rot1, int mi, uint32_t (&av)[4]) {
  if (B == 8) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    if (G == 16) {
      av[0] = w.x & 0x00FF00FFu;
      av[1] = (w.x >> 8) & 0x00FF00FFu;
      av[2] = w.y & 0x00FF00FFu;
      av[3] = (w.y >> 8) & 0x00FF00FFu;
    } else {
      av[0] = (mi ? (w.x >> 8) : w.x) & 0x00FF00FFu;
      av[1] = 0u;
      av[2] = (mi ? (w.y >> 8) : w.y) & 0x00FF00FFu;
      av[3] = 0u;
    }
  } else {
    constexpr uint32_t M = frag_mask<B>();
    const uint32_t x = nibble_codes<B>(p, p1, sh, rot1);
    if (G == 16) {
      const uint32_t y = x >> 8;
      av[0] = x & M;
      av[1] = x & (M << 4);
      av[2] = y & M;
      av[3] = y & (M << 4);
    } else {
      const uint32_t xs = mi ? (x >> 4) : x;
      av[0] = xs & M;
      av[1] = 0u;
      av[2] = (xs >> 8) & M;
      av[3] = 0u;
    }
  }
}

// Lane-constant addressing of a width class: byte offset of this lane's word in
// a block (and of its 1-bit-part word for B = 3), shift and rotation.
struct LaneAddr {
  int off4, off2, off1, off8;
  uint32_t sh2, sh1, rot1;
};

template <int B>
__device__ __forceinline__ int lane_off(const LaneAddr& L) {
  return B == 4 ? L.off4 : (B == 8 ? L.off8 : ((B == 2 || B == 3) ? L.off2 : L.off1));
}
template <int B>
__device__ __forceinline__ uint32_t lane_sh(const LaneAddr& L) {
  return B == 1 ? L.sh1 : L.sh2;
}

// Keys of one kept group for the CH tiles of a chunk: acc[tt][nt] +=
// s * (q_lat,j . code) for (token row gid, token row gid+8) x (hi, lo).
// Rows gid+8 carry the factor 16 (B = 8 scales s instead).
template <int G, int NT, int CH, int B>
__device__ __forceinline__ void key_group(const uint8_t* __restrict__ blocks, const uint8_t* __restrict__ rec,
                                          const LaneAddr& L, const uint2 (&bqj)[NT], float (&acc)[CH][NT][4]) {
  const uint8_t* p = blocks + lane_off<B>(L);
  const uint8_t* p1 = blocks + 64 + L.off1;
  uint32_t sp[CH];
#pragma unroll
  for (int h = 0; h < CH / 2; ++h) {
    const uint4 r = *reinterpret_cast<const uint4*>(rec + 16 * h);  // {s, z} of 2 tiles
    sp[2 * h] = r.x;
    sp[2 * h + 1] = r.z;
  }
#pragma unroll
  for (int tt = 0; tt < CH; ++tt) {
    constexpr int kBlockTiles = G == 16 ? 1 : 2;
    const int blk = tt / kBlockTiles;
    uint32_t av[4];
    frag_k<G, B>(p + blk * (B * 32), p1 + blk * (B * 32), lane_sh<B>(L), L.rot1, tt & 1, av);
    float sA, sB;
    half2_to_floats(sp[tt], sA, sB);
    if (B == 8) sB *= 16.f;
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

// Values of one kept group for the CH tiles of a chunk: va += code^T (p s).
// recA / recB: this lane's records of token pairs t4 and t4+4.
template <int G, int CH, int B, bool kMask>
__device__ __forceinline__ void value_group(const uint8_t* __restrict__ blocks, const uint8_t* __restrict__ recA,
                                            const uint8_t* __restrict__ recB, const LaneAddr& L,
                                            const uint32_t (&pb)[CH][2], const uint32_t (&msk)[CH][2],
                                            float (&va)[4]) {
  const uint8_t* p = blocks + lane_off<B>(L);
  const uint8_t* p1 = blocks + 64 + L.off1;
  uint32_t s0[CH], s1[CH];
#pragma unroll
  for (int h = 0; h < CH / 2; ++h) {
    const uint4 ra = *reinterpret_cast<const uint4*>(recA + 16 * h);
    const uint4 rb = *reinterpret_cast<const uint4*>(recB + 16 * h);
    s0[2 * h] = ra.x;
    s0[2 * h + 1] = ra.z;
    s1[2 * h] = rb.x;
    s1[2 * h + 1] = rb.z;
  }
#pragma unroll
  for (int tt = 0; tt < CH; ++tt) {
    constexpr int kBlockTiles = G == 16 ? 1 : 2;
    const int blk = tt / kBlockTiles;
    uint32_t av[4];
    frag_v<G, B>(p + blk * (B * 32), p1 + blk * (B * 32), lane_sh<B>(L), L.rot1, tt & 1, av);
    const uint32_t a0 = kMask ? (s0[tt] & msk[tt][0]) : s0[tt];
    const uint32_t a1 = kMask ? (s1[tt] & msk[tt][1]) : s1[tt];
    const uint32_t bj[2] = {hmul2_bits(pb[tt][0], a0), hmul2_bits(pb[tt][1], a1)};
    mma_m16n8k16(va, av, bj);
  }
}

template <int G, int NT, int CH, int B>
__device__ __forceinline__ void key_class(const DecodeTables& T, const uint8_t* sec, int chunk_blk_bytes_unit,
                                          int rec_lane, const LaneAddr& L, const uint2* bq_s, int lane,
                                          int ci, float (&acc)[CH][NT][4]) {
  const int c1 = T.cls[0][ci + 1];
#pragma unroll 1
  for (int c = T.cls[0][ci]; c < c1; ++c) {
    const int4 g = *reinterpret_cast<const int4*>(T.ord[0][c]);
    uint2 bqj[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) bqj[nt] = bq_s[(g.z * NT + nt) * 32 + lane];
    key_group<G, NT, CH, B>(sec + g.x + chunk_blk_bytes_unit * B, sec + g.y + rec_lane, L, bqj, acc);
  }
}

template <int G, int CH, int B, bool kMask>
__device__ __forceinline__ void value_class(const DecodeTables& T, const uint8_t* sec, int chunk_blk_bytes_unit,
                                            int recA_lane, int recB_lane, const LaneAddr& L, float4* vacc,
                                            int lane, int ci, bool grew, float ae, float ao,
                                            const uint32_t (&pb)[CH][2], const uint32_t (&msk)[CH][2]) {
  const int c1 = T.cls[1][ci + 1];
#pragma unroll 1
  for (int c = T.cls[1][ci]; c < c1; ++c) {
    const int4 g = *reinterpret_cast<const int4*>(T.ord[1][c]);
    float4 v4 = vacc[g.z * 32 + lane];
    if (grew) {
      v4.x *= ae;
      v4.y *= ao;
      v4.z *= ae;
      v4.w *= ao;
    }
    float va[4] = {v4.x, v4.y, v4.z, v4.w};
    value_group<G, CH, B, kMask>(sec + g.x + chunk_blk_bytes_unit * B, sec + g.y + recA_lane, sec + g.y + recB_lane,
                                 L, pb, msk, va);
    vacc[g.z * 32 + lane] = make_float4(va[0], va[1], va[2], va[3]);
  }
}

template <int G, int NT, int CH>
__global__ void __launch_bounds__(kDecWarps * 32) split_kernel(const DecodeArgs A) {
  const CodecDev* __restrict__ cd = A.cd;
  const int split = blockIdx.x, a = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, t4 = lane & 3;
  pdl_launch_dependents();
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmBars) + warp * 8;
  uint2* bq_s = reinterpret_cast<uint2*>(smem + kSmBq);
  DecodeTables& T = *reinterpret_cast<DecodeTables*>(smem + kSmGrp);
  float4* vacc_s = reinterpret_cast<float4*>(smem + kSmAcc) + warp * kMaxG * 32;
  uint8_t* region = smem + kSmStages;
  uint8_t* my_stages = region + (size_t)warp * A.stages * A.stage_bytes;

  const int P = cd->P, gq = cd->gq;
  const int tpp = P / 16;  // tiles per page
  const HeadDev* hd = &cd->head[a];
  const int sec_off = hd->sec_off, sec_bytes = hd->sec_bytes;
  const SideDev* sk = &hd->side[0];
  const SideDev* sv = &hd->side[1];
  const int nK = sk->n_groups, nV = sv->n_groups;
  const int S = A.stages;
  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  // pages per split: a multiple of the warp count, so the warps of a CTA get
  // equal shares (trailing splits may get fewer pages or none)
  auto page_range = [&](int len_, int& p0_, int& count_) {
    const int n_pages = (len_ + P - 1) / P;
    const int per = ((n_pages + A.n_split - 1) / A.n_split + kDecWarps - 1) / kDecWarps * kDecWarps;
    p0_ = min(split * per, n_pages);
    const int p1_ = min(p0_ + per, n_pages);
    count_ = (p1_ - p0_ > warp) ? (p1_ - p0_ - warp + kDecWarps - 1) / kDecWarps : 0;
  };

  auto issue_page = [&](int pg, int i) {
    const int pid = A.page_table[(size_t)b * A.max_pages + pg];
    const uint8_t* src = A.pool + (size_t)pid * (size_t)A.page_bytes + sec_off;
    uint64_t* bar = &bars[i % S];
    mbar_arrive_expect_tx(bar, (uint32_t)sec_bytes);
    bulk_copy_g2s(my_stages + (size_t)(i % S) * A.stage_bytes, src, (uint32_t)sec_bytes, bar);
  };

  // ---- 1. speculative first copies ------------------------------------------
  // Every kernel of the chain lets its successor start at its own start, so up
  // to the dependency wait below an encode's commit kernel may still be
  // advancing the length: the length read here is a hint.  The pages are
  // final: each kernel that writes pages lets no successor start before its
  // writes are complete (the commit kernel triggers only after its own wait on
  // the fused encode; the quantise kernel does not trigger early), and the
  // page table is written by no kernel.  The first copies go out for the
  // hint's page range; after the wait they are kept if the final length gives
  // this warp the same first pages, else drained and reissued.
  int hp0 = 0, hcount = 0;
  {
    // L2-only loads here and after the wait: the first read must not leave an
    // L1 line that the second one could hit
    const int hint = __ldcg(A.lengths + b);
    if (hint > 0 && (int64_t)hint <= (int64_t)A.max_pages * P) page_range(hint, hp0, hcount);
  }
  int early = min(S, hcount);
  {
    bool hb = false;
    if (lane < early) {
      const int pid = A.page_table[(size_t)b * A.max_pages + hp0 + warp + kDecWarps * lane];
      hb = pid < 0 || (int64_t)pid >= A.n_pool_pages;
    }
    if (__any_sync(0xffffffffu, hb)) early = 0;
  }
  if (lane == 0)
    for (int i = 0; i < early; ++i) issue_page(hp0 + warp + kDecWarps * i, i);

  // group tables (built on the host with the page layout)
  {
    static_assert(sizeof(DecodeTables) % 16 == 0, "DecodeTables must copy as int4");
    const int4* src = reinterpret_cast<const int4*>(&hd->dec);
    int4* dst = reinterpret_cast<int4*>(&T);
    for (int e = tid; e < (int)(sizeof(DecodeTables) / 16); e += blockDim.x) dst[e] = src[e];
  }
  for (int j = 0; j < kMaxG; ++j) vacc_s[j * 32 + lane] = make_float4(0.f, 0.f, 0.f, 0.f);

  // ---- 2. wait; then the length, this warp's page ids, its first copies -----
  // (the wait covers the fold grid, which waits before it exits, and so every
  // earlier kernel of the stream)
  pdl_wait();
  int len = __ldcg(A.lengths + b);
  if (len < 0 || (int64_t)len > (int64_t)A.max_pages * P) {  // lengths written outside the library
    if (tid == 0) device_error(cd->err, SPECTRA_ERR_INVALID);
    len = 0;
  }
  int p0, count;
  page_range(len, p0, count);
  bool bad = false;
  for (int i = lane; i < count; i += 32) {
    const int pid = A.page_table[(size_t)b * A.max_pages + p0 + warp + kDecWarps * i];
    bad |= (pid < 0 || (int64_t)pid >= A.n_pool_pages);
  }
  const bool warp_bad = __any_sync(0xffffffffu, bad);
  if (warp_bad && lane == 0) device_error(cd->err, SPECTRA_ERR_INVALID);
  int my_count = warp_bad ? 0 : count;
  // speculative copies: kept when they are this warp's first pages under the
  // final length; else each is waited for (bounded) and its stage's first phase
  // counted as used (off_mask), and the copies are reissued
  uint32_t off_mask = 0u;
  int issued = 0;
  if (early > 0) {
    if (p0 == hp0 && early <= my_count) {
      issued = early;
    } else {
      bool drained = true;
      if (lane == 0)
        for (int i = 0; i < early; ++i) drained &= mbar_wait_bounded(&bars[i], 0u, kWaitLimitNs);
      drained = __shfl_sync(0xffffffffu, drained, 0);
      if (!drained) {
        if (lane == 0) device_error(cd->err, SPECTRA_ERR_TIMEOUT);
        my_count = 0;
      }
      off_mask = (1u << early) - 1u;
    }
  }
  // parity of copy i's completion on its stage's barrier
  auto parity = [&](int i) -> uint32_t { return (uint32_t)(((i / S) + ((off_mask >> (i % S)) & 1u)) & 1u); };
  auto issue = [&](int i) { issue_page(p0 + warp + kDecWarps * i, i); };
  if (lane == 0)
    for (int i = issued; i < min(S, my_count); ++i) issue(i);

  // ---- 3. the folded query (written by the fold grid) -----------------------
  {
    // rows j*NT + nt (j < kMaxG) and the bz rows kMaxG*2 + nt
    const uint2* src = A.frag + ((size_t)b * A.n_kv + a) * kFragWords;
    for (int e = tid; e < kMaxG * NT * 32; e += blockDim.x) bq_s[e] = src[e];
    for (int e = tid; e < NT * 32; e += blockDim.x) bq_s[kMaxG * 2 * 32 + e] = src[kMaxG * 2 * 32 + e];
  }
  __syncthreads();
  uint32_t bz[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const uint2 v = bq_s[(kMaxG * 2 + nt) * 32 + lane];
    bz[nt][0] = v.x;
    bz[nt][1] = v.y;
  }
  LaneAddr L;
  L.off4 = lane * 4;
  L.off8 = lane * 8;
  L.off2 = (2 * gid + (t4 >> 1)) * 4;
  L.off1 = gid * 4;
  L.sh2 = 2u * (uint32_t)(t4 & 1);
  L.sh1 = (uint32_t)t4;
  L.rot1 = (uint32_t)(t4 - 2) & 31u;
  // record offsets (within a group's records) of this lane for chunk 0: K rows
  // use token pair gid; V uses pairs t4 and t4 + 4; the K z term uses groups
  // 2*t4 and 2*t4+1 at pair gid; the V z term group gid at pairs t4, t4+4
  const int recK = gid * tpp * 8, recVa = t4 * tpp * 8, recVb = (t4 + 4) * tpp * 8;
  const int zkA = T.rec[0][min(2 * t4, kMaxG - 1)], zkB = T.rec[0][min(2 * t4 + 1, kMaxG - 1)];
  const bool hasA = 2 * t4 < nK, hasB = 2 * t4 + 1 < nK;
  const int zv = T.rec[1][gid];
  const bool hasV = gid < nV;

  float m_run[NT], l_run[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt] = -CUDART_INF_F;
    l_run[nt] = 0.f;
  }
  float dz[4] = {0.f, 0.f, 0.f, 0.f};

  // ---- 3. stream this warp's pages, CH tiles (16 tokens each) at a time ------
  bool timed_out = false;
  int i = 0;
  for (; i < my_count; ++i) {
    const int s = i % S;
    const bool ok = mbar_wait_bounded(&bars[s], parity(i), kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ok)) {
      timed_out = true;
      break;
    }
    const uint8_t* sec = my_stages + (size_t)s * A.stage_bytes;
    const int pg = p0 + warp + kDecWarps * i;
    const int n_valid = min(P, len - pg * P);
#pragma unroll 1
    for (int c0 = 0; c0 < tpp; c0 += CH) {
      const int tok0 = c0 * 16;
      const bool partial = n_valid < tok0 + CH * 16;  // warp-uniform
      const int unit = c0 * 32 / (G == 16 ? 1 : 2);   // chunk's block bytes per code bit
      // keys
      float acc[CH][NT][4];
#pragma unroll
      for (int tt = 0; tt < CH; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[tt][nt][r] = 0.f;
      const int rk = recK + c0 * 8;
      key_class<G, NT, CH, 4>(T, sec, unit, rk, L, bq_s, lane, 0, acc);
      key_class<G, NT, CH, 2>(T, sec, unit, rk, L, bq_s, lane, 1, acc);
      key_class<G, NT, CH, 1>(T, sec, unit, rk, L, bq_s, lane, 2, acc);
      key_class<G, NT, CH, 3>(T, sec, unit, rk, L, bq_s, lane, 3, acc);
      key_class<G, NT, CH, 8>(T, sec, unit, rk, L, bq_s, lane, 4, acc);
      // z term of the keys (k = group index) and the scores (log2 units)
      uint32_t zA[CH], zB[CH];
#pragma unroll
      for (int h = 0; h < CH / 2; ++h) {
        const uint4 ra = hasA ? *reinterpret_cast<const uint4*>(sec + zkA + rk + 16 * h) : make_uint4(0, 0, 0, 0);
        const uint4 rb = hasB ? *reinterpret_cast<const uint4*>(sec + zkB + rk + 16 * h) : make_uint4(0, 0, 0, 0);
        zA[2 * h] = ra.y;
        zA[2 * h + 1] = ra.w;
        zB[2 * h] = rb.y;
        zB[2 * h + 1] = rb.w;
      }
      float sc[CH][NT][2];
#pragma unroll
      for (int tt = 0; tt < CH; ++tt) {
        const uint32_t az[4] = {__byte_perm(zA[tt], zB[tt], 0x5410), __byte_perm(zA[tt], zB[tt], 0x7632), 0u, 0u};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float d[4];
          mma_m16n8k16_z(d, az, bz[nt]);
          sc[tt][nt][0] = fmaf(acc[tt][nt][0] + acc[tt][nt][1], kTwo24, d[0] + d[1]);
          sc[tt][nt][1] = fmaf(acc[tt][nt][2] + acc[tt][nt][3], kTwo20, d[2] + d[3]);
        }
      }
      if (partial) {
#pragma unroll
        for (int tt = 0; tt < CH; ++tt) {
          const int nv = n_valid - tok0 - tt * 16;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (2 * gid >= nv) sc[tt][nt][0] = -CUDART_INF_F;
            if (2 * gid + 1 >= nv) sc[tt][nt][1] = -CUDART_INF_F;
          }
        }
      }
      // online softmax (log2 units); rescale only when a running max grows
      bool grow = false;
      float alpha[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int tt = 0; tt < CH; ++tt) mx = fmaxf(mx, fmaxf(sc[tt][nt][0], sc[tt][nt][1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        alpha[nt] = 1.f;
        if (mx > m_run[nt]) {
          alpha[nt] = ex2_approx(m_run[nt] - mx);
          m_run[nt] = mx;
          l_run[nt] *= alpha[nt];
          grow = true;
        }
      }
      const bool grew = __any_sync(0xffffffffu, grow);
      float ae = 1.f, ao = 1.f;
      if (grew) {
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
      uint32_t pb[CH][2];
      uint32_t msk[CH][2];
      float off[NT];  // p = 2^(s - m + 8)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) off[nt] = kPScaleLog2 - m_run[nt];
      const int src0 = (t4 << 2) | (gid & 3), src1 = ((t4 + 4) << 2) | (gid & 3);
#pragma unroll
      for (int tt = 0; tt < CH; ++tt) {
        uint32_t p01[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float pa = ex2_approx(sc[tt][nt][0] + off[nt]);
          const float pv = ex2_approx(sc[tt][nt][1] + off[nt]);
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
        msk[tt][0] = msk[tt][1] = 0xffffffffu;
        if (partial) {
          // tokens past the end: their records may hold anything; zero their s and z
          const int nv = n_valid - tok0 - tt * 16;
          msk[tt][0] = ((2 * t4 < nv) ? 0x0000ffffu : 0u) | ((2 * t4 + 1 < nv) ? 0xffff0000u : 0u);
          msk[tt][1] = ((2 * t4 + 8 < nv) ? 0x0000ffffu : 0u) | ((2 * t4 + 9 < nv) ? 0xffff0000u : 0u);
        }
      }
      // values: per group, sum_t (p_t s_t,j) code_t,j ...
      const int ra = recVa + c0 * 8, rb = recVb + c0 * 8;
      if (!partial) {
        value_class<G, CH, 4, false>(T, sec, unit, ra, rb, L, vacc_s, lane, 0, grew, ae, ao, pb, msk);
        value_class<G, CH, 2, false>(T, sec, unit, ra, rb, L, vacc_s, lane, 1, grew, ae, ao, pb, msk);
        value_class<G, CH, 1, false>(T, sec, unit, ra, rb, L, vacc_s, lane, 2, grew, ae, ao, pb, msk);
        value_class<G, CH, 3, false>(T, sec, unit, ra, rb, L, vacc_s, lane, 3, grew, ae, ao, pb, msk);
        value_class<G, CH, 8, false>(T, sec, unit, ra, rb, L, vacc_s, lane, 4, grew, ae, ao, pb, msk);
      } else {
        value_class<G, CH, 4, true>(T, sec, unit, ra, rb, L, vacc_s, lane, 0, grew, ae, ao, pb, msk);
        value_class<G, CH, 2, true>(T, sec, unit, ra, rb, L, vacc_s, lane, 1, grew, ae, ao, pb, msk);
        value_class<G, CH, 1, true>(T, sec, unit, ra, rb, L, vacc_s, lane, 2, grew, ae, ao, pb, msk);
        value_class<G, CH, 3, true>(T, sec, unit, ra, rb, L, vacc_s, lane, 3, grew, ae, ao, pb, msk);
        value_class<G, CH, 8, true>(T, sec, unit, ra, rb, L, vacc_s, lane, 4, grew, ae, ao, pb, msk);
      }
      // ... plus sum_t p_t z_t,j for all groups (rows = groups).  Lanes of
      // absent groups load nothing, but every lane executes the MMA.
      {
        uint32_t za[CH], zb[CH];
#pragma unroll
        for (int h = 0; h < CH / 2; ++h) {
          const uint4 x = hasV ? *reinterpret_cast<const uint4*>(sec + zv + ra + 16 * h) : make_uint4(0, 0, 0, 0);
          const uint4 y = hasV ? *reinterpret_cast<const uint4*>(sec + zv + rb + 16 * h) : make_uint4(0, 0, 0, 0);
          za[2 * h] = x.y;
          za[2 * h + 1] = x.w;
          zb[2 * h] = y.y;
          zb[2 * h + 1] = y.w;
        }
#pragma unroll
        for (int tt = 0; tt < CH; ++tt) {
          const uint32_t az[4] = {partial ? (za[tt] & msk[tt][0]) : za[tt], 0u,
                                  partial ? (zb[tt] & msk[tt][1]) : zb[tt], 0u};
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
        mbar_wait_bounded(&bars[k % S], parity(k), kWaitLimitNs);
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
  // latent accumulator of (head h, coordinate j*G + k) = 2^24 * f * vacc + the
  // z term of group j; f = 1/16 for rows k >= 8 of a G = 16 group of width <= 4
  __syncthreads();
  const int nkv = sv->n_kept;
  constexpr int rec = 2 + kMaxKept;
  float* wsm = reinterpret_cast<float*>(region);              // [warp][gq][rec]
  float* wts = wsm + kDecWarps * kMaxGQ * rec;                // [gq][kDecWarps + 2]
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
  const int h0 = 2 * t4, h1 = 2 * t4 + 1;
  for (int j = 0; j < nV; ++j) {
    const float4 v4 = vacc_s[j * 32 + lane];
    const float z0 = __shfl_sync(0xffffffffu, dz[0], j * 4 + t4);
    const float z1 = __shfl_sync(0xffffffffu, dz[1], j * 4 + t4);
    const float f_hi = (G == 16 && T.wid[1][j] <= 4) ? kTwo20 : kTwo24;
    float* r0 = wsm + (warp * gq + h0) * rec + 2 + j * G + gid;
    float* r1 = wsm + (warp * gq + h1) * rec + 2 + j * G + gid;
    if (h0 < gq) {
      r0[0] = fmaf(v4.x, kTwo24, z0);
      if (G == 16) r0[8] = fmaf(v4.z, f_hi, z0);
    }
    if (h1 < gq) {
      r1[0] = fmaf(v4.y, kTwo24, z1);
      if (G == 16) r1[8] = fmaf(v4.w, f_hi, z1);
    }
  }
  __syncthreads();
  if (tid < gq) {
    float M = -CUDART_INF_F;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wsm[(w * gq + tid) * rec]);
    float Lsum = 0.f;
    for (int w = 0; w < kDecWarps; ++w) {
      const float mw = wsm[(w * gq + tid) * rec];
      const float wt = (mw == -CUDART_INF_F) ? 0.f : ex2_approx(mw - M);
      wts[tid * (kDecWarps + 2) + w] = wt;
      Lsum = fmaf(wt, wsm[(w * gq + tid) * rec + 1], Lsum);
    }
    wts[tid * (kDecWarps + 2) + kDecWarps] = M;
    wts[tid * (kDecWarps + 2) + kDecWarps + 1] = Lsum;
  }
  __syncthreads();
  float* part = A.part + ((size_t)(b * A.n_q + a * gq) * A.n_split + split) * A.part_stride;
  for (int hl = 0; hl < gq; ++hl) {
    const float* wt = wts + hl * (kDecWarps + 2);
    float* dst = part + (size_t)hl * A.n_split * A.part_stride;
    for (int c = tid; c < 2 + nkv; c += blockDim.x) {
      float v;
      if (c < 2) {
        v = wt[kDecWarps + c];
      } else {
        v = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) v = fmaf(wt[w], wsm[(w * gq + hl) * rec + c], v);
      }
      dst[c] = v;
    }
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
  float* half_s = wgt + kMaxSplit;                       // [2][kMaxDHead]
  float* w_s = half_s + 2 * kMaxDHead;                   // [max_kept_v][d_h]
  float* p_s = w_s + A.max_kept_v * d_h;                 // [ns][stride]
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
  {
    const float* src = A.part + ((size_t)b * A.n_q + h) * ns * stride;  // stride % 4 == 0
    for (int e = tid; e < ns * stride / 4; e += blockDim.x) cp_async16(p_s + 4 * e, src + 4 * e);
    cp_async_wait_all();
  }
  __syncthreads();
  const float* pr = p_s;
  const int warp = tid >> 5, lane = tid & 31;
  float mloc = -CUDART_INF_F;
  for (int s = tid; s < ns; s += blockDim.x) mloc = fmaxf(mloc, pr[(size_t)s * stride]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
  if (lane == 0) red[warp] = mloc;
  __syncthreads();
  float M = -CUDART_INF_F;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) M = fmaxf(M, red[w]);
  __syncthreads();
  float lloc = 0.f;
  for (int s = tid; s < ns; s += blockDim.x) {
    const float ms = pr[(size_t)s * stride];
    const float w = (M == -CUDART_INF_F || ms == -CUDART_INF_F) ? 0.f : exp2f(ms - M);
    wgt[s] = w;
    lloc += w * pr[(size_t)s * stride + 1];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lloc += __shfl_xor_sync(0xffffffffu, lloc, o);
  if (lane == 0) red[warp] = lloc;
  __syncthreads();
  float L = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) L += red[w];
  const float invL = L > 0.f ? 1.f / L : 0.f;
  // latent output: each coordinate's sum over the splits in two halves
  const int hs = (ns + 1) / 2;
  for (int idx = tid; idx < 2 * nkv; idx += blockDim.x) {
    const int c = idx % nkv, hf = idx / nkv;
    float acc = 0.f;
    for (int s = hf * hs; s < min(ns, hf * hs + hs); ++s) acc = fmaf(wgt[s], pr[(size_t)s * stride + 2 + c], acc);
    half_s[hf * kMaxDHead + c] = acc;
  }
  __syncthreads();
  for (int c = tid; c < nkv; c += blockDim.x) olat[c] = (half_s[c] + half_s[kMaxDHead + c]) * invL;
  __syncthreads();
  bool ok = true;
  if (wbytes) ok = mbar_wait_bounded(bar, 0, kWaitLimitNs);
  if (!ok && tid == 0) device_error(cd->err, SPECTRA_ERR_TIMEOUT);
  // out = olat W_up^V, each output's sum over the coordinates in two halves
  const int hc = (nkv + 1) / 2;
  for (int idx = tid; idx < 2 * d_h; idx += blockDim.x) {
    const int d = idx % d_h, hf = idx / d_h;
    float acc = 0.f;
    for (int c = hf * hc; c < min(nkv, hf * hc + hc); ++c) acc = fmaf(olat[c], w_s[c * d_h + d], acc);
    half_s[hf * kMaxDHead + d] = acc;
  }
  __syncthreads();
  float* orow = A.out + ((size_t)b * A.n_q + h) * d_h;
  for (int d = tid; d < d_h; d += blockDim.x) orow[d] = ok ? half_s[d] + half_s[kMaxDHead + d] : 0.f;
}

// Shared memory of the combine kernel: barrier, reductions, W_up^V of the
// largest V side (n_kept x d_head floats) and the partial records.
int combine_smem_bytes(int max_kept_v, int d_h, int ns, int stride) {
  return 64 + (32 + kMaxKept + kMaxSplit + 2 * kMaxDHead) * 4 + max_kept_v * d_h * 4 + ns * stride * 4;
}

template <int G, int NT, int CH>
int split_occupancy(int smem) {
  int n = 0;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(split_kernel<G, NT, CH>), smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, split_kernel<G, NT, CH>, kDecWarps * 32, smem) !=
          cudaSuccess ||
      n <= 0)
    n = 1;
  return n;
}

// Tiles (16 tokens) per softmax chunk: 4 when a page holds a multiple of 64
// tokens, else 2 (pages hold a multiple of 32).
int chunk_tiles(int P) { return (P / 16) % 4 == 0 ? 4 : 2; }

int split_ctas_per_sm(int group, bool two_tiles, int P, int smem) {
  const bool c4 = chunk_tiles(P) == 4;
  if (group == 16) {
    if (two_tiles) return c4 ? split_occupancy<16, 2, 4>(smem) : split_occupancy<16, 2, 2>(smem);
    return c4 ? split_occupancy<16, 1, 4>(smem) : split_occupancy<16, 1, 2>(smem);
  }
  if (two_tiles) return c4 ? split_occupancy<8, 2, 4>(smem) : split_occupancy<8, 2, 2>(smem);
  return c4 ? split_occupancy<8, 1, 4>(smem) : split_occupancy<8, 1, 2>(smem);
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

template <int G, int NT, int CH>
cudaError_t launch_all(const DecodeArgs& args, const DecodePlan& plan, int batch, int n_kv, int n_q, cudaStream_t st) {
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(split_kernel<G, NT, CH>), plan.smem_bytes);
  if (e != cudaSuccess) return e;
  const int csm = combine_smem_bytes(args.max_kept_v, args.d_h, args.n_split, args.part_stride);
  e = ensure_dynamic_smem(reinterpret_cast<const void*>(combine_kernel), csm);
  if (e != cudaSuccess) return e;
  e = launch_dependent(fold_kernel<G, NT>, dim3(n_kv, batch, kMaxG * G / 32), dim3(kFoldThreads), 0, st, args);
  if (e != cudaSuccess) return e;
  e = launch_dependent(split_kernel<G, NT, CH>, dim3(args.n_split, n_kv, batch), dim3(kDecWarps * 32),
                       plan.smem_bytes, st, args);
  if (e != cudaSuccess) return e;
  return launch_dependent(combine_kernel, dim3(n_q, batch), dim3(256), csm, st, args);
}

template <int G, int NT>
cudaError_t launch_chunked(const DecodeArgs& args, const DecodePlan& plan, int P, int batch, int n_kv, int n_q,
                           cudaStream_t st) {
  return chunk_tiles(P) == 4 ? launch_all<G, NT, 4>(args, plan, batch, n_kv, n_q, st)
                             : launch_all<G, NT, 2>(args, plan, batch, n_kv, n_q, st);
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
  // up to 40 KB of stages per CTA: one stage per warp for 8 KB sections (four
  // CTAs fit an SM), deeper per-warp pipelines when sections are small (measured
  // best for 8, 4 and 2.5 KB sections: 1, 2 and 4 stages)
  const int budget = 40 * 1024;
  p.stages = std::max(1, std::min(4, budget / (kDecWarps * p.stage_bytes)));
  p.smem_bytes = kSmStages + std::max(kDecWarps * p.stages * p.stage_bytes, kMergeBytes);
  // context splits: fill one wave of resident CTAs when that wastes < 15% of the
  // slots, else two waves; the count does not depend on the context length, so a
  // workspace sized once fits every call (the call clamps it to the cache's pages)
  const int units = std::max(1, batch * h.n_kv);
  const int slots = split_ctas_per_sm(h.group, h.gq > 4, h.P, p.smem_bytes) * sm_count();
  int ns = std::max(1, slots / units);
  if ((double)units * ns / slots < 0.85) {
    const int ns2 = std::max(1, 2 * slots / units);
    if ((double)units * ns2 / (2.0 * slots) > (double)units * ns / slots) ns = ns2;
  }
  p.part_stride = ((2 + h.max_kept_v) + 3) / 4 * 4;
  const int ns_fit = (kMaxSmemPerBlock - combine_smem_bytes(h.max_kept_v, h.d_h, 0, 0)) / (p.part_stride * 4);
  ns = std::max(1, std::min({ns, kMaxSplit, ns_fit}));
  // at least two pages per warp for a full-length sequence: fewer, longer
  // splits amortise each CTA's fixed work
  ns = std::max(1, std::min(ns, max_pages_per_seq / (kDecWarps * 2)));
  p.n_split = ns;
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
  args.max_kept_v = h.max_kept_v;
  args.d_h = h.d_h;
  args.q_scale = 1.4426950408889634f / sqrtf((float)h.d_h);
  const bool two = h.gq > 4;
  if (h.group == 16)
    return two ? launch_chunked<16, 2>(args, plan, h.P, cache.batch, h.n_kv, h.n_q, st)
               : launch_chunked<16, 1>(args, plan, h.P, cache.batch, h.n_kv, h.n_q, st);
  return two ? launch_chunked<8, 2>(args, plan, h.P, cache.batch, h.n_kv, h.n_q, st)
             : launch_chunked<8, 1>(args, plan, h.P, cache.batch, h.n_kv, h.n_q, st);
}

}  // namespace spectra
