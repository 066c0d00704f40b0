// The decode attention kernel of libspectra (template); see decode_kernels.cu
// for what it computes and how the host plans and launches it.  Included by the
// instantiation units attend_inst_g8.cu and attend_inst_g16.cu.
#pragma once

#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <type_traits>
#include <utility>

#include "attend_args.h"
#include "device_common.cuh"
#include "kernels.h"

namespace spectra {
namespace attend {

namespace cg = cooperative_groups;

// ---- small helpers ------------------------------------------------------------
template <int I>
struct Int {
  static constexpr int value = I;
};
template <int I, int N, typename F>
__device__ __forceinline__ void static_for_impl(F&& f) {
  if constexpr (I < N) {
    f(Int<I>{});
    static_for_impl<I + 1, N>(f);
  }
}
template <int N, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  static_for_impl<0, N>(f);
}

template <int OFF>
__device__ __forceinline__ uint32_t ld_s32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(OFF));
  return v;
}
template <int OFF>
__device__ __forceinline__ uint2 ld_s64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(OFF));
  return v;
}
template <int OFF>
__device__ __forceinline__ uint4 ld_s128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4+%5];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a), "n"(OFF));
  return v;
}
__device__ __forceinline__ int ld_volatile_s(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

// mma with a zero accumulator input (no register moves for C)
__device__ __forceinline__ void mma_m16n8k16_z(float d[4], const uint32_t a[4], const uint32_t b[2]) {
  const float z = 0.f;
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "f"(z));
}

__device__ __forceinline__ void mma_m16n8k8_z(float d[4], const uint32_t a[2], uint32_t b) {
  const float z = 0.f;
  asm(
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


// Split x into fp16 hi (part 0) or the fp16 of the remainder (part 1).
__device__ __forceinline__ float split_half(float x, int part) {
  const float hi = __half2float(__float2half_rn(x));
  return part ? (x - hi) : hi;
}

// ---------------------------------------------------------------------------
// Code words -> MMA A fragments.  A block's bytes hold, for every MMA lane, its
// 8 codes (slots 0..7, see the page layout): B = 4: word `lane` as nibbles;
// B = 2: word 2*gid + t4/2, bits 2*(t4%2) + {0,1} of each nibble; B = 1: word
// gid, bit t4 of each nibble; B = 3: a B = 2 part (16 words, code bits 0-1)
// then a B = 1 part (8 words, code bit 2); B = 8: words 2*lane, 2*lane+1 hold
// bytes [s0 s1 s4 s5] [s2 s3 s6 s7].  A nibble-held code is used in place: as an
// fp16 bit pattern, bits 0-3 of a 16-bit lane are the subnormal code * 2^-24 and
// bits 4-7 are code * 16 * 2^-24, so registers a1, a3 (MMA rows gid+8) carry a
// factor 16 for B <= 4.
// ---------------------------------------------------------------------------
template <int B>
__device__ __forceinline__ constexpr uint32_t frag_mask() {
  return B >= 4 ? 0x000F000Fu : (B == 3 ? 0x00070007u : (B == 2 ? 0x00030003u : 0x00010001u));
}

// The lane's nibble word of block `OFF` (bytes from the lane's address p; p1 is
// the lane's address in the 1-bit part for B = 3).
template <int B, int OFF>
__device__ __forceinline__ uint32_t nibble_word(uint32_t p, uint32_t p1, uint32_t sh, uint32_t rot1) {
  if constexpr (B == 4) {
    return ld_s32<OFF>(p);
  } else if constexpr (B == 2 || B == 1) {
    return ld_s32<OFF>(p) >> sh;
  } else {
    // code bits 0-1 from the 2-bit part, bit 2 from the 1-bit part (rotated from
    // nibble bit t4 to nibble bit 2); bit 3 of each nibble is junk, cleared by
    // the fragment masks
    const uint32_t lo = ld_s32<OFF>(p) >> sh;
    const uint32_t w1 = ld_s32<OFF>(p1);
    const uint32_t hi = __funnelshift_r(w1, w1, rot1);
    return (lo & 0x33333333u) | (hi & 0xCCCCCCCCu);
  }
}

// K side, A = codes (rows: tokens, cols: coordinates).  G = 16: m16n8k16, four
// registers; G = 8: m16n8k8, two registers for half `MI` of a 32-token block.
template <int G, int B, int OFF, int MI>
__device__ __forceinline__ void frag_k(uint32_t p, uint32_t p1, uint32_t sh, uint32_t rot1, uint32_t (&av)[4]) {
  if constexpr (B == 8) {
    const uint2 w = ld_s64<OFF>(p);
    if constexpr (G == 16) {
      av[0] = w.x & 0x00FF00FFu;
      av[1] = (w.x >> 8) & 0x00FF00FFu;
      av[2] = w.y & 0x00FF00FFu;
      av[3] = (w.y >> 8) & 0x00FF00FFu;
    } else {
      const uint32_t x = MI ? w.y : w.x;
      av[0] = x & 0x00FF00FFu;
      av[1] = (x >> 8) & 0x00FF00FFu;
    }
  } else {
    constexpr uint32_t M = frag_mask<B>();
    const uint32_t x = nibble_word<B, OFF>(p, p1, sh, rot1);
    if constexpr (G == 16) {
      const uint32_t y = x >> 8;
      av[0] = x & M;
      av[1] = x & (M << 4);
      av[2] = y & M;
      av[3] = y & (M << 4);
    } else {
      const uint32_t y = MI ? (x >> 8) : x;
      av[0] = y & M;
      av[1] = y & (M << 4);
    }
  }
}

// V side, A = codes transposed (rows: coordinates, cols: tokens), m16n8k16.
// G = 8: rows 8..15 are zero; no factor 16 (shifts instead).
template <int G, int B, int OFF, int MI>
__device__ __forceinline__ void frag_v(uint32_t p, uint32_t p1, uint32_t sh, uint32_t rot1, uint32_t (&av)[4]) {
  if constexpr (B == 8) {
    const uint2 w = ld_s64<OFF>(p);
    if constexpr (G == 16) {
      av[0] = w.x & 0x00FF00FFu;
      av[1] = (w.x >> 8) & 0x00FF00FFu;
      av[2] = w.y & 0x00FF00FFu;
      av[3] = (w.y >> 8) & 0x00FF00FFu;
    } else {
      av[0] = (MI ? (w.x >> 8) : w.x) & 0x00FF00FFu;
      av[1] = 0u;
      av[2] = (MI ? (w.y >> 8) : w.y) & 0x00FF00FFu;
      av[3] = 0u;
    }
  } else {
    constexpr uint32_t M = frag_mask<B>();
    const uint32_t x = nibble_word<B, OFF>(p, p1, sh, rot1);
    if constexpr (G == 16) {
      const uint32_t y = x >> 8;
      av[0] = x & M;
      av[1] = x & (M << 4);
      av[2] = y & M;
      av[3] = y & (M << 4);
    } else {
      const uint32_t xs = MI ? (x >> 4) : x;
      av[0] = xs & M;
      av[1] = 0u;
      av[2] = (xs >> 8) & M;
      av[3] = 0u;
    }
  }
}

// Lane-constant addressing: byte offset of this lane's word in a block per
// width, shifts and the B = 3 rotation.
struct LaneAddr {
  uint32_t off4, off2, off1, off8;
  uint32_t sh2, sh1, rot1;
};

template <int B>
__device__ __forceinline__ uint32_t lane_off(const LaneAddr& L) {
  return B == 4 ? L.off4 : (B == 8 ? L.off8 : ((B == 2 || B == 3) ? L.off2 : L.off1));
}
template <int B>
__device__ __forceinline__ uint32_t lane_sh(const LaneAddr& L) {
  return B == 1 ? L.sh1 : L.sh2;
}

// Keys of one kept group for the CH tiles of a chunk: acc[tt][nt] +=
// s * (q_lat,j . code) for (token row gid, token row gid+8) x (hi, lo).  Rows
// gid+8 carry the factor 16 (B = 8 scales s instead).  blk: the group's first
// block of the chunk (shared address); rec: this lane's records of the chunk.
template <int G, int NT, int CH, int B>
__device__ __forceinline__ void key_group(uint32_t blk, uint32_t rec, const LaneAddr& L, const uint2 (&bqj)[NT],
                                          float (&acc)[CH][NT][4]) {
  const uint32_t p = blk + lane_off<B>(L);
  const uint32_t p1 = blk + 64 + L.off1;
  const uint32_t sh = lane_sh<B>(L);
  uint32_t sp[CH];
  static_for<CH / 2>([&](auto hi) {
    constexpr int h = decltype(hi)::value;
    const uint4 r = ld_s128<h * 16>(rec);  // {s, z} of 2 tiles
    sp[2 * h] = r.x;
    sp[2 * h + 1] = r.z;
  });
  static_for<CH>([&](auto tti) {
    constexpr int tt = decltype(tti)::value;
    constexpr int kBlockTiles = G == 16 ? 1 : 2;
    constexpr int OFF = (tt / kBlockTiles) * B * 32;
    uint32_t av[4];
    frag_k<G, B, OFF, tt & 1>(p, p1, sh, L.rot1, av);
    float sA, sB;
    half2_to_floats(sp[tt], sA, sB);
    if (B == 8) sB *= 16.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float d[4];
      const uint32_t bb[2] = {bqj[nt].x, bqj[nt].y};
      if constexpr (G == 16) mma_m16n8k16_z(d, av, bb);
      else mma_m16n8k8_z(d, av, bb[0]);
      acc[tt][nt][0] = fmaf(sA, d[0], acc[tt][nt][0]);
      acc[tt][nt][1] = fmaf(sA, d[1], acc[tt][nt][1]);
      acc[tt][nt][2] = fmaf(sB, d[2], acc[tt][nt][2]);
      acc[tt][nt][3] = fmaf(sB, d[3], acc[tt][nt][3]);
    }
  });
}

// Values of one kept group for the CH tiles of a chunk: va += code^T (p s).
// recA / recB: this lane's records of token pairs t4 and t4+4.  The chunk's
// tiles are summed by the tensor cores from zero and the chunk's sum is added to
// va in IEEE fp32: accumulating a whole context inside the MMA chain loses
// accuracy (the positive code term and the z term nearly cancel at the end).
template <int G, int CH, int B>
__device__ __forceinline__ void value_group(uint32_t blk, uint32_t recA, uint32_t recB, const LaneAddr& L,
                                            const uint32_t (&pb)[CH][2], float (&va)[4]) {
  const uint32_t p = blk + lane_off<B>(L);
  const uint32_t p1 = blk + 64 + L.off1;
  const uint32_t sh = lane_sh<B>(L);
  uint32_t s0[CH], s1[CH];
  float t[4];
  static_for<CH / 2>([&](auto hi) {
    constexpr int h = decltype(hi)::value;
    const uint4 ra = ld_s128<h * 16>(recA);
    const uint4 rb = ld_s128<h * 16>(recB);
    s0[2 * h] = ra.x;
    s0[2 * h + 1] = ra.z;
    s1[2 * h] = rb.x;
    s1[2 * h + 1] = rb.z;
  });
  static_for<CH>([&](auto tti) {
    constexpr int tt = decltype(tti)::value;
    constexpr int kBlockTiles = G == 16 ? 1 : 2;
    constexpr int OFF = (tt / kBlockTiles) * B * 32;
    uint32_t av[4];
    frag_v<G, B, OFF, tt & 1>(p, p1, sh, L.rot1, av);
    const uint32_t bj[2] = {hmul2_bits(pb[tt][0], s0[tt]), hmul2_bits(pb[tt][1], s1[tt])};
    if constexpr (tt == 0) mma_m16n8k16_z(t, av, bj);
    else mma_m16n8k16(t, av, bj);
  });
  va[0] += t[0];
  va[1] += t[1];
  va[2] += t[2];
  va[3] += t[3];
}


template <int G, int NT, int CH, int B>
__device__ __forceinline__ void key_class(const int4* ord, int c_begin, int c_end, uint32_t sec, uint32_t rk,
                                          int c0, const uint2* bq_s, int lane, const LaneAddr& L,
                                          float (&acc)[CH][NT][4]) {
  constexpr int kBT = G == 16 ? 1 : 2;
#pragma unroll 1
  for (int c = c_begin; c < c_end; ++c) {
    const int4 g = ord[c];
    uint2 bqj[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) bqj[nt] = bq_s[(g.z * NT + nt) * 32 + lane];
    key_group<G, NT, CH, B>(sec + (uint32_t)g.x + (uint32_t)((c0 / kBT) * B * 32), rk + (uint32_t)g.y, L, bqj,
                            acc);
  }
}

// ---------------------------------------------------------------------------
// attend_kernel: see the file comment.
// ---------------------------------------------------------------------------
template <int G, int NT, int CH, int MV>
__global__ void __launch_bounds__(kThreads, 2) attend_kernel(const AttendArgs A) {
  static_assert(MV == 2 || MV == 4 || MV == 8, "value-side group bound");
  extern __shared__ __align__(128) uint8_t smem[];
  const CodecDev* __restrict__ cd = A.cd;
  const int split = blockIdx.x, a = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, t4 = lane & 3;
  pdl_launch_dependents();

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
  int* issued = reinterpret_cast<int*>(smem + kOffIssued);
  int* consumed = reinterpret_cast<int*>(smem + kOffConsumed);
  int* flags = reinterpret_cast<int*>(smem + kOffFlags);
  int4* grp = reinterpret_cast<int4*>(smem + kOffGrp);
  uint2* bq_s = reinterpret_cast<uint2*>(smem + kOffBq);
  float* qlat_s = reinterpret_cast<float*>(smem + kOffQlat);  // [kMaxGQ][kMaxKept]
  float* x_s = reinterpret_cast<float*>(smem + kOffX);
  uint8_t* stages = smem + A.off_stages;
  const uint32_t stages_u32 = smem_u32(stages);

  const int P = A.P, gq = A.gq, d_h = A.d_h;
  const int tpp = P / 16;
  const int32_t* hm = A.hm[a];
  const HeadDev* hd = &cd->head[a];
  const int sec_off = hm[0], sec_bytes = hm[1];
  const int nK = hm[2], nV = hm[3];
  const int nkK = hm[4], nkV = hm[5];
  const int S = A.stages;
  const int ns = A.n_split;
  const int64_t cap = (int64_t)A.max_pages * P;
  const int32_t* ptab = A.page_table + (size_t)b * A.max_pages;
  const int k0 = 0, k1 = nkK;  // the fold covers every kept K coordinate

  // ---- 1. the independent global loads first, all in flight together -----------
  // (warp 0: the length hint and this CTA's first page ids; warp 1: the group
  // tables; the fold's rows of W_up^K; the caller's q)
  // CTA `split` owns pages split, split + n_split, ...; its warp w takes the
  // CTA's pages w, w + 8, ... in order, so the partition and the summation
  // order depend only on the final length.  The lengths only grow (appends)
  // while a kernel of this library may still be running before the dependency
  // wait, so the hint read here is at most the final length.  A running fused
  // encode may have advanced it by up to hint_lag tokens before its page
  // writes land, so pages full hint_lag tokens below the hint are final: their
  // copies go out before the wait.
  int hint_raw = 0, pid = -1;
  if (warp == 0) {
    hint_raw = __ldcg(A.lengths + b);
    const int pg = split + ns * lane;
    if (lane < S && pg < A.max_pages) pid = ptab[pg];
  }
  int4* ord = reinterpret_cast<int4*>(smem + kOffOrd);
  int* cls = reinterpret_cast<int*>(smem + kOffCls);
  static_assert(kOffCls == kOffOrd + 256 && sizeof(DecodeOrder) == 320, "class tables copy as 20 int4");
  if (warp == 1) {
    if (lane < 20) ord[lane] = reinterpret_cast<const int4*>(&hd->dec)[lane];
  }
  if (tid >= 64 && tid < 64 + 2 * kMaxG) {
    const int e = tid - 64, s = e / kMaxG, j = e % kMaxG;
    const SideDev* sd = &hd->side[s];
    int4 v = make_int4(0, 0, 0, 0);
    if (j < (s ? nV : nK)) {
      const GroupDev g = sd->grp[j];
      v = make_int4(g.plane_off - sec_off, g.sz_off - sec_off, g.b, g.col);
    }
    grp[e] = v;
  }
  // fold rows: 8 rows per warp and pass, lane (row, quarter of d_head)
  const int dq4 = d_h / 16;  // float4 chunks per quarter row
  constexpr int kWPre = 8;   // chunks held in registers from the start (d_head <= 128)
  float4 wpre[kWPre];
  {
    const int k = k0 + warp * 8 + (lane >> 2);
    const float4* wr = reinterpret_cast<const float4*>(A.cd->w_up + hm[6] + (size_t)k * d_h) + (lane & 3) * dq4;
#pragma unroll
    for (int u = 0; u < kWPre; ++u) wpre[u] = (k < k1 && u < dq4) ? __ldg(wr + u) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  {
    const float4* qs = reinterpret_cast<const float4*>(A.q + ((size_t)b * A.n_q + (size_t)a * gq) * d_h);
    float4* qd = reinterpret_cast<float4*>(x_s);
    for (int e = tid; e < gq * d_h / 4; e += kThreads) qd[e] = __ldg(qs + e);
  }

  // ---- 2. barriers and ring bookkeeping; copies of the full pages -------------------
  if (warp == 0) {
    if (lane < S) mbar_init(&bars[lane], 1);
    if (lane == 0) mbar_init(&bars[kMaxStages], 1);
    fence_mbar_init();
    issued[lane] = 0;  // kMaxStages == 32
    consumed[lane] = 0;
    flags[lane] = 0;
  }
  static_assert(kMaxStages == 32, "one lane of warp 0 per stage");
  __syncwarp();

  auto issue_copy = [&](int i, int pg_pid) {
    // copy the head section of page id pg_pid into stage i % S (one thread)
    if (i == A.drop_page && (split | a | b) == 0) return;  // test hook: a copy that never lands
    const int s = i % S;
    const uint8_t* src = A.pool + (size_t)pg_pid * (size_t)A.page_bytes + sec_off;
    mbar_arrive_expect_tx(&bars[s], (uint32_t)sec_bytes);
    bulk_copy_g2s(stages + (size_t)s * A.stage_bytes, src, (uint32_t)sec_bytes, &bars[s]);
  };
  if (warp == 0) {
    int64_t hint = (int64_t)hint_raw - A.hint_lag;
    hint = hint < 0 ? 0 : (hint > cap ? cap : hint);
    const int full_h = (int)(hint / P);
    const bool ok = lane < S && split + ns * lane < full_h && pid >= 0 && (int64_t)pid < A.n_pool_pages;
    const uint32_t m = __ballot_sync(0xffffffffu, ok);
    const int n_pre = (~m == 0u) ? 32 : (__ffs(~m) - 1);
    if (lane < n_pre) {
      issue_copy(lane, pid);
      issued[lane] = 1;
    }
    if (lane == 0) flags[kFlagPre] = n_pre;
  }
  __syncthreads();

  // ---- 4. fold this rank's slice of the K coordinates: q_lat = q W_up^K^T -------
  // lane (row, quarter) sums a quarter of the row's d_head products, two
  // shuffles finish the sum
  {
    const int qd = lane & 3;
    const float* wk = cd->w_up + hm[6];  // K side rows [n_kept][d_h]
    for (int rb = k0 + warp * 8; rb < k1; rb += kWarps * 8) {
      const int k = rb + (lane >> 2);
      float part[kMaxGQ];
#pragma unroll
      for (int h = 0; h < kMaxGQ; ++h) part[h] = 0.f;
      const float4* wr = reinterpret_cast<const float4*>(wk + (size_t)k * d_h) + qd * dq4;
      for (int c = 0; c < dq4; c += kWPre) {
        float4 w[kWPre];
#pragma unroll
        for (int u = 0; u < kWPre; ++u)
          w[u] = (rb == k0 + warp * 8 && c == 0) ? wpre[u]
                 : ((k < k1 && c + u < dq4) ? __ldg(wr + c + u) : make_float4(0.f, 0.f, 0.f, 0.f));
#pragma unroll
        for (int u = 0; u < kWPre; ++u) {
          if (c + u < dq4) {
#pragma unroll
            for (int h = 0; h < kMaxGQ; ++h) {
              if (h < gq) {
                const float4 qv = reinterpret_cast<const float4*>(x_s + h * d_h)[qd * dq4 + c + u];
                part[h] = fmaf(qv.x, w[u].x, fmaf(qv.y, w[u].y, fmaf(qv.z, w[u].z, fmaf(qv.w, w[u].w, part[h]))));
              }
            }
          }
        }
      }
#pragma unroll
      for (int h = 0; h < kMaxGQ; ++h) {
        if (h < gq) {
          float v = part[h];
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          if (qd == 0 && k < k1) qlat_s[h * kMaxKept + k] = v * A.q_scale;
        }
      }
    }
  }
  __syncthreads();

  // ---- 5. MMA B fragments of q_lat ----------------------------------------------
  // bq[j][nt][lane]: column n = lane/4 of n-tile nt is q head nt*4 + n/2, part
  // n&1 (0: fp16(q_lat), 1: fp16(q_lat - fp16(q_lat))); rows k = 2*(lane%4) +
  // {0,1} (+8).  bz[nt][lane] likewise over the group sums (rows = groups).
  // Warp j builds group j's fragments; warps 0..NT-1 the group sums.
  static_assert(kMaxG == kWarps, "one warp per kept group");
  {
    const int j = warp;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hl = nt * 4 + (gid >> 1), part = gid & 1;
      uint2 v = make_uint2(0u, 0u);
      if (hl < gq && j < nK) {
        const float* base = qlat_s + hl * kMaxKept + j * G + 2 * t4;
        v.x = pack_half2(split_half(base[0], part), split_half(base[1], part));
        if (G == 16) v.y = pack_half2(split_half(base[8], part), split_half(base[9], part));
      }
      bq_s[(j * NT + nt) * 32 + lane] = v;
    }
    if (warp < NT) {
      const int hl = warp * 4 + (gid >> 1), part = gid & 1;
      float s0 = 0.f, s1 = 0.f;
      if (hl < gq) {
        const float* base = qlat_s + hl * kMaxKept;
        if (2 * t4 < nK)
          for (int k = 0; k < G; ++k) s0 += base[2 * t4 * G + k];
        if (2 * t4 + 1 < nK)
          for (int k = 0; k < G; ++k) s1 += base[(2 * t4 + 1) * G + k];
      }
      bq_s[(kMaxG * 2 + warp) * 32 + lane] =
          make_uint2(hl < gq ? pack_half2(split_half(s0, part), split_half(s1, part)) : 0u, 0u);
    }
  }

  // ---- 6. wait for the predecessor; the final length; the remaining copies -------
  pdl_wait();
  int len = __ldcg(A.lengths + b);
  if (len < 0 || (int64_t)len > cap) {  // lengths written outside the library
    if (tid == 0 && split == 0) device_error(cd->err, SPECTRA_ERR_INVALID);
    len = 0;
  }
  const int np_f = (len + P - 1) / P;
  int n_total = np_f > split ? (np_f - split + ns - 1) / ns : 0;
  auto page_of = [&](int i) -> int { return split + ns * i; };
  const int n_pre = flags[kFlagPre];
  {
    bool bad = false;
    for (int i = n_pre + tid; i < n_total; i += kThreads) {
      const int pid = ptab[page_of(i)];
      bad |= pid < 0 || (int64_t)pid >= A.n_pool_pages;
    }
    if (__syncthreads_or(bad)) {
      if (tid == 0) device_error(cd->err, SPECTRA_ERR_INVALID);
      n_total = 0;  // this CTA's pages are skipped
    }
  }
  if (warp == 0) {
    const int i = n_pre + lane;
    if (i < min(S, n_total)) {
      issue_copy(i, ptab[page_of(i)]);
      issued[i] = 1;
    }
  }

  // lane constants
  LaneAddr L;
  L.off4 = lane * 4;
  L.off8 = lane * 8;
  L.off2 = (2 * gid + (t4 >> 1)) * 4;
  L.off1 = gid * 4;
  L.sh2 = 2u * (uint32_t)(t4 & 1);
  L.sh1 = (uint32_t)t4;
  L.rot1 = (uint32_t)(t4 - 2) & 31u;
  __syncthreads();  // fragments and group tables are complete
  uint32_t bz[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const uint2 v = bq_s[(kMaxG * 2 + nt) * 32 + lane];
    bz[nt][0] = v.x;
    bz[nt][1] = v.y;
  }
  // record offsets (within a group's records) of this lane: K rows use token pair
  // gid; V uses pairs t4 and t4 + 4; the K z term uses groups 2*t4 and 2*t4+1 at
  // pair gid; the V z term group gid at pairs t4, t4+4
  const int recK = gid * tpp * 8, recVa = t4 * tpp * 8, recVb = (t4 + 4) * tpp * 8;
  const bool hasA = 2 * t4 < nK, hasB = 2 * t4 + 1 < nK, hasV = gid < nV;
  const int zkA = hasA ? grp[2 * t4].y : 0, zkB = hasB ? grp[2 * t4 + 1].y : 0;
  const int zv = hasV ? grp[kMaxG + gid].y : 0;

  float m_run[NT], l_run[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt] = -CUDART_INF_F;
    l_run[nt] = 0.f;
  }
  float dz[4] = {0.f, 0.f, 0.f, 0.f};
  // value accumulators of the kept V groups in width-class order (slot c < MV
  // holds group ordV[c].z): lane (gid, t4) holds coordinates gid, gid+8 x heads 2t4, 2t4+1
  float va[MV][4];
#pragma unroll
  for (int c = 0; c < MV; ++c) va[c][0] = va[c][1] = va[c][2] = va[c][3] = 0.f;
  int clsK[6], clsV[6];
#pragma unroll
  for (int ci = 0; ci < 6; ++ci) {
    clsK[ci] = cls[ci];
    clsV[ci] = cls[8 + ci];
  }
  const int4* ordK = ord;
  const int4* ordV = ord + kMaxG;

  // ---- 7. main loop: warp w takes the CTA's pages w, w + 8, ... -----------------
  int s = warp % S, ph = warp / S;  // stage and phase of page i, advanced incrementally
  for (int i = warp; i < n_total; i += kWarps) {
    // the copy of page i goes out only after page i - S left stage s (maybe
    // consumed by another warp): wait for it to be issued, then for its bytes
    bool ok = true;
    if (ld_volatile_s(&issued[s]) <= ph) {
      const uint64_t t0 = global_timer_ns();
      while (ld_volatile_s(&issued[s]) <= ph) {
        if (global_timer_ns() - t0 > A.wait_ns) {
          ok = false;
          break;
        }
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[s], (uint32_t)(ph & 1), A.wait_ns));
    if (!ok) {
      if (lane == 0) {
        device_error(cd->err, SPECTRA_ERR_TIMEOUT);
        flags[kFlagStop] = 1;
      }
      break;
    }
    const uint32_t sec = stages_u32 + (uint32_t)(s * A.stage_bytes);
    const int pg = page_of(i);
    const int n_valid = min(P, len - pg * P);
    if (n_valid < P) {
      // tokens past the end (last page): their records may hold anything (NaN
      // included); zero their scales and zeros so that they add nothing to the
      // value sums (their scores are set to -inf below)
      const int u0 = n_valid >> 1, nz = (P >> 1) - u0;
      for (int e = lane; e < (nK + nV) * nz; e += 32) {
        const int gs = e / nz, u = u0 + (e - gs * nz);
        const int4 o = gs < nK ? ord[gs] : ord[kMaxG + gs - nK];
        const uint32_t ra = sec + (uint32_t)o.y + 8u * (uint32_t)((u & 7) * tpp + (u >> 3));
        if (u == u0 && (n_valid & 1)) {
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(ra + 2), "h"((unsigned short)0) : "memory");
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(ra + 6), "h"((unsigned short)0) : "memory");
        } else {
          asm volatile("st.shared.v2.u32 [%0], {%1, %1};" ::"r"(ra), "r"(0u) : "memory");
        }
      }
      __syncwarp();
    }
#pragma unroll 1
    for (int c0 = 0; c0 < tpp; c0 += CH) {
      const int tok0 = c0 * 16;
      const bool partial = n_valid < tok0 + CH * 16;  // warp-uniform
      // keys
      float acc[CH][NT][4];
#pragma unroll
      for (int tt = 0; tt < CH; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[tt][nt][r] = 0.f;
      const uint32_t rk = sec + (uint32_t)(recK + c0 * 8);
      key_class<G, NT, CH, 4>(ordK, clsK[0], clsK[1], sec, rk, c0, bq_s, lane, L, acc);
      key_class<G, NT, CH, 2>(ordK, clsK[1], clsK[2], sec, rk, c0, bq_s, lane, L, acc);
      key_class<G, NT, CH, 1>(ordK, clsK[2], clsK[3], sec, rk, c0, bq_s, lane, L, acc);
      key_class<G, NT, CH, 3>(ordK, clsK[3], clsK[4], sec, rk, c0, bq_s, lane, L, acc);
      key_class<G, NT, CH, 8>(ordK, clsK[4], clsK[5], sec, rk, c0, bq_s, lane, L, acc);
      // z term of the keys (k = group index) and the scores (log2 units)
      uint32_t zA[CH], zB[CH];
      static_for<CH / 2>([&](auto hi) {
        constexpr int h = decltype(hi)::value;
        const uint4 ra = hasA ? ld_s128<16 * h>(rk + (uint32_t)zkA) : make_uint4(0, 0, 0, 0);
        const uint4 rb = hasB ? ld_s128<16 * h>(rk + (uint32_t)zkB) : make_uint4(0, 0, 0, 0);
        zA[2 * h] = ra.y;
        zA[2 * h + 1] = ra.w;
        zB[2 * h] = rb.y;
        zB[2 * h + 1] = rb.w;
      });
      float sc[CH][NT][2];
#pragma unroll
      for (int tt = 0; tt < CH; ++tt) {
        const uint32_t az[2] = {__byte_perm(zA[tt], zB[tt], 0x5410), __byte_perm(zA[tt], zB[tt], 0x7632)};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float d[4];
          mma_m16n8k8_z(d, az, bz[nt][0]);
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
#pragma unroll
        for (int c = 0; c < MV; ++c) {
          if (c < nV) {
            va[c][0] *= ae;
            va[c][1] *= ao;
            va[c][2] *= ae;
            va[c][3] *= ao;
          }
        }
      }
      // p as the B operand (tokens x heads): lane (gid, t4) needs head gid,
      // tokens (2t4, 2t4+1) and (2t4+8, 2t4+9)
      uint32_t pb[CH][2];
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
        // (columns of heads >= gq hold copies of real heads' weights; their
        // accumulator columns are never read)
      }
      // values: per group, sum_t (p_t s_t,j) code_t,j ...
      const uint32_t ra = sec + (uint32_t)(recVa + c0 * 8), rb = sec + (uint32_t)(recVb + c0 * 8);
      static_for<MV>([&](auto ci) {
        constexpr int c = decltype(ci)::value;
        if (c < nV) {
          const int4 g = ordV[c];
          constexpr int kBT = G == 16 ? 1 : 2;
          const uint32_t gb = sec + (uint32_t)g.x + (uint32_t)(c0 / kBT) * 32u * (uint32_t)g.w;
          const uint32_t ga = ra + (uint32_t)g.y, gbr = rb + (uint32_t)g.y;
          switch (g.w) {
            case 4: value_group<G, CH, 4>(gb, ga, gbr, L, pb, va[c]); break;
            case 2: value_group<G, CH, 2>(gb, ga, gbr, L, pb, va[c]); break;
            case 1: value_group<G, CH, 1>(gb, ga, gbr, L, pb, va[c]); break;
            case 3: value_group<G, CH, 3>(gb, ga, gbr, L, pb, va[c]); break;
            default: value_group<G, CH, 8>(gb, ga, gbr, L, pb, va[c]); break;
          }
        }
      });
      // ... plus sum_t p_t z_t,j for all groups (rows = groups).  Lanes of
      // absent groups load nothing, but every lane executes the MMA.
      {
        uint32_t za[CH], zb[CH];
        static_for<CH / 2>([&](auto hi) {
          constexpr int h = decltype(hi)::value;
          const uint4 x = hasV ? ld_s128<16 * h>(ra + (uint32_t)zv) : make_uint4(0, 0, 0, 0);
          const uint4 y = hasV ? ld_s128<16 * h>(rb + (uint32_t)zv) : make_uint4(0, 0, 0, 0);
          za[2 * h] = x.y;
          za[2 * h + 1] = x.w;
          zb[2 * h] = y.y;
          zb[2 * h + 1] = y.w;
        });
        float tz[4];
#pragma unroll
        for (int tt = 0; tt < CH; ++tt) {
          const uint32_t az[4] = {za[tt], 0u, zb[tt], 0u};
          if (tt == 0) mma_m16n8k16_z(tz, az, pb[tt]);
          else mma_m16n8k16(tz, az, pb[tt]);
        }
        dz[0] += tz[0];
        dz[1] += tz[1];
        dz[2] += tz[2];
        dz[3] += tz[3];
      }
    }
    // stage s is free: count it, and send the copy of page i + S into it
    __syncwarp();
    if (lane == 0) {
      consumed[s] = ph + 1;
      if (i + S < n_total) {
        fence_proxy_async_smem();
        issue_copy(i + S, ptab[page_of(i + S)]);
        __threadfence_block();
        *reinterpret_cast<volatile int*>(&issued[s]) = ph + 2;
      }
    }
    for (s += kWarps; s >= S; s -= S) ++ph;
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

  // ---- 8. drain copies that no warp consumed (errors, a hint above the length) -----
  __syncthreads();
  if (tid < S && issued[tid] > consumed[tid]) {
    if (!mbar_wait_bounded(&bars[tid], (uint32_t)(consumed[tid] & 1), A.wait_ns))
      device_error(cd->err, SPECTRA_ERR_TIMEOUT);
  }
  __syncthreads();

  // ---- 9. merge the warps into this CTA's record (m, l, latent sums) ----------------
  // latent sum of (head h, coordinate j*G + k) = 2^24 * f * va + the z term of
  // group j; f = 1/16 for rows k >= 8 of a G = 16 group of width <= 4
  constexpr int kWs = kCpStride;
  float* wsm = reinterpret_cast<float*>(stages);            // [warp][gq][kWs]
  if (gid == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hl = nt * 4 + t4;
      if (hl < gq) {
        wsm[(warp * gq + hl) * kWs + 0] = m_run[nt];
        wsm[(warp * gq + hl) * kWs + 1] = l_run[nt];
      }
    }
  }
  {
    const int h0 = 2 * t4, h1 = 2 * t4 + 1;
#pragma unroll
    for (int c = 0; c < MV; ++c) {
      const int j = c < nV ? ordV[c].z : 0;
      const float z0 = __shfl_sync(0xffffffffu, dz[0], j * 4 + t4);
      const float z1 = __shfl_sync(0xffffffffu, dz[1], j * 4 + t4);
      if (c < nV) {
        const int w = ordV[c].w;
        const float f_hi = (G == 16 && w <= 4) ? kTwo20 : kTwo24;
        float* r0 = wsm + (warp * gq + h0) * kWs + 2 + j * G + gid;
        float* r1 = wsm + (warp * gq + h1) * kWs + 2 + j * G + gid;
        if (h0 < gq) {
          r0[0] = fmaf(va[c][0], kTwo24, z0);
          if (G == 16) r0[8] = fmaf(va[c][2], f_hi, z0);
        }
        if (h1 < gq) {
          r1[0] = fmaf(va[c][1], kTwo24, z1);
          if (G == 16) r1[8] = fmaf(va[c][3], f_hi, z1);
        }
      }
    }
  }
  __syncthreads();
  const size_t unit = (size_t)b * A.n_kv + a;
  float* recs = A.rec + unit * ns * gq * A.rec_stride;  // [split][gq][rec_stride]
  {
    // weights of the warps per head: wts[h][w]; the record's m and l
    float* wts = reinterpret_cast<float*>(smem + kOffW);  // [gq][kWarps + 2]
    float* rec = recs + (size_t)split * gq * A.rec_stride;
    if (tid < gq) {
      float M = -CUDART_INF_F;
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wsm[(w * gq + tid) * kWs]);
      float Ls = 0.f;
      for (int w = 0; w < kWarps; ++w) {
        const float mw = wsm[(w * gq + tid) * kWs];
        const float wt = (mw == -CUDART_INF_F) ? 0.f : ex2_approx(mw - M);
        wts[tid * (kWarps + 2) + w] = wt;
        Ls = fmaf(wt, wsm[(w * gq + tid) * kWs + 1], Ls);
      }
      rec[tid * A.rec_stride + 0] = M;
      rec[tid * A.rec_stride + 1] = Ls;
    }
    __syncthreads();
    for (int e = tid; e < gq * nkV; e += kThreads) {  // thread (head, coordinate)
      const int h = e / nkV, c = e - h * nkV;
      const float* wt = wts + h * (kWarps + 2);
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v = fmaf(wt[w], wsm[(w * gq + h) * kWs + 2 + c], v);
      rec[h * A.rec_stride + 4 + c] = v;
    }
  }
  // ---- 10. the last CTA of this (sequence, KV head) merges the records and lifts ------
  // The barrier orders the CTA's record writes before thread 0's fence, which
  // releases them (cumulatively) ahead of the arrival; the last CTA's thread 0
  // fences again after its arrival (acquire) and the barrier passes that on.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const int t = atomicAdd(A.cnt + unit, 1);
    const int last = t == ns - 1;
    if (last) __threadfence();
    flags[kFlagLast] = last;
  }
  __syncthreads();
  if (!flags[kFlagLast]) return;
  const uint32_t wv_bytes = (uint32_t)nkV * d_h * 4;
  const bool wv_staged = A.wv_staged != 0;
  float* wv_s = reinterpret_cast<float*>(stages);
  float* wts = reinterpret_cast<float*>(smem + kOffQlat);   // [gq][kMaxSplit] weights (q_lat is dead)
  float* part = reinterpret_cast<float*>(smem + kOffX);     // [ch][gq][4 n4] partial merges
  float* lsum = reinterpret_cast<float*>(smem + kOffW);     // [gq] sum of weights x l
  const size_t hs = (size_t)gq * A.rec_stride;              // floats between splits' records
  // thread (chunk k, head h, 4 consecutive coordinates c4) sums splits k, k + ch,
  // ... of the records; the chunks are added in order afterwards (a fixed order)
  const int n4 = (nkV + 3) / 4;
  const int pairs = gq * n4;
  int ch = pairs > 0 ? kThreads / pairs : 1;
  ch = ch < ns ? ch : ns;
  const int ch_cap = pairs > 0 ? (kXBytes / 16) / pairs : 1;
  ch = ch < ch_cap ? ch : ch_cap;
  ch = ch > 1 ? ch : 1;
  const int pr = pairs > 0 ? tid % pairs : 0, k = pairs > 0 ? tid / pairs : ch;
  const bool act = k < ch;
  const int hh = pairs > 0 ? pr / n4 : 0, c4 = pairs > 0 ? pr - hh * n4 : 0;
  const int nsp = act ? (ns - k + ch - 1) / ch : 0;  // splits of this thread
  const float4* xb = reinterpret_cast<const float4*>(recs + (size_t)hh * A.rec_stride + 4) + c4;
  // the first 16 of this thread's records are loaded while the weights are formed
  float4 x[16];
#pragma unroll
  for (int u = 0; u < 16; ++u)
    x[u] = u < nsp ? __ldcg(xb + (size_t)(k + u * ch) * (hs / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
  // W_up^V of this head into the (idle) stage ring while the records merge
  if (tid == 0 && wv_staged && wv_bytes > 0) {
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&bars[kMaxStages], wv_bytes);
    bulk_copy_g2s(wv_s, cd->w_up + hm[7], wv_bytes, &bars[kMaxStages]);
  }
  if (warp < gq) {  // warp h: the maximum and the weights of the splits for head h
    const int h = warp;
    float2 ml[kMaxSplit / 32];
    float M = -CUDART_INF_F;
#pragma unroll
    for (int r = 0; r < kMaxSplit / 32; ++r) {
      const int sp = lane + 32 * r;
      ml[r] = sp < ns ? __ldcg(reinterpret_cast<const float2*>(recs + sp * hs + h * A.rec_stride))
                      : make_float2(-CUDART_INF_F, 0.f);
      M = fmaxf(M, ml[r].x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Ls = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxSplit / 32; ++r) {
      const int sp = lane + 32 * r;
      if (sp < ns) {
        const float wt = (ml[r].x == -CUDART_INF_F) ? 0.f : ex2_approx(ml[r].x - M);
        wts[h * kMaxSplit + sp] = wt;
        Ls = fmaf(wt, ml[r].y, Ls);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    if (lane == 0) lsum[h] = Ls;
  }
  __syncthreads();
  if (act) {
    const float* wt = wts + hh * kMaxSplit + k;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const float w = u < nsp ? wt[u * ch] : 0.f;
      v.x = fmaf(w, x[u].x, v.x);
      v.y = fmaf(w, x[u].y, v.y);
      v.z = fmaf(w, x[u].z, v.z);
      v.w = fmaf(w, x[u].w, v.w);
    }
    for (int u0 = 16; u0 < nsp; u0 += 16) {
#pragma unroll
      for (int u = 0; u < 16; ++u)
        x[u] = u0 + u < nsp ? __ldcg(xb + (size_t)(k + (u0 + u) * ch) * (hs / 4))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float w = u0 + u < nsp ? wt[(u0 + u) * ch] : 0.f;
        v.x = fmaf(w, x[u].x, v.x);
        v.y = fmaf(w, x[u].y, v.y);
        v.z = fmaf(w, x[u].z, v.z);
        v.w = fmaf(w, x[u].w, v.w);
      }
    }
    reinterpret_cast<float4*>(part)[(size_t)k * pairs + pr] = v;
  }
  bool wv_ok = true;
  if (wv_staged && wv_bytes > 0) wv_ok = mbar_wait_bounded(&bars[kMaxStages], 0u, A.wait_ns);
  if (!wv_ok && tid == 0) device_error(cd->err, SPECTRA_ERR_TIMEOUT);
  __syncthreads();
  // chunks added in order into chunk 0: acc[h][c] = part[h * 4 n4 + c]
  for (int e = tid; e < pairs * 4; e += kThreads) {
    float v = part[e];
    for (int kk = 1; kk < ch; ++kk) v += part[(size_t)kk * pairs * 4 + e];
    part[e] = v;
  }
  __syncthreads();
  const float* acc = part;
  const int acc_ld = 4 * n4;
  // out = (merged latent sums / L) W_up^V: thread (h, 4 consecutive dims)
  const float* wv = wv_staged ? wv_s : cd->w_up + hm[7];
  for (int e = tid; e < gq * (d_h / 4); e += kThreads) {
    const int h = e / (d_h / 4), d4 = e - h * (d_h / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (wv_ok) {
      for (int c = 0; c < nkV; ++c) {
        const float x = acc[h * acc_ld + c];
        const float4 w = reinterpret_cast<const float4*>(wv + (size_t)c * d_h)[d4];
        v.x = fmaf(x, w.x, v.x);
        v.y = fmaf(x, w.y, v.y);
        v.z = fmaf(x, w.z, v.z);
        v.w = fmaf(x, w.w, v.w);
      }
    }
    const float Ls = lsum[h];
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    reinterpret_cast<float4*>(A.out + ((size_t)b * A.n_q + (size_t)a * gq + h) * d_h)[d4] =
        make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
  }
  // every CTA of this unit has arrived: the counter is free for the next call
  // (which starts only after this grid has completed)
  if (tid == 0) A.cnt[unit] = 0;
}


}  // namespace attend
}  // namespace spectra
