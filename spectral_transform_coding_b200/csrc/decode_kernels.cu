// Decode side of libspectra: attention over the packed latent cache, computed in
// the latent space ("SPECTRA: Pushing the KV Cache Beyond the 2-Bit Cliff via
// Spectral Transform Coding", "Significance and claims": the latent structure
// allows attention directly in latent space; "SPECTRA pipeline" stage 3: the
// rebuilt keys/values feed standard softmax attention).
//
// For q head h of KV head a and latent key c_K = code*s + z (per group):
//   q . k = q . (c_K W_up^K) = q_lat . c_K,   q_lat = q W_up^K^T,
//   q_lat . c_K = sum_j [ s_j (q_lat,j . code_j) + z_j (sum_{k in j} q_lat,k) ].
// The integer codes are exact in fp16, so the per-group dot products run on the
// tensor cores (mma.sync m16n8k16 / m16n8k8, fp32 accumulate) with q_lat split
// into fp16 hi + lo columns; scales and the z term are applied in fp32.  Values
// are accumulated as sum_t p_t c_V,t (fp16 dequantised codes x fp16 p, fp32
// accumulate) and W_up^V is applied once per head after the split-K merge.
#include <cuda_fp16.h>
#include <math_constants.h>

#include <algorithm>

#include "device_common.cuh"
#include "kernels.h"

namespace spectra {

namespace {

constexpr int kDecWarps = 4;
constexpr int kMaxG = 8;         // kept groups per side handled by the decode kernel
constexpr int kQStride = 128;    // q_lat row stride (max kept K coordinates)
constexpr uint64_t kWaitLimitNs = 200ull * 1000ull * 1000ull;  // bounded mbarrier waits
constexpr float kPScaleLog2 = 8.f;  // p is formed as 2^(s - m + 8) so fp16 keeps small weights

struct DecodeArgs {
  const CodecDev* cd;
  const uint8_t* pool;
  const int32_t* page_table;
  const int32_t* lengths;
  const float* qlat;
  const float* qsum;
  float* part;
  int64_t n_pool_pages;
  int64_t page_bytes;
  int max_pages;
  int n_split;
  int stages;
  int stage_bytes;
  int part_stride;
  int n_q;
};

__device__ __forceinline__ uint32_t sel4(const uint32_t (&v)[kMaxG], int t4, int odd) {
  const uint32_t a = odd ? v[1] : v[0];
  const uint32_t b = odd ? v[3] : v[2];
  const uint32_t c = odd ? v[5] : v[4];
  const uint32_t d = odd ? v[7] : v[6];
  return (t4 & 2) ? ((t4 & 1) ? d : c) : ((t4 & 1) ? b : a);
}

// Gather the codes of one plane set into 4-bit fields: rotating plane p's word
// right by (t4 - p) lands this lane's 8 bits of the block at bits 4*slot + p.
template <int MAXB>
__device__ __forceinline__ void gather_nibbles(const uint8_t* pw, int plane_stride, int b, int t4,
                                               uint32_t& lo, uint32_t& hi) {
  lo = 0u;
  hi = 0u;
#pragma unroll
  for (int p = 0; p < MAXB; ++p) {
    if (p < b) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(pw + p * plane_stride);
      const uint32_t r = __funnelshift_r(w, w, (uint32_t)(t4 - (p & 3)) & 31u);
      if (p < 4) lo |= r & (0x11111111u << p);
      else hi |= r & (0x11111111u << (p - 4));
    }
  }
}

// Element pair (slot i, slot i+4) as two 16-bit integers (code in bits 0..7).
__device__ __forceinline__ uint32_t slot_pair(uint32_t lo, uint32_t hi, int i, int b) {
  uint32_t v = (lo >> (4 * i)) & 0x000F000Fu;
  if (b > 4) v |= ((hi >> (4 * i)) & 0x000F000Fu) << 4;
  return v;
}

// ---- keys: scores of one 16-token tile -------------------------------------
// Returns sc[nt][r]: score (log2 units) of token 2*gid + r of the tile for head
// nt*4 + t4 of this KV head (before masking).
template <int G, int NT>
__device__ __forceinline__ void key_tile(const uint8_t* __restrict__ sec, int t, int P, int nK,
                                         uint32_t kw, const int (&kpl)[kMaxG],
                                         const uint32_t (&bq)[kMaxG][NT][2],
                                         const uint32_t (&bz)[NT][2], int gid, int t4,
                                         float (&sc)[NT][2]) {
  const int plane_stride = P * G / 8;
  const int blk = (G == 16) ? t : (t >> 1);
  const int mi = (G == 16) ? 0 : (t & 1);
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[nt][r] = 0.f;
  uint32_t zz[kMaxG];
#pragma unroll
  for (int j = 0; j < kMaxG; ++j) {
    zz[j] = 0u;
    if (j < nK) {
      const int bj = (kw >> (4 * j)) & 15;
      uint32_t lo, hi;
      gather_nibbles<8>(sec + kpl[j] + blk * 32 + gid * 4, plane_stride, bj, t4, lo, hi);
      const uint2 rec =
          *reinterpret_cast<const uint2*>(sec + kpl[j] + bj * plane_stride + (t * 8 + gid) * 8);
      zz[j] = rec.y;
      const float sA = half_lo(rec.x), sB = half_hi(rec.x);
      // Codes enter the MMA as fp16 subnormals (value code * 2^-24, exact); the
      // 2^24 is restored after the loop.
      if (G == 16) {
        uint32_t av[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = slot_pair(lo, hi, i, bj);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float d[4] = {0.f, 0.f, 0.f, 0.f};
          mma_m16n8k16(d, av, bq[j][nt]);
          acc[nt][0] = fmaf(sA, d[0], acc[nt][0]);
          acc[nt][1] = fmaf(sA, d[1], acc[nt][1]);
          acc[nt][2] = fmaf(sB, d[2], acc[nt][2]);
          acc[nt][3] = fmaf(sB, d[3], acc[nt][3]);
        }
      } else {
        uint32_t av[2];
        av[0] = slot_pair(lo, hi, 2 * mi, bj);
        av[1] = slot_pair(lo, hi, 2 * mi + 1, bj);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float d[4] = {0.f, 0.f, 0.f, 0.f};
          mma_m16n8k8(d, av, bq[j][nt][0]);
          acc[nt][0] = fmaf(sA, d[0], acc[nt][0]);
          acc[nt][1] = fmaf(sA, d[1], acc[nt][1]);
          acc[nt][2] = fmaf(sB, d[2], acc[nt][2]);
          acc[nt][3] = fmaf(sB, d[3], acc[nt][3]);
        }
      }
    }
  }
  // z term for all groups at once: rows = tokens, k = group index, n = (head, hi/lo).
  const uint32_t zA = sel4(zz, t4, 0), zB = sel4(zz, t4, 1);
  const uint32_t az[4] = {__byte_perm(zA, zB, 0x5410), __byte_perm(zA, zB, 0x7632), 0u, 0u};
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float dz[4] = {0.f, 0.f, 0.f, 0.f};
    mma_m16n8k16(dz, az, bz[nt]);
    sc[nt][0] = fmaf(acc[nt][0] + acc[nt][1], 16777216.f, dz[0] + dz[1]);
    sc[nt][1] = fmaf(acc[nt][2] + acc[nt][3], 16777216.f, dz[2] + dz[3]);
  }
}

// ---- values: accumulate sum_t p_t c_V,t of one 16-token tile ------------------
template <int G>
__device__ __forceinline__ void value_tile(const uint8_t* __restrict__ sec, int t, int P, int nV,
                                           uint32_t vw, const int (&vpl)[kMaxG], const uint32_t (&pb)[2],
                                           int gid, int t4, int n_valid, float (&vacc)[kMaxG][4]) {
  const int plane_stride = P * G / 8;
  const int blk = (G == 16) ? t : (t >> 1);
  const int mi = (G == 16) ? 0 : (t & 1);
  uint32_t m0 = 0xffffffffu, m1 = 0xffffffffu;
  if (n_valid < 16) {
    m0 = ((2 * t4 < n_valid) ? 0x0000ffffu : 0u) | ((2 * t4 + 1 < n_valid) ? 0xffff0000u : 0u);
    m1 = ((2 * t4 + 8 < n_valid) ? 0x0000ffffu : 0u) | ((2 * t4 + 9 < n_valid) ? 0xffff0000u : 0u);
  }
  const uint32_t k1024 = 0x64006400u;  // half2(1024, 1024)
#pragma unroll
  for (int j = 0; j < kMaxG; ++j) {
    if (j < nV) {
      const int bj = (vw >> (4 * j)) & 15;
      uint32_t lo, hi;
      gather_nibbles<8>(sec + vpl[j] + blk * 32 + gid * 4, plane_stride, bj, t4, lo, hi);
      const uint8_t* rb = sec + vpl[j] + bj * plane_stride + t * 64;
      const uint2 r0 = *reinterpret_cast<const uint2*>(rb + t4 * 8);
      const uint2 r1 = *reinterpret_cast<const uint2*>(rb + (t4 + 4) * 8);
      const uint32_t s0 = r0.x & m0, z0 = r0.y & m0, s1 = r1.x & m1, z1 = r1.y & m1;
      uint32_t av[4];
      if (G == 16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = hsub2_u32(slot_pair(lo, hi, i, bj) | k1024, k1024);
        av[0] = hfma2_u32(av[0], s0, z0);
        av[1] = hfma2_u32(av[1], s0, z0);
        av[2] = hfma2_u32(av[2], s1, z1);
        av[3] = hfma2_u32(av[3], s1, z1);
      } else {
        av[0] = hfma2_u32(hsub2_u32(slot_pair(lo, hi, mi, bj) | k1024, k1024), s0, z0);
        av[2] = hfma2_u32(hsub2_u32(slot_pair(lo, hi, mi + 2, bj) | k1024, k1024), s1, z1);
        av[1] = 0u;
        av[3] = 0u;
      }
      mma_m16n8k16(vacc[j], av, pb);
    }
  }
}

template <int G, int NT>
__global__ void __launch_bounds__(kDecWarps * 32) decode_split_kernel(const DecodeArgs A) {
  const CodecDev* __restrict__ cd = A.cd;
  const int split = blockIdx.x, a = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, t4 = lane & 3;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem) + warp * 8;
  uint8_t* region = smem + 128 * 4;
  uint8_t* my_stages = region + (size_t)warp * A.stages * A.stage_bytes;

  const int P = cd->P, gq = cd->gq;
  const HeadDev* hd = &cd->head[a];
  const int sec_off = hd->sec_off, sec_bytes = hd->sec_bytes;
  const int len = A.lengths[b];
  const int n_pages = (len + P - 1) / P;
  const int per = (n_pages + A.n_split - 1) / A.n_split;
  const int p0 = min(split * per, n_pages), p1 = min(p0 + per, n_pages);
  const int count = (p1 - p0 > warp) ? (p1 - p0 - warp + kDecWarps - 1) / kDecWarps : 0;

  // group descriptors of this head: widths packed 4 bits each, plane offsets
  // relative to the head section
  const SideDev* sk = &hd->side[0];
  const SideDev* sv = &hd->side[1];
  const int nK = sk->n_groups, nV = sv->n_groups;
  uint32_t kw = 0, vw = 0;
  int kpl[kMaxG], vpl[kMaxG];
#pragma unroll
  for (int j = 0; j < kMaxG; ++j) {
    kpl[j] = 0;
    vpl[j] = 0;
    if (j < nK) {
      kw |= (uint32_t)sk->grp[j].b << (4 * j);
      kpl[j] = sk->grp[j].plane_off - sec_off;
    }
    if (j < nV) {
      vw |= (uint32_t)sv->grp[j].b << (4 * j);
      vpl[j] = sv->grp[j].plane_off - sec_off;
    }
  }

  // q_lat as B fragments: column n = gid of n-tile nt is head nt*4 + gid/2,
  // part gid&1 (0: fp16(q), 1: fp16(q - fp16(q))).
  uint32_t bq[kMaxG][NT][2];
  uint32_t bz[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hl = nt * 4 + (gid >> 1);
    const int part = gid & 1;
    const bool live = hl < gq;
    const size_t row = (size_t)(b * A.n_q + a * gq + (live ? hl : 0));
    const float* ql = A.qlat + row * kQStride;
    const float* qs = A.qsum + row * kMaxG;
    auto split_h = [&](float v) -> float {
      const float hi = __half2float(__float2half_rn(v));
      return part ? (v - hi) : hi;
    };
#pragma unroll
    for (int j = 0; j < kMaxG; ++j) {
      bq[j][nt][0] = 0u;
      bq[j][nt][1] = 0u;
      if (live && j < nK) {
        const float* base = ql + j * G;
        bq[j][nt][0] = pack_half2(split_h(base[2 * t4]), split_h(base[2 * t4 + 1]));
        if (G == 16) bq[j][nt][1] = pack_half2(split_h(base[2 * t4 + 8]), split_h(base[2 * t4 + 9]));
      }
    }
    bz[nt][0] = live ? pack_half2(split_h(2 * t4 < nK ? qs[2 * t4] : 0.f),
                                  split_h(2 * t4 + 1 < nK ? qs[2 * t4 + 1] : 0.f))
                     : 0u;
    bz[nt][1] = 0u;
  }

  float m_run[NT], l_run[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt] = -CUDART_INF_F;
    l_run[nt] = 0.f;
  }
  float vacc[kMaxG][4];
#pragma unroll
  for (int j = 0; j < kMaxG; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) vacc[j][c] = 0.f;

  // validate this warp's page ids before any copy is issued
  bool bad = false;
  for (int i = lane; i < count; i += 32) {
    const int pid = A.page_table[(size_t)b * A.max_pages + p0 + warp + kDecWarps * i];
    bad |= (pid < 0 || (int64_t)pid >= A.n_pool_pages);
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) device_error(cd->err, SPECTRA_ERR_INVALID);
    return;
  }

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
    for (int i = 0; i < min(S, count); ++i) issue(i);

  bool timed_out = false;
  int i = 0;
  for (; i < count; ++i) {
    const int s = i % S;
    const bool ok = mbar_wait_bounded(&bars[s], (uint32_t)((i / S) & 1), kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ok)) {
      timed_out = true;
      break;
    }
    const uint8_t* sec = my_stages + (size_t)s * A.stage_bytes;
    const int pg = p0 + warp + kDecWarps * i;
    const int n_valid = min(P, len - pg * P);
    for (int c0 = 0; c0 < P / 16 && c0 * 16 < n_valid; c0 += 4) {
      float sc[4][NT][2];
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const int t = c0 + tt;
        if (t < P / 16 && t * 16 < n_valid) {
          key_tile<G, NT>(sec, t, P, nK, kw, kpl, bq, bz, gid, t4, sc[tt]);
          const int nv = n_valid - t * 16;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (2 * gid >= nv) sc[tt][nt][0] = -CUDART_INF_F;
            if (2 * gid + 1 >= nv) sc[tt][nt][1] = -CUDART_INF_F;
          }
        } else {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) sc[tt][nt][0] = sc[tt][nt][1] = -CUDART_INF_F;
        }
      }
      // online softmax over this chunk of up to 64 tokens
      float alpha[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) mx = fmaxf(mx, fmaxf(sc[tt][nt][0], sc[tt][nt][1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run[nt], mx);
        alpha[nt] = exp2f(m_run[nt] - m_new);
        m_run[nt] = m_new;
        l_run[nt] *= alpha[nt];
      }
      {
        // V accumulators hold heads 2*t4 and 2*t4+1
        float ae = __shfl_sync(0xffffffffu, alpha[0], (2 * t4) & 3);
        float ao = __shfl_sync(0xffffffffu, alpha[0], (2 * t4 + 1) & 3);
        if (NT == 2) {
          const float be = __shfl_sync(0xffffffffu, alpha[NT - 1], (2 * t4) & 3);
          const float bo = __shfl_sync(0xffffffffu, alpha[NT - 1], (2 * t4 + 1) & 3);
          if (t4 >= 2) {
            ae = be;
            ao = bo;
          }
        }
#pragma unroll
        for (int j = 0; j < kMaxG; ++j) {
          vacc[j][0] *= ae;
          vacc[j][1] *= ao;
          vacc[j][2] *= ae;
          vacc[j][3] *= ao;
        }
      }
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const int t = c0 + tt;
        if (t < P / 16 && t * 16 < n_valid) {
          uint32_t p01[NT];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const float pa = exp2f(sc[tt][nt][0] - m_run[nt] + kPScaleLog2);
            const float pbv = exp2f(sc[tt][nt][1] - m_run[nt] + kPScaleLog2);
            l_run[nt] += pa + pbv;
            p01[nt] = pack_half2(pa, pbv);
          }
          const int src0 = (t4 << 2) | (gid & 3), src1 = ((t4 + 4) << 2) | (gid & 3);
          uint32_t pb[2];
          pb[0] = __shfl_sync(0xffffffffu, p01[0], src0);
          pb[1] = __shfl_sync(0xffffffffu, p01[0], src1);
          if (NT == 2) {
            const uint32_t y0 = __shfl_sync(0xffffffffu, p01[NT - 1], src0);
            const uint32_t y1 = __shfl_sync(0xffffffffu, p01[NT - 1], src1);
            if (gid >= 4) {
              pb[0] = y0;
              pb[1] = y1;
            }
          }
          if (gid >= gq) pb[0] = pb[1] = 0u;
          value_tile<G>(sec, t, P, nV, vw, vpl, pb, gid, t4, n_valid - t * 16, vacc);
        }
      }
    }
    __syncwarp();
    if (lane == 0 && i + S < count) {
      fence_proxy_async_smem();
      issue(i + S);
    }
  }
  if (timed_out) {
    if (lane == 0) {
      device_error(cd->err, SPECTRA_ERR_TIMEOUT);
      for (int k = i; k < min(i + S, count); ++k)  // let copies still in flight land
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

  // merge the warps of this CTA, then write one partial record per q head
  __syncthreads();
  const int maxV = cd->max_kept_v;
  const int rec = 2 + maxV;
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
#pragma unroll
  for (int j = 0; j < kMaxG; ++j) {
    if (j < nV) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int hl = 2 * t4 + (c & 1);
        const int coord = j * G + gid + ((c >> 1) ? 8 : 0);
        if (hl < gq && (G == 16 || c < 2)) wsm[(warp * gq + hl) * rec + 2 + coord] = vacc[j][c];
      }
    }
  }
  __syncthreads();
  const int nkv = sv->n_kept;
  for (int idx = threadIdx.x; idx < gq * (2 + nkv); idx += blockDim.x) {
    const int hl = idx / (2 + nkv), c = idx % (2 + nkv);
    float M = -CUDART_INF_F;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wsm[(w * gq + hl) * rec]);
    float v = 0.f;
    if (c == 0) {
      v = M;
    } else if (M != -CUDART_INF_F) {
      for (int w = 0; w < kDecWarps; ++w) {
        const float mw = wsm[(w * gq + hl) * rec];
        if (mw != -CUDART_INF_F) {
          const float wgt = exp2f(mw - M);
          v += wgt * wsm[(w * gq + hl) * rec + (c == 1 ? 1 : c)];
        }
      }
    }
    const int h = a * gq + hl;
    A.part[((size_t)(b * A.n_q + h) * A.n_split + split) * A.part_stride + c] = v;
  }
}

// q_lat = (q W_up^K^T) * log2(e)/sqrt(d_h) for the kept K coordinates, and the
// per-group sums of q_lat.  One block per (q head, sequence), one warp per row.
__global__ void __launch_bounds__(128) fold_query_kernel(const CodecDev* __restrict__ cd,
                                                         const float* __restrict__ q,
                                                         float* __restrict__ qlat,
                                                         float* __restrict__ qsum, float scale) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int n_q = cd->n_q, d_h = cd->d_h, gq = cd->gq;
  const int a = h / gq;
  const SideDev& sk = cd->head[a].side[0];
  __shared__ float qs[kMaxDHead];
  __shared__ float ql[kQStride];
  const float* qrow = q + ((size_t)b * n_q + h) * d_h;
  for (int d = threadIdx.x; d < d_h; d += blockDim.x) qs[d] = qrow[d];
  __syncthreads();
  const float* W = cd->w_up + sk.wup_off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row = (size_t)b * n_q + h;
  for (int c = warp; c < sk.n_kept; c += 4) {
    float acc = 0.f;
    for (int d = lane; d < d_h; d += 32) acc = fmaf(qs[d], W[(size_t)c * d_h + d], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      ql[c] = acc * scale;
      qlat[row * kQStride + c] = acc * scale;
    }
  }
  __syncthreads();
  const int G = cd->group;
  if (threadIdx.x < kMaxG) {
    const int j = threadIdx.x;
    float s = 0.f;
    if (j < sk.n_groups)
      for (int k = 0; k < G; ++k) s += ql[j * G + k];
    qsum[row * kMaxG + j] = s;
  }
}

// Merge the split partials of one (sequence, q head) and apply W_up^V:
// out = (sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s) W_up^V.
__global__ void __launch_bounds__(128) combine_kernel(const CodecDev* __restrict__ cd,
                                                      const float* __restrict__ part, int n_split,
                                                      int part_stride, float* __restrict__ out) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int n_q = cd->n_q, d_h = cd->d_h, gq = cd->gq;
  const int a = h / gq;
  const SideDev& sv = cd->head[a].side[1];
  const int nkv = sv.n_kept;
  extern __shared__ float sm[];
  float* wgt = sm;              // [n_split]
  float* olat = sm + n_split;   // [nkv]
  __shared__ float L_sh;
  const float* pr = part + ((size_t)b * n_q + h) * n_split * part_stride;
  if (threadIdx.x == 0) {
    float M = -CUDART_INF_F;
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, pr[(size_t)s * part_stride]);
    float L = 0.f;
    for (int s = 0; s < n_split; ++s) {
      const float ms = pr[(size_t)s * part_stride];
      const float w = (M == -CUDART_INF_F || ms == -CUDART_INF_F) ? 0.f : exp2f(ms - M);
      wgt[s] = w;
      L += w * pr[(size_t)s * part_stride + 1];
    }
    L_sh = L;
  }
  __syncthreads();
  const float L = L_sh;
  const float invL = L > 0.f ? 1.f / L : 0.f;
  for (int c = threadIdx.x; c < nkv; c += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < n_split; ++s) acc = fmaf(wgt[s], pr[(size_t)s * part_stride + 2 + c], acc);
    olat[c] = acc * invL;
  }
  __syncthreads();
  const float* W = cd->w_up + sv.wup_off;  // [nkv][d_h]
  float* orow = out + ((size_t)b * n_q + h) * d_h;
  for (int d = threadIdx.x; d < d_h; d += blockDim.x) {
    float acc = 0.f;
    for (int c = 0; c < nkv; ++c) acc = fmaf(olat[c], W[(size_t)c * d_h + d], acc);
    orow[d] = acc;
  }
}

template <int G, int NT>
cudaError_t launch_split(const DecodeArgs& args, dim3 grid, int smem, cudaStream_t st) {
  static int configured_smem = -1;
  if (smem > configured_smem) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<G, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured_smem = smem;
  }
  decode_split_kernel<G, NT><<<grid, kDecWarps * 32, smem, st>>>(args);
  return cudaGetLastError();
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

}  // namespace

DecodePlan make_decode_plan(const CodecDev& h, int batch, int max_pages_per_seq) {
  DecodePlan p{};
  p.stage_bytes = ((h.max_sec_bytes + 15) / 16) * 16;
  if (p.stage_bytes < 16) p.stage_bytes = 16;
  const int budget = 100 * 1024;
  p.stages = std::max(2, std::min(6, budget / (kDecWarps * p.stage_bytes)));
  const int merge_bytes = kDecWarps * h.gq * (2 + h.max_kept_v) * 4;
  p.smem_bytes = 128 * 4 + std::max(kDecWarps * p.stages * p.stage_bytes, merge_bytes);
  const int units = std::max(1, batch * h.n_kv);
  const int slots = 2 * sm_count();
  int ns = (2 * slots + units - 1) / units;
  ns = std::max(1, std::min(ns, std::max(1, max_pages_per_seq)));
  p.n_split = ns;
  p.part_stride = 2 + h.max_kept_v;
  size_t off = 0;
  auto carve = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  };
  p.qlat_off = carve((size_t)batch * h.n_q * kQStride * 4);
  p.qsum_off = carve((size_t)batch * h.n_q * kMaxG * 4);
  p.part_off = carve((size_t)batch * h.n_q * ns * p.part_stride * 4);
  p.ws_bytes = off;
  return p;
}

cudaError_t launch_decode(const CodecDev& h, const CodecDev* d, const spectra_cache& cache,
                          const float* q, float* out, void* ws, const DecodePlan& plan,
                          cudaStream_t st) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* qlat = reinterpret_cast<float*>(w + plan.qlat_off);
  float* qsum = reinterpret_cast<float*>(w + plan.qsum_off);
  float* part = reinterpret_cast<float*>(w + plan.part_off);
  const float scale = 1.4426950408889634f / sqrtf((float)h.d_h);
  fold_query_kernel<<<dim3(h.n_q, cache.batch), 128, 0, st>>>(d, q, qlat, qsum, scale);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  DecodeArgs args;
  args.cd = d;
  args.pool = static_cast<const uint8_t*>(cache.pool);
  args.page_table = cache.page_table;
  args.lengths = cache.lengths;
  args.qlat = qlat;
  args.qsum = qsum;
  args.part = part;
  args.n_pool_pages = cache.n_pages;
  args.page_bytes = h.page_bytes;
  args.max_pages = cache.max_pages_per_seq;
  args.n_split = plan.n_split;
  args.stages = plan.stages;
  args.stage_bytes = plan.stage_bytes;
  args.part_stride = plan.part_stride;
  args.n_q = h.n_q;
  const dim3 grid(plan.n_split, h.n_kv, cache.batch);
  const bool two = h.gq > 4;
  if (h.group == 16)
    e = two ? launch_split<16, 2>(args, grid, plan.smem_bytes, st)
            : launch_split<16, 1>(args, grid, plan.smem_bytes, st);
  else
    e = two ? launch_split<8, 2>(args, grid, plan.smem_bytes, st)
            : launch_split<8, 1>(args, grid, plan.smem_bytes, st);
  if (e != cudaSuccess) return e;
  const int csm = (plan.n_split + h.max_kept_v) * 4;
  combine_kernel<<<dim3(h.n_q, cache.batch), 128, csm, st>>>(d, part, plan.n_split, plan.part_stride,
                                                              out);
  return cudaGetLastError();
}

}  // namespace spectra
