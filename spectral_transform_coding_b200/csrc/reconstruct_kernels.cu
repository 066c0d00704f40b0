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

#include <algorithm>
#include <cmath>
#include <string>

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

// ---------------------------------------------------------------------------
// Reconstruct-then-attend decode ("SPECTRA pipeline" stage 3 as the pages
// integrate it: keys and values rebuilt from the latents, then standard
// attention).  With rotary position embedding the query cannot be folded into
// the latent space (the rotation depends on the key's position), so each tile
// of keys is rebuilt in shared memory, rotated, and scored there:
//
//   k^_t = R(t) (c^_K,t W_up^K),  q' = R(L-1) q,  p = softmax(q' k^^T / sqrt(d_h))
//   o = sum_t p_t v^_t = (sum_t p_t c^_V,t) W_up^V
//
// v^ is never materialised: by linearity the V lift runs once per head on the
// probability-weighted latent sum, after the splits are merged.  R(p) turns the
// pair (i, i + d_h/2) by p * theta^(-2i/d_h); theta = 0 means no rotation.
//
// One CTA per (KV head, sequence, context split), 256 threads, 32-token tiles:
//   1. unpack the tile's K codes into shared memory as fp16 (exact: codes are
//      integers below 256) with their per-group s and z, and dequantise the V
//      latents (fp32);
//   2. lift on the tensor cores (mma.sync): per group j,
//        P_j = code_j W_j  (W_up^K rows of group j split into fp16 hi + lo,
//                           so P_j keeps about 22 bits; fp32 accumulate)
//        k^ += s_j P_j + z_j (sum of the rows of W_j)
//      in 16-token x 8-dim tiles, a warp holding a dim and its rotation
//      partner d + d_h/2 in the same registers; then the rotation, the keys
//      overwriting the consumed codes (two CTAs fit an SM at d_h = 128);
//   3. scores of the KV head's q heads, online softmax (exp2 domain), and the
//      probability-weighted sum of the V latents in registers.
// A combine kernel merges the splits and applies W_up^V.
// ---------------------------------------------------------------------------
constexpr int kRtTokens = 32;
constexpr int kRtPairsPerWarp = 2;  // m-tiles (16 tokens) per warp and tile for its 8-dim pair: d_h <= 128
constexpr int kRtThreads = 256;
constexpr int kRtMaxSplit = 64;
constexpr int kRtAccSlots = kMaxGQ * kRtMaxDHead / kRtThreads;  // V accumulators per thread

// Byte offsets of the split kernel's shared-memory regions (max_k, max_v:
// largest kept coordinates per side over the heads; G: group size).
struct RtSmem {
  int om, bf, ws, ck, sz, cv, kh, qs, sc, ml, rb, pg, gt, rw, total;
  int ck_stride, n_grp;  // halves per K code row; groups per side (max)
  // raw_bytes: bytes of one tile's slice of a page's head section
  __host__ __device__ RtSmem(int d_h, int max_k, int max_v, int gq, int G, int raw_bytes) {
    ck_stride = max_k + 8;
    n_grp = max_k / G > 0 ? max_k / G : 1;
    int o = 0;
    om = o;  // rotation frequencies in half-turns per position, double [d_h / 2]
    o += kRtMaxDHead / 2 * 8;
    bf = o;  // W_up^K as MMA B fragments: fp16 hi and lo, [group][n-tile][hi, lo][G/8][32 lanes] words
    o += max_k * d_h * 4;
    ws = o;  // per group, the sum of its rows of W_up^K [group][d_h]
    o += n_grp * d_h * 4;
    // K codes, fp16 [kRtTokens][ck_stride], then K scale and zero, fp32
    // [2][kRtTokens][n_grp]; once the lift has read them, the same bytes hold
    // the rotated keys [kRtTokens][d_h + 1]
    ck = o;
    sz = ck + (kRtTokens * ck_stride * 2 + 15) / 16 * 16;
    const int lift_in = sz - ck + 2 * kRtTokens * n_grp * 4;
    const int keys = kRtTokens * (d_h + 1) * 4;
    kh = ck;
    o += ((lift_in > keys ? lift_in : keys) + 15) / 16 * 16;
    cv = o;  // V latents [kRtTokens][max_v + 1]
    o += (kRtTokens * (max_v + 1) * 4 + 15) / 16 * 16;
    qs = o;  // rotated, scaled queries [gq][d_h]
    o += gq * d_h * 4;
    sc = o;  // scores, then probabilities [gq][kRtTokens]
    o += gq * kRtTokens * 4;
    ml = o;  // running max, sum and correction per q head
    o += 3 * kMaxGQ * 4;
    o = (o + 15) / 16 * 16;
    rb = o;  // rotation of the tile's first position: {cos, sin} [d_h / 2]
    o += kRtMaxDHead / 2 * 8;
    pg = o;  // byte offset of the current and the next tile's page in the pool (-1: bad page id)
    o += 16;
    gt = o;  // per kept group {plane_off, sz_off, width, offset in rw}: at most 32 over both sides
    o += kMaxGroups * 16;
    rw = o;  // the tile's codes and records, per kept group
    o += (raw_bytes + 15) / 16 * 16;
    total = o;
  }
};

struct RtArgs {
  const CodecDev* cd;
  const uint8_t* pool;
  const int32_t* page_table;
  const int32_t* lengths;
  int64_t n_pool_pages;
  int max_pages;
  int n_split;
  int part_stride;  // floats per partial record: max, sum, then the V latent sum
  double theta;     // rotary base; 0 = no rotation
  float qscale;     // log2(e) / sqrt(d_h)
  const float* q;
  float* part;
};

// cos and sin of `turns` * pi radians.  The angle, in half-turns, is reduced to
// [-1, 1] in double (turns - 2 rint(turns / 2), exact up to the rounding of
// `turns` itself), then sin(pi r) and cos(pi r) run in fp32.
__device__ __forceinline__ float2 rope_cos_sin(double turns) {
  const double k = rint(turns * 0.5);
  const float r = (float)fma(-2.0, k, turns);
  float sn, cs;
  sincospif(r, &sn, &cs);
  return make_float2(cs, sn);
}

// Turns (x, y) by the angle whose {cos, sin} is cs.
__device__ __forceinline__ void rope_apply(float& x, float& y, float2 cs) {
  const float x2 = x * cs.x - y * cs.y, y2 = y * cs.x + x * cs.y;
  x = x2;
  y = y2;
}

__device__ __forceinline__ void rope_rotate(float& x, float& y, double turns) { rope_apply(x, y, rope_cos_sin(turns)); }

// The rotation of the sum of two angles from their {cos, sin}.
__device__ __forceinline__ float2 rope_add(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.y * b.x + a.x * b.y);
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The G codes of one token in one group of width b (warp-uniform) from its
// block staged in shared memory; G and the side are compile-time, so the
// fragment positions fold to constants and the word loads issue together.
template <int G, int SIDE>
__device__ __forceinline__ void unpack_token(const uint32_t* blk, int b, int tb, uint32_t (&code)[G]) {
  int gid[G], t4[G], slot[G];
#pragma unroll
  for (int k = 0; k < G; ++k) frag_pos(G, SIDE, tb, k, &gid[k], &t4[k], &slot[k]);
  switch (b) {
    case 4:
#pragma unroll
      for (int k = 0; k < G; ++k) code[k] = (blk[4 * gid[k] + t4[k]] >> (4 * slot[k])) & 0xFu;
      break;
    case 2:
#pragma unroll
      for (int k = 0; k < G; ++k) code[k] = (blk[2 * gid[k] + (t4[k] >> 1)] >> (4 * slot[k] + 2 * (t4[k] & 1))) & 0x3u;
      break;
    case 1:
#pragma unroll
      for (int k = 0; k < G; ++k) code[k] = (blk[gid[k]] >> (4 * slot[k] + t4[k])) & 0x1u;
      break;
    case 3:
#pragma unroll
      for (int k = 0; k < G; ++k)
        code[k] = ((blk[2 * gid[k] + (t4[k] >> 1)] >> (4 * slot[k] + 2 * (t4[k] & 1))) & 0x3u) |
                  (((blk[16 + gid[k]] >> (4 * slot[k] + t4[k])) & 0x1u) << 2);
      break;
    default:
#pragma unroll
      for (int k = 0; k < G; ++k)
        code[k] = (blk[2 * (4 * gid[k] + t4[k]) + ((slot[k] >> 1) & 1)] >> (8 * ((slot[k] & 1) + 2 * (slot[k] >> 2)))) &
                  0xFFu;
      break;
  }
}

template <int G>
__global__ void __launch_bounds__(kRtThreads) rt_split_kernel(const RtArgs A) {
  extern __shared__ __align__(16) uint8_t sm[];
  const CodecDev* cd = A.cd;
  const int a = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d_h = cd->d_h, half = d_h / 2, gq = cd->gq, P = cd->P;
  constexpr int TB = 256 / G;
  const SideDev& sk = cd->head[a].side[0];
  const SideDev& sv = cd->head[a].side[1];
  const int nkK = sk.n_kept, nkV = sv.n_kept, cvs = cd->max_kept_v + 1;
  // P is a multiple of the tile (the codec requires a multiple of 32), so a
  // tile never straddles a page: each tile's slice of the head section is
  // staged in shared memory by async copies issued one tile ahead
  const RtSmem L(d_h, cd->max_kept_k, cd->max_kept_v, gq, G, cd->max_sec_bytes / P * kRtTokens);
  const int cks = L.ck_stride, ngs = L.n_grp, n_nt = d_h / 8, half_nt = n_nt / 2;
  constexpr int KQ = G / 8;  // B fragment registers per lane (m16n8k16: 2, m16n8k8: 1)
  double* om = reinterpret_cast<double*>(sm + L.om);
  uint32_t* bf = reinterpret_cast<uint32_t*>(sm + L.bf);
  float* wsum = reinterpret_cast<float*>(sm + L.ws);
  __half* ck = reinterpret_cast<__half*>(sm + L.ck);
  float* szk = reinterpret_cast<float*>(sm + L.sz);  // [0]: s, [kRtTokens * ngs]: z
  float* cV = reinterpret_cast<float*>(sm + L.cv);
  float* kh = reinterpret_cast<float*>(sm + L.kh);  // shares its bytes with ck and szk
  float* qs = reinterpret_cast<float*>(sm + L.qs);
  float* sc = reinterpret_cast<float*>(sm + L.sc);
  float* ml = reinterpret_cast<float*>(sm + L.ml);  // [0, 8) max, [8, 16) sum, [16, 24) correction
  float2* rb = reinterpret_cast<float2*>(sm + L.rb);
  int64_t* pg = reinterpret_cast<int64_t*>(sm + L.pg);
  int4* gt = reinterpret_cast<int4*>(sm + L.gt);
  uint8_t* rw = sm + L.rw;
  const bool rot = A.theta > 0.0;

  // W_up^K (stored transposed, W[c][d] = wk[d * n_kept + c]) as B fragments of
  // an m16n8k(G) MMA per (group j, n-tile of 8 dims): lane (gid, t4) register q
  // holds rows c = jG + 2 t4 + 8 q + {0, 1} of column d = 8 n-tile + gid, as
  // fp16 hi = rn(W) and lo = rn(W - hi); and the column sums of each group
  const float* wk = cd->w_up + sk.wup_off;
  const int ngK = sk.n_groups;
  for (int e = tid; e < ngK * n_nt * KQ * 32; e += kRtThreads) {
    const int ln = e & 31, r = e >> 5, q = r % KQ, nt = (r / KQ) % n_nt, j = r / (KQ * n_nt);
    const int d = 8 * nt + (ln >> 2), c = j * G + 2 * (ln & 3) + 8 * q;
    const float w0 = wk[(size_t)d * nkK + c], w1 = wk[(size_t)d * nkK + c + 1];
    const float h0 = __half2float(__float2half_rn(w0)), h1 = __half2float(__float2half_rn(w1));
    uint32_t* dst = bf + ((j * n_nt + nt) * 2 * KQ + q) * 32 + ln;
    dst[0] = pack_half2(w0, w1);
    dst[KQ * 32] = pack_half2(w0 - h0, w1 - h1);
  }
  for (int e = tid; e < ngK * d_h; e += kRtThreads) {
    const int j = e / d_h, d = e % d_h;
    float acc = 0.f;
    for (int k = 0; k < G; ++k) acc += wk[(size_t)d * nkK + j * G + k];
    wsum[j * d_h + d] = acc;
  }
  if (rot)
    for (int i = tid; i < half; i += kRtThreads) om[i] = pow(A.theta, -2.0 * i / d_h) / 3.141592653589793;
  if (tid < kMaxGQ) {
    ml[tid] = -INFINITY;
    ml[kMaxGQ + tid] = 0.f;
  }
  const int ngAll = sk.n_groups + sv.n_groups;
  if (warp == 1) {
    // per kept group (K then V): page offsets, width and its slot in rw (the
    // tile's 4 G b code bytes, then 8 record pieces of 16 bytes)
    int acc_off = 0, mine = 0;
    for (int jj = 0; jj < ngAll; ++jj) {
      const int bw = (jj < sk.n_groups ? sk.grp[jj] : sv.grp[jj - sk.n_groups]).b;
      if (jj == lane) mine = acc_off;
      acc_off += 4 * G * bw + 128;
    }
    if (lane < ngAll) {
      const GroupDev gd = lane < sk.n_groups ? sk.grp[lane] : sv.grp[lane - sk.n_groups];
      gt[lane] = make_int4(gd.plane_off, gd.sz_off, gd.b, mine);
    }
  }
  int len = A.lengths[b];
  if (len < 0 || (int64_t)len > (int64_t)A.max_pages * P) {
    if (tid == 0) device_error(cd->err, SPECTRA_ERR_INVALID);
    len = 0;
  }
  __syncthreads();
  // queries of this KV head's q heads, turned to position len - 1 and scaled
  for (int e = tid; e < gq * half; e += kRtThreads) {
    const int h = e / half, i = e % half;
    const float* qv = A.q + ((size_t)b * cd->n_q + (size_t)a * gq + h) * d_h;
    float x = qv[i], y = qv[i + half];
    if (rot && len > 0) rope_rotate(x, y, (double)(len - 1) * om[i]);
    qs[h * d_h + i] = x * A.qscale;
    qs[h * d_h + i + half] = y * A.qscale;
  }

  const int tiles = (len + kRtTokens - 1) / kRtTokens;
  const int per = (tiles + A.n_split - 1) / A.n_split;
  const int tok_begin = min(split * per, tiles) * kRtTokens;
  const int tok_end = min(min((split + 1) * per, tiles) * kRtTokens, len);
  const int n_items = kRtTokens * (ngK + sv.n_groups);
  const int n_acc = gq * nkV;
  // The key rotation at position t0 + t is the tile's rotation at t0 (rb, per
  // tile) followed by the rotation at offset t; this thread's (offset, dim)
  // entries of the lift are the same in every tile, so their offset rotations
  // are computed once, here
  float2 roff[kRtPairsPerWarp][4];
  // lift work of this warp: the n-tile pair np (dims 8 np.. and their rotation
  // partners) for the m-tiles mt = q + mi * step (warps that share an np split
  // the m-tiles), so that each B fragment is read once per tile
  const int lift_np = warp % half_nt, lift_q = warp / half_nt, lift_step = max(1, 8 / half_nt);
  const bool lift_on = lift_q < lift_step;
  {
    const int gid = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int mi = 0; mi < kRtPairsPerWarp; ++mi) {
      const int mt = lift_q + mi * lift_step;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = mt * 16 + gid + (r < 2 ? 0 : 8), d = 8 * lift_np + 2 * t4 + (r & 1);
        roff[mi][r] = (rot && lift_on && mt < kRtTokens / 16) ? rope_cos_sin((double)t * om[d])
                                                               : make_float2(1.f, 0.f);
      }
    }
  }

  float acc[kRtAccSlots];
#pragma unroll
  for (int k = 0; k < kRtAccSlots; ++k) acc[k] = 0.f;

  // staged tiles: byte offset of the tile's page in the pool (-1: bad page id),
  // read by thread 0 one tile ahead; the copies of a tile go out while the
  // previous tile is lifted, scored and summed
  auto tile_page = [&](int t0n) -> int64_t {
    const int pid = A.page_table[(size_t)b * A.max_pages + t0n / P];
    if (pid < 0 || (int64_t)pid >= A.n_pool_pages) {
      device_error(cd->err, SPECTRA_ERR_INVALID);
      return -1;
    }
    return (int64_t)pid * cd->page_bytes;
  };
  auto issue_tile = [&](int t0n, int64_t poff) {
    if (poff >= 0) {
      const int tau0 = t0n % P;
      const uint8_t* page = A.pool + poff;
      for (int jj = warp; jj < ngAll; jj += kRtThreads / 32) {
        const int4 g = gt[jj];  // {plane_off, sz_off, width, slot}
        uint8_t* dst = rw + g.w;
        const int ncode = G * g.z / 4;  // 16-byte pieces of the tile's codes (<= 32)
        if (lane < ncode) cp_async16(dst + 16 * lane, page + g.x + (size_t)(tau0 / TB) * 32 * g.z + 16 * lane);
        // records of pairs tau0/2 .. tau0/2 + 15: two per row (u % 8) of the record grid
        if (lane < 8) cp_async16(dst + 4 * G * g.z + 16 * lane, page + g.y + 8 * (lane * (P >> 4) + tau0 / 16));
      }
    }
    cp_async_commit();
  };
  __syncthreads();  // the group table is complete
  if (tid == 0) pg[0] = tok_begin < tok_end ? tile_page(tok_begin) : -1;
  __syncthreads();
  if (tok_begin < tok_end) issue_tile(tok_begin, pg[0]);

  for (int t0 = tok_begin; t0 < tok_end; t0 += kRtTokens) {
    const int nt = min(kRtTokens, tok_end - t0);
    // ---- 1. dequantised latents of the tile (rows past the end are zero) ----
    {
      const int64_t cur = pg[0];
      cp_async_wait_all();
      if (rot)
        for (int i = tid; i < half; i += kRtThreads) rb[i] = rope_cos_sin((double)t0 * om[i]);
      if (tid == 0 && t0 + kRtTokens < tok_end) pg[1] = tile_page(t0 + kRtTokens);
      __syncthreads();  // the tile's bytes have landed (every thread's copies)
      for (int e = tid; e < n_items; e += kRtThreads) {
        const int t = e % kRtTokens, jj = e / kRtTokens;
        const int side = jj < ngK ? 0 : 1, j = side ? jj - ngK : jj;
        uint32_t code[G];
        float sv_ = 0.f, zv = 0.f;
        if (cur < 0 || t >= nt) {
#pragma unroll
          for (int k = 0; k < G; ++k) code[k] = 0u;
        } else {
          const int4 g = gt[jj];
          const uint8_t* slot = rw + g.w;
          const int ul = t >> 1;
          const uint2 rec = *reinterpret_cast<const uint2*>(slot + 4 * G * g.z + 16 * (ul & 7) + 8 * (ul >> 3));
          sv_ = (t & 1) ? half_hi(rec.x) : half_lo(rec.x);
          zv = (t & 1) ? half_hi(rec.y) : half_lo(rec.y);
          const uint32_t* blk = reinterpret_cast<const uint32_t*>(slot + (t / TB) * 32 * g.z);
          if (side == 0)
            unpack_token<G, 0>(blk, g.z, t % TB, code);
          else
            unpack_token<G, 1>(blk, g.z, t % TB, code);
        }
        if (side == 0) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(ck + t * cks + j * G);
#pragma unroll
          for (int k = 0; k < G; k += 2) dst[k / 2] = pack_half2((float)code[k], (float)code[k + 1]);
          szk[t * ngs + j] = sv_;
          szk[(kRtTokens + t) * ngs + j] = zv;
        } else {
          float* dst = cV + t * cvs + j * G;
#pragma unroll
          for (int k = 0; k < G; ++k) dst[k] = fmaf((float)code[k], sv_, zv);
        }
      }
      __syncthreads();  // rw is consumed: the next tile's copies may land in it
      if (t0 + kRtTokens < tok_end) {
        if (tid == 0) pg[0] = pg[1];
        issue_tile(t0 + kRtTokens, pg[1]);
      }
    }
    // ---- 2. k^ = sum_j s_j (code_j W_j) + z_j (sum of W_j) on the tensor cores ----
    {
      const int gid = lane >> 2, t4 = lane & 3;
      constexpr int kMT = kRtTokens / 16;
      float acc[kRtPairsPerWarp][2][4];
#pragma unroll
      for (int mi = 0; mi < kRtPairsPerWarp; ++mi)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[mi][h2][r] = 0.f;
      const int np = lift_np;
      if (lift_on) {  // warp-uniform
        for (int j = 0; j < ngK; ++j) {
          // B fragments (hi, lo) and column sums of the pair's two n-tiles
          uint32_t bh[2][2], bl[2][2];
          float w0[2], w1[2];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int ntl = np + h2 * half_nt;
            const uint32_t* bp = bf + (j * n_nt + ntl) * 2 * KQ * 32 + lane;
            if (G == 16) {
              bh[h2][0] = bp[0];
              bh[h2][1] = bp[32];
              bl[h2][0] = bp[64];
              bl[h2][1] = bp[96];
            } else {
              bh[h2][0] = bp[0];
              bl[h2][0] = bp[32];
              bh[h2][1] = bl[h2][1] = 0u;
            }
            w0[h2] = wsum[j * d_h + 8 * ntl + 2 * t4];
            w1[h2] = wsum[j * d_h + 8 * ntl + 2 * t4 + 1];
          }
#pragma unroll
          for (int mi = 0; mi < kRtPairsPerWarp; ++mi) {
            const int mt = lift_q + mi * lift_step;
            if (mt < kMT) {  // warp-uniform
              const int r0 = mt * 16 + gid, r1 = r0 + 8;
              const __half* a0p = ck + r0 * cks + j * G + 2 * t4;
              const __half* a1p = ck + r1 * cks + j * G + 2 * t4;
              uint32_t af[4];
              af[0] = *reinterpret_cast<const uint32_t*>(a0p);
              af[1] = *reinterpret_cast<const uint32_t*>(a1p);
              if (G == 16) {
                af[2] = *reinterpret_cast<const uint32_t*>(a0p + 8);
                af[3] = *reinterpret_cast<const uint32_t*>(a1p + 8);
              }
              const float s0 = szk[r0 * ngs + j], s1 = szk[r1 * ngs + j];
              const float z0 = szk[(kRtTokens + r0) * ngs + j], z1 = szk[(kRtTokens + r1) * ngs + j];
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                float pr[4] = {0.f, 0.f, 0.f, 0.f};
                if (G == 16) {
                  mma_m16n8k16(pr, af, bh[h2]);
                  mma_m16n8k16(pr, af, bl[h2]);
                } else {
                  mma_m16n8k8(pr, af, bh[h2][0]);
                  mma_m16n8k8(pr, af, bl[h2][0]);
                }
                acc[mi][h2][0] = fmaf(s0, pr[0], fmaf(z0, w0[h2], acc[mi][h2][0]));
                acc[mi][h2][1] = fmaf(s0, pr[1], fmaf(z0, w1[h2], acc[mi][h2][1]));
                acc[mi][h2][2] = fmaf(s1, pr[2], fmaf(z1, w0[h2], acc[mi][h2][2]));
                acc[mi][h2][3] = fmaf(s1, pr[3], fmaf(z1, w1[h2], acc[mi][h2][3]));
              }
            }
          }
        }
      }
      __syncthreads();  // the codes are consumed: their bytes now take the keys
      // rows r0 / r1, dims d (n-tile np) and d + d_h/2 (n-tile np + half_nt)
      if (lift_on) {
#pragma unroll
        for (int mi = 0; mi < kRtPairsPerWarp; ++mi) {
          const int mt = lift_q + mi * lift_step;
          if (mt < kMT) {
            const int r0 = mt * 16 + gid, r1 = r0 + 8;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const int t = r < 2 ? r0 : r1, d = 8 * np + 2 * t4 + (r & 1);
              float x = acc[mi][0][r], y = acc[mi][1][r];
              if (rot) rope_apply(x, y, rope_add(rb[d], roff[mi][r]));
              kh[t * (d_h + 1) + d] = x;
              kh[t * (d_h + 1) + half + d] = y;
            }
          }
        }
      }
    }
    __syncthreads();
    // ---- 3. scores (log2 units), online softmax, V latent sums --------------
    // two threads per (q head, token), each over half of the dims; the second
    // half is walked from a quarter in, so that the pair's rows fall in
    // different banks
    for (int e2 = tid; e2 < 2 * gq * kRtTokens; e2 += kRtThreads) {  // kRtThreads even: pairs stay in a warp
      const int e = e2 >> 1, part = e2 & 1;
      const int h = e / kRtTokens, t = e % kRtTokens;
      float v = 0.f;
      if (t < nt) {
        const float* qr = qs + h * d_h + part * half;
        const float* kr = kh + t * (d_h + 1) + part * half;
        const int q4 = part ? (half / 4) & ~3 : 0;  // a multiple of 4, as half is
        float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
        for (int i = 0; i < half; i += 4) {
          int d = i + q4;
          d = d >= half ? d - half : d;  // d..d+3 stay within the half
          v0 = fmaf(qr[d], kr[d], v0);
          v1 = fmaf(qr[d + 1], kr[d + 1], v1);
          v2 = fmaf(qr[d + 2], kr[d + 2], v2);
          v3 = fmaf(qr[d + 3], kr[d + 3], v3);
        }
        v = (v0 + v1) + (v2 + v3);
      }
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      if (part == 0) sc[h * kRtTokens + t] = t < nt ? v : -INFINITY;
    }
    __syncthreads();
    if (warp < gq) {
      float* row = sc + warp * kRtTokens;
      float mx = -INFINITY;
      for (int t = lane; t < kRtTokens; t += 32) mx = fmaxf(mx, row[t]);
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = ml[warp], m_new = fmaxf(m_old, mx);
      float sum = 0.f;
      for (int t = lane; t < kRtTokens; t += 32) {
        const float p = exp2f(row[t] - m_new);
        row[t] = p;
        sum += p;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      __syncwarp();
      if (lane == 0) {
        const float corr = exp2f(m_old - m_new);
        ml[warp] = m_new;
        ml[kMaxGQ + warp] = ml[kMaxGQ + warp] * corr + sum;
        ml[2 * kMaxGQ + warp] = corr;
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kRtAccSlots; ++k) {
      const int e = tid + k * kRtThreads;
      if (e < n_acc) {
        const int h = e / nkV, c = e % nkV;
        const float* p = sc + h * kRtTokens;
        const float* cc = cV + c;
        float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
        int t = 0;
        for (; t + 4 <= nt; t += 4) {
          v0 = fmaf(p[t], cc[t * cvs], v0);
          v1 = fmaf(p[t + 1], cc[(t + 1) * cvs], v1);
          v2 = fmaf(p[t + 2], cc[(t + 2) * cvs], v2);
          v3 = fmaf(p[t + 3], cc[(t + 3) * cvs], v3);
        }
        for (; t < nt; ++t) v0 = fmaf(p[t], cc[t * cvs], v0);
        acc[k] = fmaf(acc[k], ml[2 * kMaxGQ + h], (v0 + v1) + (v2 + v3));
      }
    }
    __syncthreads();  // the next tile overwrites the latents and probabilities
  }
  // ---- partial record per q head: max, sum, V latent sum ---------------------
  const size_t rec0 = ((size_t)b * cd->n_q + (size_t)a * gq) * A.n_split + split;
#pragma unroll
  for (int k = 0; k < kRtAccSlots; ++k) {
    const int e = tid + k * kRtThreads;
    if (e < n_acc) {
      const int h = e / nkV, c = e % nkV;
      A.part[(rec0 + (size_t)h * A.n_split) * A.part_stride + 2 + c] = acc[k];
    }
  }
  if (tid < gq) {
    A.part[(rec0 + (size_t)tid * A.n_split) * A.part_stride] = ml[tid];
    A.part[(rec0 + (size_t)tid * A.n_split) * A.part_stride + 1] = ml[kMaxGQ + tid];
  }
}

// Merges the splits of one (q head, sequence) and lifts with W_up^V.
__global__ void __launch_bounds__(128) rt_combine_kernel(const CodecDev* __restrict__ cd,
                                                         const float* __restrict__ part, int n_split, int stride,
                                                         float* __restrict__ out) {
  __shared__ float wgt[kRtMaxSplit];
  __shared__ float lat[kRtMaxDHead];
  __shared__ float inv_l;
  const int hq = blockIdx.x, b = blockIdx.y, a = hq / cd->gq, tid = threadIdx.x;
  const SideDev& sv = cd->head[a].side[1];
  const int nkV = sv.n_kept, d_h = cd->d_h;
  const float* rec = part + ((size_t)b * cd->n_q + hq) * n_split * stride;
  if (tid < 32) {
    float M = -INFINITY;
    for (int s = tid; s < n_split; s += 32) M = fmaxf(M, rec[(size_t)s * stride]);
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Lsum = 0.f;
    for (int s = tid; s < n_split; s += 32) {
      const float m = rec[(size_t)s * stride];
      const float w = m == -INFINITY ? 0.f : exp2f(m - M);
      wgt[s] = w;
      Lsum = fmaf(w, rec[(size_t)s * stride + 1], Lsum);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
    if (tid == 0) inv_l = Lsum > 0.f ? 1.f / Lsum : 0.f;
  }
  __syncthreads();
  for (int c = tid; c < nkV; c += blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < n_split; ++s) v = fmaf(wgt[s], rec[(size_t)s * stride + 2 + c], v);
    lat[c] = v * inv_l;
  }
  __syncthreads();
  const float* wv = cd->w_up + sv.wup_off;  // [n_kept][d_h]
  for (int d = tid; d < d_h; d += blockDim.x) {
    float o = 0.f;
    for (int c = 0; c < nkV; ++c) o = fmaf(lat[c], wv[(size_t)c * d_h + d], o);
    out[((size_t)b * cd->n_q + hq) * d_h + d] = o;
  }
}

int rt_sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

// Resident split CTAs per SM at `smem` bytes of dynamic shared memory.
int rt_ctas_per_sm(int group, int smem) {
  const void* kern = group == 16 ? reinterpret_cast<const void*>(rt_split_kernel<16>)
                                 : reinterpret_cast<const void*>(rt_split_kernel<8>);
  int n = 0;
  if (ensure_dynamic_smem(kern, smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kRtThreads, smem) != cudaSuccess || n <= 0)
    n = 1;
  return n;
}

}  // namespace

RtPlan make_rt_plan(const CodecDev& h, int batch, int max_pages_per_seq, bool upper_bound) {
  RtPlan p{};
  const int64_t max_tiles = ((int64_t)max_pages_per_seq * h.P + kRtTokens - 1) / kRtTokens;
  // split the context so that the (KV head, sequence) pairs fill the resident
  // CTA slots once (two CTAs per SM fit at d_h = 128: about 106 KB each; more
  // are not used, so that the bound below holds for any call)
  p.smem_bytes = RtSmem(h.d_h, h.max_kept_k, h.max_kept_v, h.gq, h.group, h.max_sec_bytes / h.P * kRtTokens).total;
  const int pairs = h.n_kv * batch;
  const int per_sm = upper_bound ? 2 : std::min(2, rt_ctas_per_sm(h.group, p.smem_bytes));
  int ns = rt_sm_count() * per_sm / pairs;
  ns = (int)std::max<int64_t>(1, std::min<int64_t>({(int64_t)ns, (int64_t)kRtMaxSplit, max_tiles}));
  p.n_split = ns;
  p.part_stride = (2 + h.max_kept_v + 3) / 4 * 4;
  p.ws_bytes = ((size_t)batch * h.n_q * ns * p.part_stride * 4 + 255) / 256 * 256;
  return p;
}

bool rt_supported(const CodecDev& h, std::string* why) {
  if (h.d_h > kRtMaxDHead || h.d_h % 16 != 0) {
    *why = "reconstruct-then-attend needs d_head a multiple of 16 and at most 128";
    return false;
  }
  if (h.max_kept_k > kRtMaxDHead || h.max_kept_v > kRtMaxDHead) {
    *why = "reconstruct-then-attend needs at most 128 kept coordinates per side";
    return false;
  }
  if (h.gq > kMaxGQ) {
    *why = "reconstruct-then-attend needs at most 8 q heads per KV head";
    return false;
  }
  return true;
}

cudaError_t launch_decode_reconstruct(const CodecDev& h, const CodecDev* d, const spectra_cache& cache,
                                      const float* q, double theta, float* out, void* ws, const RtPlan& plan,
                                      cudaStream_t st) {
  RtArgs A{};
  A.cd = d;
  A.pool = static_cast<const uint8_t*>(cache.pool);
  A.page_table = cache.page_table;
  A.lengths = cache.lengths;
  A.n_pool_pages = cache.n_pages;
  A.max_pages = cache.max_pages_per_seq;
  A.n_split = plan.n_split;
  A.part_stride = plan.part_stride;
  A.theta = theta;
  A.qscale = (float)(1.4426950408889634 / std::sqrt((double)h.d_h));
  A.q = q;
  A.part = static_cast<float*>(ws);
  auto kern = h.group == 16 ? rt_split_kernel<16> : rt_split_kernel<8>;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), plan.smem_bytes);
  if (e != cudaSuccess) return e;
  kern<<<dim3(h.n_kv, cache.batch, plan.n_split), kRtThreads, plan.smem_bytes, st>>>(A);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  rt_combine_kernel<<<dim3(h.n_q, cache.batch), 128, 0, st>>>(d, A.part, plan.n_split, plan.part_stride, out);
  return cudaGetLastError();
}

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
