// Per-token group quantiser and the packed page writer of libspectra, shared by
// the encode kernels (quantise/pack after a separate projection, the fused
// decode-step encode, and the projection GEMM with the quantiser in its
// epilogue), so that every encode route writes the same bits.
//
// Quantiser ("SPECTRA pipeline" stage 2: groups of adjacent latent coordinates
// share one width; stage 3: tokens are quantised per token): per token and
// group of G fp32 latents at width b, every step one IEEE fp32 operation,
//   s = fp16(sat((max - min) / (2^b - 1))), z = fp16(sat(min)),
//   code = clamp(rint((x - z) / s), 0, 2^b - 1), all codes 0 when s == 0.
// Page writer: code bits at the canonical (word, bit) addresses of the page
// layout (fragment position of the entry, then the width rule), scale/zero
// records per token pair.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

namespace spectra {
namespace pack {

__device__ __forceinline__ float sat16(float x) { return fminf(fmaxf(x, -65504.f), 65504.f); }

// Scale and zero of a group with extremes mn, mx at width b:
// s = fp16(sat((mx - mn) / (2^b - 1))), z = fp16(sat(mn)).
__device__ __forceinline__ void scale_zero(float mn, float mx, int b, __half& s_h, __half& z_h) {
  const float levels = (float)((1 << b) - 1);
  s_h = __float2half_rn(sat16(__fdiv_rn(__fsub_rn(mx, mn), levels)));
  z_h = __float2half_rn(sat16(mn));
}

// code = clamp(rint((x - z) / s), 0, 2^b - 1), 0 when s == 0.
__device__ __forceinline__ uint32_t code_of(float x, int b, __half s_h, __half z_h) {
  const float sf = __half2float(s_h), zf = __half2float(z_h);
  if (!(sf > 0.f)) return 0u;
  const float t = __fdiv_rn(__fsub_rn(x, zf), sf);
  return (uint32_t)fminf(fmaxf(rintf(t), 0.f), (float)((1 << b) - 1));
}

// One token's group of G fp32 latents at width b (every step one IEEE fp32
// operation): s = fp16(sat((max - min) / (2^b - 1))), z = fp16(sat(min)),
// code = clamp(rint((x - z) / s), 0, 2^b - 1), all codes 0 when s == 0.
template <int G>
__device__ __forceinline__ void quantize_group(const float (&x)[G], int b, __half& s_h, __half& z_h,
                                               uint32_t (&code)[G]) {
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int k = 1; k < G; ++k) {
    mn = fminf(mn, x[k]);
    mx = fmaxf(mx, x[k]);
  }
  scale_zero(mn, mx, b, s_h, z_h);
#pragma unroll
  for (int k = 0; k < G; ++k) code[k] = code_of(x[k], b, s_h, z_h);
}

// The same quantiser with the group spread over the 16 lanes of a half warp:
// lane k of the half holds latent k (lanes k >= G repeat latent 0, which leaves
// the extremes unchanged) and gets code k; s and z are the same in every lane.
__device__ __forceinline__ uint32_t quantize_half_warp(float x, int b, __half& s_h, __half& z_h) {
  const unsigned half = 0xFFFFu << (threadIdx.x & 16);
  float mn = x, mx = x;
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(half, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(half, mx, o));
  }
  scale_zero(mn, mx, b, s_h, z_h);
  return code_of(x, b, s_h, z_h);
}

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

// Block word(s) and bits of one code of width b at fragment position (gid, t4,
// slot), the page layout's width rule:
//   b = 4: word 4 gid + t4, nibble `slot`;
//   b = 2: word 2 gid + t4/2, bits 4 slot + 2 (t4 % 2) + {0, 1};
//   b = 1: word gid, bit 4 slot + t4;
//   b = 3: bits 0-1 as b = 2, bit 2 as b = 1 in word 16 + gid (the second word);
//   b = 8: word 2 (4 gid + t4) + (slot / 2) % 2, byte (slot % 2) + 2 (slot / 4).
// w1 < 0 when the code has no second word.
struct CodeBits {
  int w0, w1;
  uint32_t m0, v0, m1, v1;
};

__device__ __forceinline__ CodeBits code_bits(int b, int gid, int t4, int slot, uint32_t code) {
  CodeBits r{-1, -1, 0u, 0u, 0u, 0u};
  int sh;
  uint32_t wm;
  switch (b) {
    case 4: r.w0 = 4 * gid + t4; sh = 4 * slot; wm = 0xFu; break;
    case 2: r.w0 = 2 * gid + (t4 >> 1); sh = 4 * slot + 2 * (t4 & 1); wm = 0x3u; break;
    case 1: r.w0 = gid; sh = 4 * slot + t4; wm = 0x1u; break;
    case 3:
      r.w0 = 2 * gid + (t4 >> 1);
      sh = 4 * slot + 2 * (t4 & 1);
      wm = 0x3u;
      r.w1 = 16 + gid;
      r.m1 = 1u << (4 * slot + t4);
      r.v1 = ((code >> 2) & 1u) << (4 * slot + t4);
      break;
    default: r.w0 = 2 * (4 * gid + t4) + ((slot >> 1) & 1); sh = 8 * ((slot & 1) + 2 * (slot >> 2)); wm = 0xFFu; break;
  }
  r.m0 = wm << sh;
  r.v0 = (code & wm) << sh;
  return r;
}

// Pending bits of one block word: consecutive entries that land in the same word
// are merged.  Global words (kShared = false) are written with one atomicAnd /
// atomicOr pair (other tokens of the block may be written concurrently or may
// hold stale bits); a zeroed shared-memory copy of the block only needs the OR.
struct WordBits {
  int w;
  uint32_t mask, val;
};

template <bool kShared>
__device__ __forceinline__ void flush_word(uint32_t* blk, WordBits& a) {
  if (a.w >= 0) {
    if (!kShared) atomicAnd(blk + a.w, ~a.mask);
    atomicOr(blk + a.w, a.val);
  }
  a.w = -1;
  a.mask = a.val = 0u;
}

template <bool kShared>
__device__ __forceinline__ void put_bits(uint32_t* blk, WordBits& a, int w, uint32_t mask, uint32_t val) {
  if (w != a.w) {
    flush_word<kShared>(blk, a);
    a.w = w;
  }
  a.mask |= mask;
  a.val |= val;
}

// Writes one code (width b) of fragment position (gid, t4, slot) into a block.
template <bool kShared>
__device__ __forceinline__ void put_code(uint32_t* blk, WordBits& a, WordBits& a1, int b, int gid, int t4,
                                         int slot, uint32_t code) {
  const CodeBits c = code_bits(b, gid, t4, slot, code);
  put_bits<kShared>(blk, a, c.w0, c.m0, c.v0);
  if (c.w1 >= 0) put_bits<kShared>(blk, a1, c.w1, c.m1, c.v1);
}

// Scale/zero of page token tau: record of its pair u = tau/2 at index
// (u % 8) * (P/16) + u / 8, fp16 {s[2u], s[2u+1], z[2u], z[2u+1]}.
__device__ __forceinline__ void put_record(uint8_t* recs, int P, int tau, __half s_h, __half z_h) {
  const int u = tau >> 1;
  __half* rec = reinterpret_cast<__half*>(recs + 8 * ((u & 7) * (P >> 4) + (u >> 3)));
  rec[tau & 1] = s_h;
  rec[2 + (tau & 1)] = z_h;
}

template <int G, bool kShared>
__device__ __forceinline__ void put_codes(uint32_t* blk, int side, int tb, int b, const uint32_t (&code)[G]) {
  WordBits acc{-1, 0u, 0u}, acc1{-1, 0u, 0u};
#pragma unroll
  for (int k = 0; k < G; ++k) {
    int gid, t4, slot;
    if (side == 0) k_side_pos<G>(tb, k, &gid, &t4, &slot);
    else v_side_pos<G>(tb, k, &gid, &t4, &slot);
    put_code<kShared>(blk, acc, acc1, b, gid, t4, slot, code[k]);
  }
  flush_word<kShared>(blk, acc);
  flush_word<kShared>(blk, acc1);
}


}  // namespace pack
}  // namespace spectra

namespace spectra {
namespace pack {

// ---------------------------------------------------------------------------
// Whole-block writer.  The TB = 256/G lanes of a lane set hold the TB tokens of
// one code block (token tb of the block per lane).  Each lane scatters its G
// codes into a 256-byte shared buffer in fragment order, byte 32 gid + 8 t4 +
// slot; then the block's 8b words are assembled from consecutive bytes of
// that buffer, four words per lane (lanes sub < 2b), and stored with one 16-byte
// store each.  Word and bit of each entry as in the page layout's width rule.
// ---------------------------------------------------------------------------
template <int G>
__device__ __forceinline__ void frag_bytes(uint8_t* fb, int side, int tb, const uint32_t (&code)[G]) {
  if constexpr (G == 16) {
    if (side == 0) {  // K: row = tb/2 (tb even) or 8 + tb/2, col = k
      const int row = (tb & 1) ? 8 + (tb >> 1) : (tb >> 1);
      uint8_t* p = fb + (row & 7) * 32 + (row >> 3);
#pragma unroll
      for (int k = 0; k < 16; ++k) p[((k & 7) >> 1) * 8 + 2 * (k >> 3) + 4 * (k & 1)] = (uint8_t)code[k];
    } else {  // V: row = k, col = tb
      uint8_t* p = fb + ((tb & 7) >> 1) * 8 + 2 * (tb >> 3) + 4 * (tb & 1);
#pragma unroll
      for (int k = 0; k < 16; ++k) p[(k & 7) * 32 + (k >> 3)] = (uint8_t)code[k];
    }
  } else {
    const int mi = tb >> 4, tl = tb & 15;
    if (side == 0) {
      const int row = (tl & 1) ? 8 + (tl >> 1) : (tl >> 1);
      uint8_t* p = fb + (row & 7) * 32 + (row >> 3) + 2 * mi;
#pragma unroll
      for (int k = 0; k < 8; ++k) p[(k >> 1) * 8 + 4 * (k & 1)] = (uint8_t)code[k];
    } else {
      uint8_t* p = fb + ((tl & 7) >> 1) * 8 + mi + 2 * (tl >> 3) + 4 * (tl & 1);
#pragma unroll
      for (int k = 0; k < 8; ++k) p[k * 32] = (uint8_t)code[k];
    }
  }
}

// four bytes (each < 16) -> their nibbles in bits 0-15
__device__ __forceinline__ uint32_t nib4(uint32_t x) {
  x = (x | (x >> 4)) & 0x00FF00FFu;
  return (x | (x >> 8)) & 0x0000FFFFu;
}

// Words [4i, 4i + 4) of a block of width b from the fragment-ordered bytes
// (f[2e], f[2e + 1]: slots 0-3 and 4-7 of entry e = 4 gid + t4).
__device__ __forceinline__ uint4 block_words(const uint8_t* fb, int b, int i) {
  const uint32_t* f = reinterpret_cast<const uint32_t*>(fb);
  uint32_t w[4];
  if (b == 4) {  // word e: nibble slot = code(e, slot)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = 4 * i + j;
      w[j] = nib4(f[2 * e]) | (nib4(f[2 * e + 1]) << 16);
    }
  } else if (b == 8) {  // word 2e + h: bytes of slots {0,1,4,5} (h = 0) or {2,3,6,7}
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int e = 2 * i + j;
      w[2 * j] = __byte_perm(f[2 * e], f[2 * e + 1], 0x5410);
      w[2 * j + 1] = __byte_perm(f[2 * e], f[2 * e + 1], 0x7632);
    }
  } else if (b == 2 || (b == 3 && i < 4)) {  // word d: entries 2d, 2d + 1 in bits 0-1, 2-3 of a nibble
    const uint32_t m = b == 3 ? 0x03030303u : 0xFFFFFFFFu;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = 2 * (4 * i + j);
      w[j] = nib4((f[2 * e] & m) | ((f[2 * e + 2] & m) << 2)) |
             (nib4((f[2 * e + 1] & m) | ((f[2 * e + 3] & m) << 2)) << 16);
    }
  } else {  // b = 1 (word gid), or bit 2 of b = 3 (word 16 + gid): bit 4 slot + t4
    const int g0 = b == 3 ? 4 * (i - 4) : 4 * i;
    const int sh = b == 3 ? 2 : 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = 4 * (g0 + j);
      uint32_t lo = 0u, hi = 0u;
#pragma unroll
      for (int t4 = 0; t4 < 4; ++t4) {
        lo |= ((f[2 * (e + t4)] >> sh) & 0x01010101u) << t4;
        hi |= ((f[2 * (e + t4) + 1] >> sh) & 0x01010101u) << t4;
      }
      w[j] = nib4(lo) | (nib4(hi) << 16);
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace pack
}  // namespace spectra
