// Internal declarations of libspectra (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <string>
#include <vector>

#include "spectra.h"

namespace spectra {

constexpr int kMaxKV = 32;       // KV heads per layer
constexpr int kMaxGroups = 32;   // rank / group (rank <= 256, group >= 8)
constexpr int kMaxGQ = 8;        // q heads per KV head handled by the decode kernel
constexpr int kMaxDHead = 256;

// Placement of one kept group inside a page (byte offsets from the page start)
// and its first latent column inside its (head, side).
struct GroupDev {
  int32_t b;
  int32_t plane_off;
  int32_t sz_off;
  int32_t col;
};

struct SideDev {
  int32_t n_groups;  // kept groups
  int32_t n_kept;    // kept coordinates = group * n_groups
  int32_t c_col0;    // first column of this (head, side) in the latent matrix [T][n_eff]
  int32_t wup_off;   // offset (floats) of this side's W_up in the codec buffer:
                     // V side rows [n_kept][d_head], K side transposed [d_head][n_kept]
  GroupDev grp[kMaxGroups];
};

// Kept groups of a head side in the order the decode kernel walks them: width
// classes 4, 2, 1, 3, 8; entry {block offset, record offset (both from the head
// section start), group index, width}; class bounds cls[0..5] (the rest pad).
constexpr int kDecMaxGroups = 8;  // kept groups per side the decode kernel handles
struct DecodeOrder {
  int32_t ord[2][kDecMaxGroups][4];
  int32_t cls[2][8];
};

// 16-byte aligned: kernels copy the group and class tables with 16-byte loads.
struct alignas(16) HeadDev {
  SideDev side[2];
  int32_t sec_off;        // byte offset of the head section in a page
  int32_t sec_bytes;      // bytes of the head section (K + V)
  int32_t wupk_rows_off;  // offset (floats) of the K side's W_up rows [n_kept][d_head] (the query fold)
  int32_t pad;
  DecodeOrder dec;        // filled when both sides have <= kDecMaxGroups kept groups
};

// Device-resident description of a codec; kernels read it from global memory.
struct alignas(16) CodecDev {
  int32_t d_model, n_q, n_kv, gq, d_h, group, P, n_eff;
  int32_t n_eff_pad, max_kept_k, max_kept_v, max_sec_bytes;
  int64_t page_bytes;
  int32_t* err;                      // device error word (first error wins)
  const uint16_t* wt_down;           // bf16 bits, [n_eff_pad][d_model] (W_down transposed)
  const float* w_up;                 // kept rows of V_r^T per (head, side), see SideDev::wup_off
  const int32_t* col_groups;         // per group of G latent columns: {b, plane_off, sz_off, side}
  HeadDev head[kMaxKV];
};

static_assert(sizeof(GroupDev) == 16 && offsetof(SideDev, grp) % 16 == 0 && sizeof(SideDev) % 16 == 0,
              "group tables are read with 16-byte loads");
static_assert(offsetof(HeadDev, dec) % 16 == 0 && sizeof(HeadDev) % 16 == 0 && offsetof(CodecDev, head) % 16 == 0,
              "class tables are read with 16-byte loads");

// ---- host math (host_math.cpp), no CUDA needed ------------------------------
int allocate_widths(const double* sigma2, int rank, int group, int budget, bool overhead,
                    int32_t* widths, double* distortion);
int allocate_widths_uniform(const double* sigma2, int rank, int group, int n_eligible, int budget,
                            bool overhead, int32_t* widths, double* distortion);
int energy_rank(const double* sigma2, int n, double threshold, int* r);
int water_fill(const double* sigma2, int n, double rate, double* theta, double* rates);
int sym_eigen(const double* M, int n, double* vals, double* vecs);
// Fills the layout part of `cd` (head sections, group offsets, n_eff ...).
int build_layout(const spectra_config& cfg, const int32_t* widths, CodecDev* cd);
bool valid_config(const spectra_config& cfg, std::string* why);
uint16_t f32_to_bf16_bits(float x);
float bf16_bits_to_f32(uint16_t b);

// ---- error reporting ---------------------------------------------------------
void set_error(const std::string& msg);
spectra_status fail(spectra_status st, const std::string& msg);

}  // namespace spectra
