// Launch arguments, shared-memory layout and limits of the decode attention
// kernel (attend_kernel.cuh), shared by the host planner (decode_kernels.cu)
// and the kernel's instantiation units.
#pragma once

#include <cstdint>

#include "spectra_internal.h"

namespace spectra {
namespace attend {

constexpr int kThreads = 256;     // 8 warps per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kMaxG = 8;          // kept groups per side handled by the decode kernel
constexpr int kMaxKept = 128;     // kept coordinates per side
constexpr int kMaxStages = 32;    // page stages per CTA
constexpr int kMaxSplit = 128;    // context splits per (sequence, KV head)
constexpr uint64_t kWaitLimitNs = 200ull * 1000ull * 1000ull;  // bounded waits
constexpr float kPScaleLog2 = 8.f;   // p = 2^(s - m + 8): fp16 keeps small weights normal
constexpr float kTwo24 = 16777216.f; // undo the 2^-24 of subnormal codes
constexpr float kTwo20 = 1048576.f;  // the same for codes held at nibble bits 4-7 (x16)

// shared-memory carve-up (bytes); the stage ring starts at AttendArgs::off_stages
constexpr int kOffBars = 0;                          // uint64 [kMaxStages + 1] (last: W_up^V slice)
constexpr int kOffIssued = 512;                      // int [kMaxStages]: copies issued per stage
constexpr int kOffConsumed = 640;                    // int [kMaxStages]: pages consumed per stage
constexpr int kOffFlags = 768;                       // int [32]
constexpr int kOffGrp = 896;                         // int4 [2][kMaxG]: {block off, record off, width, col}
// (kOffGrp + 256: int4 [2][kMaxG] the same groups in width-class order {block off,
// record off, group, width}; int [2][8] class bounds)
constexpr int kOffOrd = kOffGrp + 256;
constexpr int kOffCls = kOffOrd + 256;
constexpr int kOffBq = kOffCls + 128;                // uint2 [(kMaxG*2 + 2) * 32] fragments
constexpr int kBqWords = (kMaxG * 2 + 2) * 32;
constexpr int kOffQlat = kOffBq + kBqWords * 8;      // float [kMaxGQ][kMaxKept]
constexpr int kOffX = kOffQlat + kMaxGQ * kMaxKept * 4;  // q (prologue) / merged latent sums (last CTA)
constexpr int kXBytes = kMaxGQ * kMaxDHead * 4;
constexpr int kOffW = kOffX + kXBytes;               // float [kMaxGQ][kWarps + 2]: merge weights, sums
constexpr int kOffFixedEnd = kOffW + kMaxGQ * (kWarps + 2) * 4;  // then the stage ring
constexpr int kCpStride = 2 + kMaxKept;              // floats per q head in a warp's partial

enum { kFlagPre = 0, kFlagStop = 1, kFlagLast = 2 };

struct AttendArgs {
  const CodecDev* cd;
  const uint8_t* pool;
  const int32_t* page_table;
  const int32_t* lengths;
  const float* q;
  float* out;
  float* rec;       // split records [B][n_kv][n_split][gq][rec_stride]: m, l, -, -, latent sums
  int32_t* cnt;     // [B][n_kv] arrival counters, zero between calls
  int64_t n_pool_pages;
  int64_t page_bytes;
  int max_pages;
  int n_split;
  int stages;
  int stage_bytes;
  int off_stages;
  int rec_stride;
  int wv_staged;    // the last CTA bulk-copies the head's W_up^V into its stage ring
  int n_q;
  int n_kv;
  int d_h;
  int hint_lag;     // tokens taken off the length hint (16, plus a test offset; see launch_decode)
  int drop_page;    // test hook: page of CTA (0, 0, 0) whose copy is never issued; -1: none
  unsigned long long wait_ns;  // limit of every bounded wait (kWaitLimitNs unless a test shortens it)
  float q_scale;
  int P;            // tokens per page
  int gq;           // q heads per KV head
  // per KV head (launch parameters, so the prologue needs no global round trip):
  // {section offset, section bytes, kept K groups, kept V groups, kept K
  //  coordinates, kept V coordinates, W_up^K rows offset, W_up^V offset}
  int32_t hm[kMaxKV][8];
};

// The kernel for groups of G coordinates, NT n-tiles of q heads (1: <= 4 q heads
// per KV head, 2: <= 8), CH tiles of 16 tokens per softmax chunk and at most MV
// kept groups on a head's value side (2, 4 or 8); nullptr for other values.
using AttendKernel = void (*)(const AttendArgs);
AttendKernel attend_kernel_ptr(int G, int NT, int CH, int MV);
AttendKernel attend_kernel_ptr_g8(int NT, int CH, int MV);
AttendKernel attend_kernel_ptr_g16(int NT, int CH, int MV);

}  // namespace attend
}  // namespace spectra
