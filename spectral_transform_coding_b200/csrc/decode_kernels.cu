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
// One kernel per decode step (attend_kernel, attend_kernel.cuh); this file holds
// its host side: the launch plan and the launch.  The grid is (context split,
// KV head, sequence), one CTA per split:
//   prologue (before the dependency wait; reads only the caller's q, read-only
//     codec data, the lengths as a hint and pages that are full 16 tokens below
//     the hint):
//     bulk copies of the first pages into a CTA-wide ring of shared-memory
//     stages; the fold q_lat = q W_up^K^T of all kept K coordinates; the MMA B
//     fragments of q_lat;
//   main loop (after the wait): 8 warps take the CTA's pages in turn and stream
//     them through an online softmax, one page (64 tokens) per step;
//   merges: the warps of a CTA into one record per q head in the workspace;
//     the last CTA of a (sequence, KV head) to arrive (a self-resetting counter
//     in the workspace) merges the splits' records in split order and lifts the
//     value latents with W_up^V.
// The split partition (page i of a sequence goes to split i mod n_split) and the
// merge order depend only on the final length, so results are deterministic.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "attend_args.h"
#include "kernels.h"

namespace spectra {

namespace {

using attend::AttendArgs;
using attend::AttendKernel;
using attend::kThreads;
using attend::kWarps;
using attend::kMaxStages;
using attend::kMaxKept;
using attend::kMaxSplit;
using attend::kOffFixedEnd;
using attend::kCpStride;

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

// Tiles (16 tokens) per softmax chunk: 4 when a page holds a multiple of 64
// tokens, else 2 (pages hold a multiple of 32).
// 16-token tiles per softmax chunk: 8 (pages of 128 tokens or more, one n-tile
// of q heads), else 4 or 2 as the page allows.  Longer chunks amortise the
// per-chunk work (softmax, z terms, group set-up) over more tokens.
int chunk_tiles(int P, int NT) {
  if (NT == 1 && (P / 16) % 8 == 0) return 8;
  return (P / 16) % 4 == 0 ? 4 : 2;
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

namespace {

using AttendKernel = void (*)(const AttendArgs);

// Kept groups on the value side of the head with the most, rounded up to the
// kernel's register bound (2, 4 or 8 accumulators).
int value_group_bound(const CodecDev& h) {
  int n = 0;
  for (int a = 0; a < h.n_kv; ++a) n = std::max(n, h.head[a].side[1].n_groups);
  return n <= 2 ? 2 : (n <= 4 ? 4 : 8);
}

AttendKernel attend_kernel_for(const CodecDev& h) {
  const int NT = h.gq > 4 ? 2 : 1;
  return attend::attend_kernel_ptr(h.group, NT, chunk_tiles(h.P, NT), value_group_bound(h));
}

// CTAs with `smem` bytes of dynamic shared memory that one SM holds.
int ctas_per_sm(AttendKernel kern, int smem) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int>, int> memo;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_tuple(reinterpret_cast<const void*>(kern), smem, dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = memo.find(key);
    if (it != memo.end()) return it->second;
  }
  int n = 0;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, smem) != cudaSuccess)
    n = 0;
  (void)cudaGetLastError();
  if (n <= 0) n = 2;  // no device answer: what the shared-memory budget is sized for
  std::lock_guard<std::mutex> lock(mu);
  memo[key] = n;
  return n;
}

}  // namespace

// Plan of one decode step (memoised per shape, batch and device).
// Shared memory: fixed tables and a ring of page stages, ~112 KB per CTA so
// that two CTAs fit an SM; the last CTA of a (sequence, KV head) reuses its
// ring for W_up^V when the head's rows fit.
// Splits per (sequence, KV head): few units (batch-1 decode) mean little
// streaming work per CTA, so a launch takes one CTA slot per SM and the other
// slot lets the next launch's CTAs become resident, fold and prefetch while
// this one runs; many units fill both slots.  The count minimises an estimated
// step time, a nominal 16 us of streaming over the slots one wave fills plus
// 2 us of fixed work (fold, merges) per wave; it does not depend on the
// context length, so a workspace sized once fits every call.
DecodePlan make_decode_plan(const CodecDev& h, int batch, int max_pages_per_seq) {
  (void)max_pages_per_seq;
  static std::mutex mu;
  static std::map<std::vector<int64_t>, DecodePlan> memo;
  int dev = 0;
  cudaGetDevice(&dev);
  const std::vector<int64_t> key = {h.n_kv, h.gq, h.d_h, h.group, h.P, h.max_sec_bytes, h.max_kept_k,
                                    h.max_kept_v, value_group_bound(h), batch, dev};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = memo.find(key);
    if (it != memo.end()) return it->second;
  }
  DecodePlan p{};
  p.cl = 1;
  p.stage_bytes = std::max(16, ((h.max_sec_bytes + 15) / 16) * 16);
  p.off_stages = ((kOffFixedEnd + 127) / 128) * 128;
  const int budget = 112 * 1024 - p.off_stages;
  p.stages = std::max(1, std::min(kMaxStages, budget / p.stage_bytes));
  const int merge_bytes = kWarps * kMaxGQ * kCpStride * 4;
  const int wv_bytes = h.max_kept_v * h.d_h * 4;
  int ring = std::max(p.stages * p.stage_bytes, merge_bytes);
  p.wv_staged = wv_bytes <= std::max(ring, budget) ? 1 : 0;
  if (p.wv_staged) ring = std::max(ring, wv_bytes);
  p.smem_bytes = p.off_stages + ring;
  p.rec_stride = 4 + kMaxKept;  // {m, l, -, -} then the latent sums (16-byte aligned rows)
  p.slice_k = h.max_kept_k;
  p.slice_v = h.max_kept_v;
  const AttendKernel kern = attend_kernel_for(h);
  const int units = std::max(1, batch * h.n_kv);
  const bool one_per_sm = units * 2 < sm_count();
  const int slots = (one_per_sm ? 1 : std::max(1, ctas_per_sm(kern, p.smem_bytes))) * sm_count();
  int best_ns = 1;
  double best_t = 1e30;
  for (int ns = 1; ns <= kMaxSplit; ++ns) {
    const long ctas = (long)units * ns;
    const long waves = (ctas + slots - 1) / slots;
    const double eff = (double)ctas / (double)(waves * slots);
    const double t = 16.0 / eff + 2.0 * waves;
    if (t < best_t - 1e-9) {
      best_t = t;
      best_ns = ns;
    }
  }
  p.n_split = best_ns;
  size_t off = 0;
  auto carve = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  };
  p.cnt_off = carve((size_t)batch * h.n_kv * 4);
  p.rec_off = carve((size_t)batch * h.n_kv * p.n_split * h.gq * p.rec_stride * 4);
  p.ws_bytes = off;
  std::lock_guard<std::mutex> lock(mu);
  memo[key] = p;
  return p;
}

cudaError_t launch_decode(const CodecDev& h, const CodecDev* d, const spectra_cache& cache, const float* q,
                          float* out, void* ws, const DecodePlan& plan, cudaStream_t st) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  AttendArgs args;
  args.cd = d;
  args.pool = static_cast<const uint8_t*>(cache.pool);
  args.page_table = cache.page_table;
  args.lengths = cache.lengths;
  args.q = q;
  args.out = out;
  args.rec = reinterpret_cast<float*>(w + plan.rec_off);
  args.cnt = reinterpret_cast<int32_t*>(w + plan.cnt_off);
  args.n_pool_pages = cache.n_pages;
  args.page_bytes = h.page_bytes;
  args.max_pages = cache.max_pages_per_seq;
  args.n_split = plan.n_split;
  args.stages = plan.stages;
  args.stage_bytes = plan.stage_bytes;
  args.off_stages = plan.off_stages;
  args.rec_stride = plan.rec_stride;
  args.wv_staged = plan.wv_staged;
  args.n_q = h.n_q;
  args.n_kv = h.n_kv;
  args.d_h = h.d_h;
  args.q_scale = 1.4426950408889634f / sqrtf((float)h.d_h);
  args.P = h.P;
  args.gq = h.gq;
  for (int a = 0; a < kMaxKV; ++a) {
    int32_t* m = args.hm[a];
    if (a < h.n_kv) {
      const HeadDev& hd = h.head[a];
      m[0] = hd.sec_off;
      m[1] = hd.sec_bytes;
      m[2] = hd.side[0].n_groups;
      m[3] = hd.side[1].n_groups;
      m[4] = hd.side[0].n_kept;
      m[5] = hd.side[1].n_kept;
      m[6] = hd.wupk_rows_off;
      m[7] = hd.side[1].wup_off;
    } else {
      for (int k = 0; k < 8; ++k) m[k] = 0;
    }
  }
  {
    // test hook: SPECTRA_DECODE_HINT_LAG offsets the kernel's length hint (a
    // positive lag sends the copies of more pages after the dependency wait, a
    // negative one makes the kernel copy pages beyond the length, which it must
    // then drain); the result may not change
    // The built-in lag: a fused decode-step encode that is still running may
    // have advanced the lengths by up to kFusedMaxT tokens per sequence before
    // its page writes land (only one such encode at a time: it writes the
    // lengths after its own wait, when every earlier kernel has completed).
    const char* e = std::getenv("SPECTRA_DECODE_HINT_LAG");
    args.hint_lag = kFusedMaxT + (e ? std::atoi(e) : 0);
    // test hooks for the bounded waits: SPECTRA_DECODE_TEST_DROP_PAGE makes the
    // first CTA skip the copy of that page of its list (its wait for the page
    // then gives up and the call reports SPECTRA_ERR_TIMEOUT), and
    // SPECTRA_DECODE_TEST_WAIT_NS shortens every wait's limit
    const char* d = std::getenv("SPECTRA_DECODE_TEST_DROP_PAGE");
    args.drop_page = d ? std::atoi(d) : -1;
    const char* w = std::getenv("SPECTRA_DECODE_TEST_WAIT_NS");
    const long long wn = w ? std::atoll(w) : 0;
    args.wait_ns = wn > 0 ? (unsigned long long)wn : attend::kWaitLimitNs;
  }
  const auto kern = attend_kernel_for(h);
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), plan.smem_bytes);
  if (e != cudaSuccess) return e;
  static bool pdl_ok = true;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.n_split, h.n_kv, cache.batch);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = plan.smem_bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_ok ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, args);
  if (e != cudaSuccess && pdl_ok) {
    // without programmatic serialisation: plain stream order
    (void)cudaGetLastError();
    pdl_ok = false;
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, kern, args);
  }
  return e;
}

namespace attend {
AttendKernel attend_kernel_ptr(int G, int NT, int CH, int MV) {
  return G == 16 ? attend_kernel_ptr_g16(NT, CH, MV) : (G == 8 ? attend_kernel_ptr_g8(NT, CH, MV) : nullptr);
}
}  // namespace attend

}  // namespace spectra
