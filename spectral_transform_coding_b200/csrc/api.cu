// C ABI entry points of libspectra.  Argument checks, codec ownership, the
// calibration driver (GPU Gram and W^T G W, host fp64 eigen-decomposition and
// bit allocation) and the hot-path launch sequences.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <memory>
#include <mutex>
#include <string>
#include <vector>

#include "kernels.h"
#include "spectra_internal.h"

using namespace spectra;

struct spectra_codec {
  spectra_config cfg{};
  int n_groups = 0;
  int device = 0;
  bool decode_ok = false;
  std::string decode_why;
  std::vector<int32_t> widths;    // [n_kv][2][n_groups]
  std::vector<double> sigma2;     // [n_kv][2][rank]
  std::vector<double> theta;      // [n_kv][2]
  std::vector<uint16_t> wdown;    // bf16 bits, [d_model][n_eff]
  std::vector<float> wup;         // [n_kv][2][rank][d_head]
  CodecDev h{};                   // host mirror of the device description
  CodecDev* d = nullptr;          // device copy
  void* dmem = nullptr;           // device allocation holding d, err, factors
  int32_t* err = nullptr;
  ~spectra_codec() {
    if (dmem) cudaFree(dmem);
  }
};

namespace {

#define CUDA_TRY(expr)                                                                        \
  do {                                                                                        \
    cudaError_t e_ = (expr);                                                                  \
    if (e_ != cudaSuccess)                                                                    \
      return fail(SPECTRA_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(e_));     \
  } while (0)

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

spectra_status check_device(const spectra_codec* c) {
  int dev = -1;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev != c->device) return fail(SPECTRA_ERR_INVALID, "codec belongs to another CUDA device");
  return SPECTRA_OK;
}

// Owns a temporary device allocation for the duration of a host call.
struct DevBuf {
  void* p = nullptr;
  ~DevBuf() {
    if (p) cudaFree(p);
  }
};

spectra_status build_codec(const spectra_config& cfg, const int32_t* widths, const float* W_down,
                           const float* W_up, const double* sigma2, const double* theta,
                           const uint16_t* W_down_bits, spectra_codec** out) {
  std::string why;
  if (!valid_config(cfg, &why)) return fail(SPECTRA_ERR_INVALID, why);
  std::unique_ptr<spectra_codec> c(new spectra_codec());
  c->cfg = cfg;
  c->n_groups = cfg.rank / cfg.group;
  const size_t nw = (size_t)cfg.n_kv_heads * 2 * c->n_groups;
  c->widths.assign(widths, widths + nw);
  const int rc = build_layout(cfg, widths, &c->h);
  if (rc == 1) return fail(SPECTRA_ERR_INVALID, "width must be one of 0,1,2,3,4,8");
  if (rc) return fail(SPECTRA_ERR_UNSUPPORTED, "page too large");
  const size_t ns = (size_t)cfg.n_kv_heads * 2 * cfg.rank;
  c->sigma2.assign(ns, 0.0);
  if (sigma2) std::copy(sigma2, sigma2 + ns, c->sigma2.begin());
  c->theta.assign((size_t)cfg.n_kv_heads * 2, 0.0);
  if (theta) std::copy(theta, theta + c->theta.size(), c->theta.begin());
  const int n_eff = c->h.n_eff, dm = cfg.d_model, dh = cfg.d_head;
  c->wdown.assign((size_t)dm * n_eff, 0);
  for (size_t i = 0; i < c->wdown.size(); ++i)
    c->wdown[i] = W_down_bits ? W_down_bits[i] : f32_to_bf16_bits(W_down[i]);
  c->wup.assign(W_up, W_up + ns * dh);
  for (float v : c->wup)
    if (!std::isfinite(v)) return fail(SPECTRA_ERR_NUMERIC, "W_up has non-finite entries");

  // decode kernel limits
  c->decode_ok = true;
  for (int a = 0; a < cfg.n_kv_heads; ++a)
    for (int s = 0; s < 2; ++s)
      if (c->h.head[a].side[s].n_groups > 8) {
        c->decode_ok = false;
        c->decode_why = "decode supports at most 8 kept groups per head and side";
      }
  if (cfg.d_head % 16 != 0 || cfg.d_head > 256) {
    c->decode_ok = false;
    c->decode_why = "decode needs d_head a multiple of 16 and at most 256";
  }
  if (c->h.max_sec_bytes > 27 * 1024) {
    c->decode_ok = false;
    c->decode_why = "head section of a page exceeds 27 KB; use fewer page_tokens";
  }

  // device image: [CodecDev][err][wt_down][w_up]
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  c->device = dev;
  const size_t off_err = (sizeof(CodecDev) + 255) / 256 * 256;
  const size_t off_wt = off_err + 256;
  const size_t wt_bytes = (size_t)c->h.n_eff_pad * dm * 2;
  const size_t off_wu = off_wt + (wt_bytes + 255) / 256 * 256;
  size_t kept_total = 0;  // floats of W_up: per-side blocks, then the K sides again as rows
  for (int a = 0; a < cfg.n_kv_heads; ++a)
    kept_total += 2 * (size_t)c->h.head[a].side[0].n_kept + c->h.head[a].side[1].n_kept;
  const size_t wu_bytes = std::max<size_t>(kept_total * dh * 4, 4);
  const size_t off_cg = off_wu + (wu_bytes + 255) / 256 * 256;
  const size_t n_cg = std::max<size_t>((size_t)n_eff / cfg.group, 1);
  const size_t total = off_cg + n_cg * 16;
  CUDA_TRY(cudaMalloc(&c->dmem, total));
  uint8_t* base = static_cast<uint8_t*>(c->dmem);
  c->err = reinterpret_cast<int32_t*>(base + off_err);
  c->h.err = c->err;
  c->h.wt_down = reinterpret_cast<const uint16_t*>(base + off_wt);
  c->h.w_up = reinterpret_cast<const float*>(base + off_wu);
  c->h.col_groups = reinterpret_cast<const int32_t*>(base + off_cg);
  c->d = reinterpret_cast<CodecDev*>(base);

  std::vector<uint16_t> wt((size_t)c->h.n_eff_pad * dm, 0);
  for (int k = 0; k < dm; ++k)
    for (int n = 0; n < n_eff; ++n) wt[(size_t)n * dm + k] = c->wdown[(size_t)k * n_eff + n];
  std::vector<float> wu(kept_total * dh, 0.f);
  for (int a = 0; a < cfg.n_kv_heads; ++a)
    for (int s = 0; s < 2; ++s) {
      const SideDev& sd = c->h.head[a].side[s];
      // V side row-major [n_kept][d_h]; K side transposed [d_h][n_kept] (the query
      // fold reads it column-wise)
      int row = 0;
      for (int j = 0; j < c->n_groups; ++j) {
        if (widths[((size_t)a * 2 + s) * c->n_groups + j] == 0) continue;
        for (int k = 0; k < cfg.group; ++k, ++row) {
          const int src = j * cfg.group + k;
          const float* from = W_up + (((size_t)a * 2 + s) * cfg.rank + src) * dh;
          for (int d = 0; d < dh; ++d) {
            const size_t at = s == 0 ? (size_t)d * sd.n_kept + row : (size_t)row * dh + d;
            wu[sd.wup_off + at] = from[d];
            if (s == 0) wu[c->h.head[a].wupk_rows_off + (size_t)row * dh + d] = from[d];
          }
        }
      }
    }
  // groups of G latent columns (head-major, K then V, kept groups ascending):
  // {width, code block offset, scale/zero offset, side} for the GEMM epilogue
  std::vector<int32_t> cg(n_cg * 4, 0);
  for (int a = 0; a < cfg.n_kv_heads; ++a)
    for (int s = 0; s < 2; ++s) {
      const SideDev& sd = c->h.head[a].side[s];
      for (int j = 0; j < sd.n_groups; ++j) {
        const size_t g = (size_t)(sd.c_col0 + sd.grp[j].col) / cfg.group;
        cg[4 * g] = sd.grp[j].b;
        cg[4 * g + 1] = sd.grp[j].plane_off;
        cg[4 * g + 2] = sd.grp[j].sz_off;
        cg[4 * g + 3] = s;
      }
    }
  CUDA_TRY(cudaMemset(c->dmem, 0, off_wt));
  CUDA_TRY(cudaMemcpy(base, &c->h, sizeof(CodecDev), cudaMemcpyHostToDevice));
  CUDA_TRY(cudaMemcpy(base + off_wt, wt.data(), wt.size() * 2, cudaMemcpyHostToDevice));
  CUDA_TRY(cudaMemcpy(base + off_wu, wu.data(), wu.size() * 4, cudaMemcpyHostToDevice));
  CUDA_TRY(cudaMemcpy(base + off_cg, cg.data(), cg.size() * 4, cudaMemcpyHostToDevice));
  *out = c.release();
  return SPECTRA_OK;
}

// Encode workspace: [counters of the fused decode-step path][positions][flag]
// [latents, or the fused path's partial sums].
constexpr size_t kEncCounterBytes = ((1 + kMaxFusedGroups) * 4 + 255) / 256 * 256;
constexpr int64_t kGemmMinT = 64;  // rows from which the projection runs on the tcgen05 GEMM
size_t encode_ws_bytes(const spectra_codec* c, int64_t T) {
  const size_t pos = ((size_t)std::max<int64_t>(T, 1) * 4 + 255) / 256 * 256;
  const size_t flag = 256;
  size_t lat = (size_t)std::max<int64_t>(T, 1) * c->h.n_eff * 4;
  lat = std::max(lat, encode_fused_partial_bytes(c->h, (int)std::min<int64_t>(std::max<int64_t>(T, 1), kFusedMaxT)));
  lat = (lat + 255) / 256 * 256;
  return kEncCounterBytes + pos + flag + lat;
}

spectra_status check_cache(const spectra_codec* c, const spectra_cache* cache) {
  if (!cache || !cache->pool || !cache->page_table || !cache->lengths)
    return fail(SPECTRA_ERR_INVALID, "cache has a null pointer");
  if (cache->batch <= 0 || cache->max_pages_per_seq <= 0 || cache->n_pages <= 0)
    return fail(SPECTRA_ERR_INVALID, "cache sizes must be positive");
  if (!aligned(cache->pool, 16)) return fail(SPECTRA_ERR_INVALID, "cache pool must be 16-byte aligned");
  (void)c;
  return SPECTRA_OK;
}

spectra_status do_project(const spectra_codec* c, const void* H, int64_t T, float* C, cudaStream_t st) {
  // T >= 64 rows: tcgen05 tensor-core GEMM; fewer rows: the projection is a
  // weight-streaming GEMV bounded by HBM, done on CUDA cores.
  if (T >= kGemmMinT) {
    CUDA_TRY(launch_project_tcgen05(c->h, c->h.wt_down, static_cast<const uint16_t*>(H), (int)T, C,
                                    c->h.n_eff, st));
  } else {
    CUDA_TRY(launch_project_gemv(c->h, c->h.wt_down, static_cast<const uint16_t*>(H), (int)T, C,
                                 c->h.n_eff, st));
  }
  return SPECTRA_OK;
}

spectra_status do_quantize_append(const spectra_codec* c, const spectra_cache* cache, const float* C,
                                  const int32_t* seq_ids, int64_t T, void* ws, cudaStream_t st) {
  uint8_t* w = static_cast<uint8_t*>(ws) + kEncCounterBytes;
  int32_t* pos = reinterpret_cast<int32_t*>(w);
  int32_t* flag = reinterpret_cast<int32_t*>(w + ((size_t)T * 4 + 255) / 256 * 256);
  CUDA_TRY(launch_append_plan(seq_ids, (int)T, *cache, c->cfg.page_tokens, pos, flag, c->err, st));
  CUDA_TRY(launch_quantize_append(c->h, c->d, C, c->h.n_eff, seq_ids, pos, flag, (int)T, *cache, st));
  return SPECTRA_OK;
}

// Gaussian elimination with partial pivoting: X = A^-1 B, A n x n, B n x m (fp64).
bool solve_dense(std::vector<double> A, std::vector<double>& B, int n, int m) {
  for (int k = 0; k < n; ++k) {
    int piv = k;
    for (int i = k + 1; i < n; ++i)
      if (std::fabs(A[(size_t)i * n + k]) > std::fabs(A[(size_t)piv * n + k])) piv = i;
    if (A[(size_t)piv * n + k] == 0.0) return false;
    if (piv != k) {
      for (int j = 0; j < n; ++j) std::swap(A[(size_t)k * n + j], A[(size_t)piv * n + j]);
      for (int j = 0; j < m; ++j) std::swap(B[(size_t)k * m + j], B[(size_t)piv * m + j]);
    }
    const double d = A[(size_t)k * n + k];
    for (int i = k + 1; i < n; ++i) {
      const double f = A[(size_t)i * n + k] / d;
      if (f == 0.0) continue;
      for (int j = k; j < n; ++j) A[(size_t)i * n + j] -= f * A[(size_t)k * n + j];
      for (int j = 0; j < m; ++j) B[(size_t)i * m + j] -= f * B[(size_t)k * m + j];
    }
  }
  for (int k = n - 1; k >= 0; --k) {
    for (int j = 0; j < m; ++j) {
      double v = B[(size_t)k * m + j];
      for (int i = k + 1; i < n; ++i) v -= A[(size_t)k * n + i] * B[(size_t)i * m + j];
      B[(size_t)k * m + j] = v / A[(size_t)k * n + k];
    }
  }
  return true;
}

}  // namespace

extern "C" {

spectra_status spectra_codec_create(const spectra_config* cfg, const int32_t* widths,
                                    const float* W_down, const float* W_up, const double* sigma2,
                                    spectra_codec** out) {
  if (!cfg || !widths || !W_down || !W_up || !out) return fail(SPECTRA_ERR_INVALID, "null pointer");
  *out = nullptr;
  return build_codec(*cfg, widths, W_down, W_up, sigma2, nullptr, nullptr, out);
}

void spectra_codec_destroy(spectra_codec* codec) { delete codec; }

spectra_status spectra_codec_get_info(const spectra_codec* c, spectra_codec_info* out) {
  if (!c || !out) return fail(SPECTRA_ERR_INVALID, "null pointer");
  out->config = c->cfg;
  out->n_groups = c->n_groups;
  out->n_eff = c->h.n_eff;
  out->page_bytes = c->h.page_bytes;
  out->bits_per_token = c->h.page_bytes * 8 / c->cfg.page_tokens;
  out->max_kept = std::max(c->h.max_kept_k, c->h.max_kept_v);
  return SPECTRA_OK;
}

spectra_status spectra_codec_get_state(const spectra_codec* c, int32_t* widths, double* sigma2,
                                       double* theta, float* W_down, float* W_up) {
  if (!c) return fail(SPECTRA_ERR_INVALID, "null codec");
  if (widths) std::copy(c->widths.begin(), c->widths.end(), widths);
  if (sigma2) std::copy(c->sigma2.begin(), c->sigma2.end(), sigma2);
  if (theta) std::copy(c->theta.begin(), c->theta.end(), theta);
  if (W_down)
    for (size_t i = 0; i < c->wdown.size(); ++i) W_down[i] = bf16_bits_to_f32(c->wdown[i]);
  if (W_up) std::copy(c->wup.begin(), c->wup.end(), W_up);
  return SPECTRA_OK;
}

static const uint32_t kMagic = 0x54435053u;  // "SPCT"
static const uint32_t kBlobVersion = 1;

spectra_status spectra_codec_serialize(const spectra_codec* c, void* buf, size_t* bytes) {
  if (!c || !bytes) return fail(SPECTRA_ERR_INVALID, "null pointer");
  const size_t need = 8 + sizeof(spectra_config) + c->widths.size() * 4 + c->sigma2.size() * 8 +
                      c->theta.size() * 8 + c->wdown.size() * 2 + c->wup.size() * 4;
  if (!buf) {
    *bytes = need;
    return SPECTRA_OK;
  }
  if (*bytes < need) return fail(SPECTRA_ERR_INVALID, "buffer too small");
  uint8_t* p = static_cast<uint8_t*>(buf);
  auto put = [&](const void* src, size_t n) {
    std::memcpy(p, src, n);
    p += n;
  };
  put(&kMagic, 4);
  put(&kBlobVersion, 4);
  put(&c->cfg, sizeof(spectra_config));
  put(c->widths.data(), c->widths.size() * 4);
  put(c->sigma2.data(), c->sigma2.size() * 8);
  put(c->theta.data(), c->theta.size() * 8);
  put(c->wdown.data(), c->wdown.size() * 2);
  put(c->wup.data(), c->wup.size() * 4);
  *bytes = need;
  return SPECTRA_OK;
}

spectra_status spectra_codec_deserialize(const void* buf, size_t bytes, spectra_codec** out) {
  if (!buf || !out) return fail(SPECTRA_ERR_INVALID, "null pointer");
  *out = nullptr;
  const uint8_t* p = static_cast<const uint8_t*>(buf);
  const uint8_t* end = p + bytes;
  auto get = [&](void* dst, size_t n) {
    if ((size_t)(end - p) < n) return false;
    std::memcpy(dst, p, n);
    p += n;
    return true;
  };
  uint32_t magic = 0, ver = 0;
  spectra_config cfg{};
  if (!get(&magic, 4) || !get(&ver, 4) || magic != kMagic || ver != kBlobVersion)
    return fail(SPECTRA_ERR_INVALID, "not a libspectra codec blob (magic/version)");
  if (!get(&cfg, sizeof(cfg))) return fail(SPECTRA_ERR_INVALID, "truncated blob");
  std::string why;
  if (!valid_config(cfg, &why)) return fail(SPECTRA_ERR_INVALID, "blob config: " + why);
  const int ng = cfg.rank / cfg.group;
  std::vector<int32_t> w((size_t)cfg.n_kv_heads * 2 * ng);
  std::vector<double> s2((size_t)cfg.n_kv_heads * 2 * cfg.rank), th((size_t)cfg.n_kv_heads * 2);
  if (!get(w.data(), w.size() * 4) || !get(s2.data(), s2.size() * 8) || !get(th.data(), th.size() * 8))
    return fail(SPECTRA_ERR_INVALID, "truncated blob");
  CodecDev* tmp = new CodecDev();
  const int rc = build_layout(cfg, w.data(), tmp);
  const int n_eff = tmp->n_eff;
  delete tmp;
  if (rc) return fail(SPECTRA_ERR_INVALID, "blob widths invalid");
  std::vector<uint16_t> wd((size_t)cfg.d_model * n_eff);
  std::vector<float> wu((size_t)cfg.n_kv_heads * 2 * cfg.rank * cfg.d_head);
  if (!get(wd.data(), wd.size() * 2) || !get(wu.data(), wu.size() * 4))
    return fail(SPECTRA_ERR_INVALID, "truncated blob");
  if (p != end) return fail(SPECTRA_ERR_INVALID, "trailing bytes in blob");
  return build_codec(cfg, w.data(), nullptr, wu.data(), s2.data(), th.data(), wd.data(), out);
}

spectra_status spectra_calibrate(const spectra_config* cfg, int32_t dtype, const void* H,
                                 int64_t n_tokens, const void* W_K, const void* W_V,
                                 spectra_codec** out, void* stream) {
  return spectra_calibrate_ex(cfg, dtype, H, n_tokens, W_K, W_V, SPECTRA_ALLOC_WATERFILL, 0.0, out, stream);
}

spectra_status spectra_calibrate_ex(const spectra_config* cfg, int32_t dtype, const void* H,
                                    int64_t n_tokens, const void* W_K, const void* W_V, int32_t allocation,
                                    double energy_threshold, spectra_codec** out, void* stream) {
  if (!cfg || !H || !W_K || !W_V || !out) return fail(SPECTRA_ERR_INVALID, "null pointer");
  if (allocation != SPECTRA_ALLOC_WATERFILL && allocation != SPECTRA_ALLOC_UNIFORM)
    return fail(SPECTRA_ERR_INVALID, "unknown allocation");
  if (!(energy_threshold >= 0.0) || energy_threshold > 1.0)
    return fail(SPECTRA_ERR_INVALID, "energy_threshold must be 0 (off) or in (0, 1]");
  *out = nullptr;
  std::string why;
  if (!valid_config(*cfg, &why)) return fail(SPECTRA_ERR_INVALID, why);
  if (dtype != SPECTRA_F32 && dtype != SPECTRA_BF16) return fail(SPECTRA_ERR_INVALID, "dtype must be F32 or BF16");
  if (n_tokens < 2 || n_tokens > ((int64_t)1 << 30)) return fail(SPECTRA_ERR_INVALID, "n_tokens out of range");
  if (!aligned(H, 16) || !aligned(W_K, 16) || !aligned(W_V, 16))
    return fail(SPECTRA_ERR_INVALID, "inputs must be 16-byte aligned");
  const bool bf = dtype == SPECTRA_BF16;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int dm = cfg->d_model, dh = cfg->d_head, nkv = cfg->n_kv_heads, kvw = nkv * dh;
  const int r = cfg->rank, g = cfg->group, ng = r / g;

  DevBuf buf;
  const size_t off_flag = 0, off_G = 256;
  const size_t off_GW = off_G + ((size_t)dm * dm * 4 + 255) / 256 * 256;
  const size_t off_M = off_GW + ((size_t)dm * kvw * 4 + 255) / 256 * 256;
  const size_t off_V = off_M + ((size_t)nkv * 2 * dh * dh * 4 + 255) / 256 * 256;
  const size_t off_D = off_V + ((size_t)dh * dh * 4 + 255) / 256 * 256;
  const size_t total = off_D + ((size_t)dm * dh * 4 + 255) / 256 * 256;
  CUDA_TRY(cudaMalloc(&buf.p, total));
  uint8_t* base = static_cast<uint8_t*>(buf.p);
  int32_t* flag = reinterpret_cast<int32_t*>(base + off_flag);
  float* G = reinterpret_cast<float*>(base + off_G);
  float* GW = reinterpret_cast<float*>(base + off_GW);
  float* Mdev = reinterpret_cast<float*>(base + off_M);
  float* Vdev = reinterpret_cast<float*>(base + off_V);
  float* Ddev = reinterpret_cast<float*>(base + off_D);

  CUDA_TRY(cudaMemsetAsync(flag, 0, 4, st));
  CUDA_TRY(launch_check_finite(H, bf, n_tokens * dm, flag, st));
  CUDA_TRY(launch_check_finite(W_K, bf, (int64_t)dm * kvw, flag, st));
  CUDA_TRY(launch_check_finite(W_V, bf, (int64_t)dm * kvw, flag, st));
  // G = sum_t h_t^T h_t
  if (bf) {
    CUDA_TRY(launch_gram_tcgen05(static_cast<const uint16_t*>(H), n_tokens, dm, G, st));
  } else {
    CUDA_TRY(launch_gram_f32(static_cast<const float*>(H), n_tokens, dm, G, st));
  }
  // M_a = W_a^T G W_a per head and side
  for (int s = 0; s < 2; ++s) {
    const void* W = s == 0 ? W_K : W_V;
    CUDA_TRY(launch_gemm_nn_f32(G, false, dm, W, bf, kvw, GW, kvw, dm, kvw, dm, st));
    for (int a = 0; a < nkv; ++a) {
      const size_t esz = bf ? 2 : 4;
      const void* Wa = static_cast<const uint8_t*>(W) + (size_t)a * dh * esz;
      CUDA_TRY(launch_gemm_tn_f32(Wa, bf, kvw, GW + (size_t)a * dh, false, kvw,
                                  Mdev + ((size_t)a * 2 + s) * dh * dh, dh, dh, dh, dm, st));
    }
  }
  int32_t hflag = 0;
  std::vector<float> Mh((size_t)nkv * 2 * dh * dh);
  CUDA_TRY(cudaMemcpyAsync(&hflag, flag, 4, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaMemcpyAsync(Mh.data(), Mdev, Mh.size() * 4, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  if (hflag) return fail(SPECTRA_ERR_NUMERIC, "calibration inputs contain non-finite values");

  std::vector<int32_t> widths((size_t)nkv * 2 * ng);
  std::vector<double> sigma2((size_t)nkv * 2 * r), theta((size_t)nkv * 2);
  std::vector<float> wup((size_t)nkv * 2 * r * dh, 0.f);
  std::vector<double> Mdbl((size_t)dh * dh), vals(dh), vecs((size_t)dh * dh);
  std::vector<std::vector<double>> basis((size_t)nkv * 2);
  for (int a = 0; a < nkv; ++a)
    for (int s = 0; s < 2; ++s) {
      const size_t hs = (size_t)a * 2 + s;
      for (size_t i = 0; i < Mdbl.size(); ++i) Mdbl[i] = (double)Mh[hs * dh * dh + i] / (double)n_tokens;
      if (sym_eigen(Mdbl.data(), dh, vals.data(), vecs.data()))
        return fail(SPECTRA_ERR_NUMERIC, "eigen-decomposition of W^T G W failed");
      const double tol = 1e-6 * std::max(vals[0], 1e-300);
      for (int i = 0; i < dh; ++i) {
        if (vals[i] < -tol) return fail(SPECTRA_ERR_NUMERIC, "W^T G W is not positive semi-definite");
        if (vals[i] < 0) vals[i] = 0;
      }
      std::copy(vals.begin(), vals.begin() + r, sigma2.begin() + hs * r);
      // groups eligible for bits: all, or those holding the leading coordinates
      // up to the energy rank (rounded up to whole groups)
      int n_elig = ng;
      if (energy_threshold > 0.0) {
        int re = dh;
        energy_rank(vals.data(), dh, energy_threshold, &re);
        n_elig = std::min(ng, (re + g - 1) / g);
      }
      int32_t* wj = widths.data() + hs * ng;
      std::fill(wj, wj + ng, 0);
      if (allocation == SPECTRA_ALLOC_UNIFORM)
        allocate_widths_uniform(vals.data(), r, g, n_elig, cfg->budget_bits, cfg->count_overhead != 0, wj, nullptr);
      else
        allocate_widths(vals.data(), n_elig * g, g, cfg->budget_bits, cfg->count_overhead != 0, wj, nullptr);
      int payload = 0;
      for (int j = 0; j < ng; ++j) payload += g * widths[hs * ng + j];
      water_fill(vals.data(), r, (double)payload, &theta[hs], nullptr);
      for (int i = 0; i < r; ++i)
        for (int d = 0; d < dh; ++d) wup[(hs * r + i) * dh + d] = (float)vecs[(size_t)d * dh + i];
      basis[hs] = vecs;
    }

  // W_down = W V_r, kept columns only, in the latent order of the codec
  CodecDev lay{};
  if (build_layout(*cfg, widths.data(), &lay)) return fail(SPECTRA_ERR_INVALID, "layout failed");
  const int n_eff = lay.n_eff;
  std::vector<float> wdown((size_t)dm * std::max(n_eff, 1), 0.f);
  std::vector<float> vkeep, dtmp((size_t)dm * dh);
  for (int a = 0; a < nkv; ++a)
    for (int s = 0; s < 2; ++s) {
      const size_t hs = (size_t)a * 2 + s;
      const SideDev& sd = lay.head[a].side[s];
      if (sd.n_kept == 0) continue;
      vkeep.assign((size_t)dh * sd.n_kept, 0.f);
      int col = 0;
      for (int j = 0; j < ng; ++j) {
        if (widths[hs * ng + j] == 0) continue;
        for (int k = 0; k < g; ++k, ++col)
          for (int d = 0; d < dh; ++d)
            vkeep[(size_t)d * sd.n_kept + col] = (float)basis[hs][(size_t)d * dh + j * g + k];
      }
      const void* W = s == 0 ? W_K : W_V;
      const void* Wa = static_cast<const uint8_t*>(W) + (size_t)a * dh * (bf ? 2 : 4);
      CUDA_TRY(cudaMemcpyAsync(Vdev, vkeep.data(), vkeep.size() * 4, cudaMemcpyHostToDevice, st));
      CUDA_TRY(launch_gemm_nn_f32(Wa, bf, kvw, Vdev, false, sd.n_kept, Ddev, sd.n_kept, dm,
                                  sd.n_kept, dh, st));
      CUDA_TRY(cudaMemcpyAsync(dtmp.data(), Ddev, (size_t)dm * sd.n_kept * 4, cudaMemcpyDeviceToHost, st));
      CUDA_TRY(cudaStreamSynchronize(st));
      for (int k = 0; k < dm; ++k)
        for (int c = 0; c < sd.n_kept; ++c)
          wdown[(size_t)k * n_eff + sd.c_col0 + c] = dtmp[(size_t)k * sd.n_kept + c];
    }
  return build_codec(*cfg, widths.data(), wdown.data(), wup.data(), sigma2.data(), theta.data(),
                     nullptr, out);
}

spectra_status spectra_wo_correction(const spectra_codec* c, int32_t dtype, const void* H,
                                     int64_t n_tokens, const void* W_Q, const void* W_K,
                                     const void* W_V, const void* W_O, float* W_O_out,
                                     void* stream) {
  if (!c || !H || !W_Q || !W_K || !W_V || !W_O || !W_O_out) return fail(SPECTRA_ERR_INVALID, "null pointer");
  if (dtype != SPECTRA_F32 && dtype != SPECTRA_BF16) return fail(SPECTRA_ERR_INVALID, "dtype must be F32 or BF16");
  if (n_tokens < 2 || n_tokens > 4096) return fail(SPECTRA_ERR_INVALID, "n_tokens must be in 2..4096");
  spectra_status stt = check_device(c);
  if (stt != SPECTRA_OK) return stt;
  const bool bf = dtype == SPECTRA_BF16;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const spectra_config& cfg = c->cfg;
  const int dm = cfg.d_model, dh = cfg.d_head, nkv = cfg.n_kv_heads, nq = cfg.n_q_heads;
  const int gq = nq / nkv, n = (int)n_tokens, ng = c->n_groups;
  const size_t esz = bf ? 2 : 4;
  // kept directions per (head, side): columns of V_r for groups with b > 0
  auto kept_basis = [&](int a, int s, std::vector<float>& U) {
    const size_t hs = (size_t)a * 2 + s;
    std::vector<int> rows;
    for (int j = 0; j < ng; ++j)
      if (c->widths[hs * ng + j] != 0)
        for (int k = 0; k < cfg.group; ++k) rows.push_back(j * cfg.group + k);
    U.assign((size_t)dh * rows.size(), 0.f);  // [dh][kept]
    for (size_t r = 0; r < rows.size(); ++r)
      for (int d = 0; d < dh; ++d) U[(size_t)d * rows.size() + r] = c->wup[(hs * cfg.rank + rows[r]) * dh + d];
    return (int)rows.size();
  };
  DevBuf buf;
  const size_t szQ = (size_t)n * nq * dh, szKV = (size_t)n * nkv * dh;
  const size_t total = (szQ + 4 * szKV + 2 * (size_t)n * dh + (size_t)dh * dh) * 4 + 4096;
  CUDA_TRY(cudaMalloc(&buf.p, total));
  float* Q = static_cast<float*>(buf.p);
  float* K = Q + szQ;
  float* V = K + szKV;
  float* Kt = V + szKV;    // truncated keys, [n][nkv*dh]
  float* Vl = Kt + szKV;   // latent values per head, [n][nkv*dh] (first kept columns used)
  float* O = Vl + szKV;    // [n][dh]
  float* Ol = O + (size_t)n * dh;
  float* Pm = Ol + (size_t)n * dh;
  CUDA_TRY(launch_gemm_nn_f32(H, bf, dm, W_Q, bf, nq * dh, Q, nq * dh, n, nq * dh, dm, st));
  CUDA_TRY(launch_gemm_nn_f32(H, bf, dm, W_K, bf, nkv * dh, K, nkv * dh, n, nkv * dh, dm, st));
  CUDA_TRY(launch_gemm_nn_f32(H, bf, dm, W_V, bf, nkv * dh, V, nkv * dh, n, nkv * dh, dm, st));
  std::vector<int> keptV(nkv);
  std::vector<std::vector<float>> UV(nkv);
  for (int a = 0; a < nkv; ++a) {
    std::vector<float> Uk;
    const int kk = kept_basis(a, 0, Uk);
    std::vector<float> P((size_t)dh * dh, 0.f);  // U_k U_k^T
    for (int x = 0; x < dh; ++x)
      for (int y = 0; y < dh; ++y) {
        double acc = 0.0;
        for (int r = 0; r < kk; ++r) acc += (double)Uk[(size_t)x * kk + r] * Uk[(size_t)y * kk + r];
        P[(size_t)x * dh + y] = (float)acc;
      }
    CUDA_TRY(cudaMemcpyAsync(Pm, P.data(), P.size() * 4, cudaMemcpyHostToDevice, st));
    CUDA_TRY(launch_gemm_nn_f32(K + (size_t)a * dh, false, nkv * dh, Pm, false, dh, Kt + (size_t)a * dh, nkv * dh,
                                n, dh, dh, st));
    keptV[a] = kept_basis(a, 1, UV[a]);
    if (keptV[a] > 0) {
      CUDA_TRY(cudaMemcpyAsync(Pm + (size_t)dh * dh, UV[a].data(), UV[a].size() * 4, cudaMemcpyHostToDevice, st));
      CUDA_TRY(launch_gemm_nn_f32(V + (size_t)a * dh, false, nkv * dh, Pm + (size_t)dh * dh, false, keptV[a],
                                  Vl + (size_t)a * dh, nkv * dh, n, keptV[a], dh, st));
    }
    CUDA_TRY(cudaStreamSynchronize(st));  // host buffers are reused for the next head
  }
  std::vector<float> Lh((size_t)n * dh), Oh((size_t)n * dh), Ms((size_t)dh * dh);
  for (int h = 0; h < nq; ++h) {
    const int a = h / gq, kv = keptV[a];
    std::fill(Ms.begin(), Ms.end(), 0.f);
    if (kv > 0) {
      const float* Qh = Q + (size_t)h * dh;
      CUDA_TRY(launch_causal_attention(Qh, K + (size_t)a * dh, V + (size_t)a * dh, O, n, dh, dh, nq * dh,
                                       nkv * dh, nkv * dh, dh, st));
      CUDA_TRY(launch_causal_attention(Qh, Kt + (size_t)a * dh, Vl + (size_t)a * dh, Ol, n, dh, kv, nq * dh,
                                       nkv * dh, nkv * dh, kv, st));
      CUDA_TRY(cudaMemcpyAsync(Lh.data(), Ol, (size_t)n * kv * 4, cudaMemcpyDeviceToHost, st));
      CUDA_TRY(cudaMemcpyAsync(Oh.data(), O, (size_t)n * dh * 4, cudaMemcpyDeviceToHost, st));
      CUDA_TRY(cudaStreamSynchronize(st));
      // normal equations formed in fp64 from the fp32 attention outputs: the
      // solve then loses about cond(L) (not cond(L)^2) digits of the fp32 inputs
      std::vector<double> A2((size_t)kv * kv, 0.0), B2((size_t)kv * dh, 0.0);
      for (int t = 0; t < n; ++t) {
        const float* lr = Lh.data() + (size_t)t * kv;
        const float* orow = Oh.data() + (size_t)t * dh;
        for (int i = 0; i < kv; ++i) {
          const double li = lr[i];
          for (int j = 0; j < kv; ++j) A2[(size_t)i * kv + j] += li * lr[j];
          for (int j = 0; j < dh; ++j) B2[(size_t)i * dh + j] += li * orow[j];
        }
      }
      double tr = 0.0;
      for (int i = 0; i < kv; ++i) tr += A2[(size_t)i * kv + i];
      const double eps = 1e-8 * tr / kv;
      for (int i = 0; i < kv; ++i) A2[(size_t)i * kv + i] += eps;
      if (!solve_dense(A2, B2, kv, dh)) return fail(SPECTRA_ERR_NUMERIC, "singular W_O correction system");
      // M = U M'  (dh x dh)
      for (int x = 0; x < dh; ++x)
        for (int y = 0; y < dh; ++y) {
          double acc = 0.0;
          for (int r = 0; r < kv; ++r) acc += (double)UV[a][(size_t)x * kv + r] * B2[(size_t)r * dh + y];
          Ms[(size_t)x * dh + y] = (float)acc;
        }
    }
    CUDA_TRY(cudaMemcpyAsync(Pm, Ms.data(), Ms.size() * 4, cudaMemcpyHostToDevice, st));
    const void* WOh = static_cast<const uint8_t*>(W_O) + (size_t)h * dh * dm * esz;
    CUDA_TRY(launch_gemm_nn_f32(Pm, false, dh, WOh, bf, dm, W_O_out + (size_t)h * dh * dm, dm, dh, dm, dh, st));
    CUDA_TRY(cudaStreamSynchronize(st));
  }
  return SPECTRA_OK;
}

spectra_status spectra_encode_workspace_bytes(const spectra_codec* c, int64_t max_tokens, size_t* bytes) {
  if (!c || !bytes || max_tokens < 0) return fail(SPECTRA_ERR_INVALID, "bad arguments");
  *bytes = encode_ws_bytes(c, max_tokens);
  return SPECTRA_OK;
}

spectra_status spectra_decode_workspace_bytes(const spectra_codec* c, int32_t batch, int64_t max_len,
                                              size_t* bytes) {
  if (!c || !bytes || batch <= 0 || max_len < 0) return fail(SPECTRA_ERR_INVALID, "bad arguments");
  const DecodePlan p = make_decode_plan(c->h, batch, 1 << 30);
  *bytes = p.ws_bytes;
  return SPECTRA_OK;
}

spectra_status spectra_project(const spectra_codec* c, const void* H, int64_t T, float* latents,
                               void* stream) {
  if (!c || !H || !latents) return fail(SPECTRA_ERR_INVALID, "null pointer");
  if (T <= 0 || T > (1 << 24)) return fail(SPECTRA_ERR_INVALID, "T out of range");
  if (!aligned(H, 16) || !aligned(latents, 16)) return fail(SPECTRA_ERR_INVALID, "H and latents must be 16-byte aligned");
  spectra_status s = check_device(c);
  if (s != SPECTRA_OK) return s;
  return do_project(c, H, T, latents, static_cast<cudaStream_t>(stream));
}

spectra_status spectra_quantize_append(const spectra_codec* c, const spectra_cache* cache,
                                       const float* latents, const int32_t* seq_ids, int64_t T,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  if (!c || !latents || !seq_ids || !workspace) return fail(SPECTRA_ERR_INVALID, "null pointer");
  if (T <= 0 || T > (1 << 24)) return fail(SPECTRA_ERR_INVALID, "T out of range");
  if (!aligned(latents, 16) || !aligned(workspace, 256)) return fail(SPECTRA_ERR_INVALID, "misaligned buffer");
  if (workspace_bytes < kEncCounterBytes + ((size_t)T * 4 + 255) / 256 * 256 + 256)
    return fail(SPECTRA_ERR_INVALID, "workspace too small");
  spectra_status s = check_cache(c, cache);
  if (s != SPECTRA_OK) return s;
  s = check_device(c);
  if (s != SPECTRA_OK) return s;
  return do_quantize_append(c, cache, latents, seq_ids, T, workspace, static_cast<cudaStream_t>(stream));
}

spectra_status spectra_encode_append(const spectra_codec* c, const spectra_cache* cache, const void* H,
                                     const int32_t* seq_ids, int64_t T, float* latents_out,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  if (!c || !H || !seq_ids || !workspace) return fail(SPECTRA_ERR_INVALID, "null pointer");
  if (T <= 0 || T > (1 << 24)) return fail(SPECTRA_ERR_INVALID, "T out of range");
  if (!aligned(H, 16) || !aligned(workspace, 256) || (latents_out && !aligned(latents_out, 16)))
    return fail(SPECTRA_ERR_INVALID, "misaligned buffer");
  if (workspace_bytes < encode_ws_bytes(c, T)) return fail(SPECTRA_ERR_INVALID, "workspace too small");
  spectra_status s = check_cache(c, cache);
  if (s != SPECTRA_OK) return s;
  s = check_device(c);
  if (s != SPECTRA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T <= kFusedMaxT) {
    // decode steps: projection, quantisation and packing fused per kept group
    uint8_t* w = static_cast<uint8_t*>(workspace);
    float* part = reinterpret_cast<float*>(w + kEncCounterBytes + ((size_t)T * 4 + 255) / 256 * 256 + 256);
    CUDA_TRY(launch_encode_fused(c->h, c->d, static_cast<const uint16_t*>(H), seq_ids, (int)T, *cache,
                                 latents_out, reinterpret_cast<int32_t*>(w), part, st));
    return SPECTRA_OK;
  }
  if (!latents_out && T >= kGemmMinT) {
    // prefill: the append plan, then the projection GEMM with quantise/pack in
    // its epilogue (no fp32 latents in memory)
    uint8_t* w = static_cast<uint8_t*>(workspace) + kEncCounterBytes;
    int32_t* pos = reinterpret_cast<int32_t*>(w);
    int32_t* flag = reinterpret_cast<int32_t*>(w + ((size_t)T * 4 + 255) / 256 * 256);
    CUDA_TRY(launch_append_plan(seq_ids, (int)T, *cache, c->cfg.page_tokens, pos, flag, c->err, st));
    CUDA_TRY(launch_encode_gemm(c->h, c->d, static_cast<const uint16_t*>(H), (int)T, seq_ids, pos, flag, *cache,
                                st));
    return SPECTRA_OK;
  }
  uint8_t* w = static_cast<uint8_t*>(workspace);
  const size_t lat_off = kEncCounterBytes + ((size_t)T * 4 + 255) / 256 * 256 + 256;
  float* C = latents_out ? latents_out : reinterpret_cast<float*>(w + lat_off);
  s = do_project(c, H, T, C, st);
  if (s != SPECTRA_OK) return s;
  return do_quantize_append(c, cache, C, seq_ids, T, workspace, st);
}

spectra_status spectra_decode_attend(const spectra_codec* c, const spectra_cache* cache, const float* q,
                                     float* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!c || !q || !out || !workspace) return fail(SPECTRA_ERR_INVALID, "null pointer");
  if (!c->decode_ok) return fail(SPECTRA_ERR_UNSUPPORTED, c->decode_why);
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256))
    return fail(SPECTRA_ERR_INVALID, "misaligned buffer");
  spectra_status s = check_cache(c, cache);
  if (s != SPECTRA_OK) return s;
  s = check_device(c);
  if (s != SPECTRA_OK) return s;
  const DecodePlan plan = make_decode_plan(c->h, cache->batch, cache->max_pages_per_seq);
  if (workspace_bytes < plan.ws_bytes) return fail(SPECTRA_ERR_INVALID, "workspace too small");
  CUDA_TRY(launch_decode(c->h, c->d, *cache, q, out, workspace, plan, static_cast<cudaStream_t>(stream)));
  return SPECTRA_OK;
}

spectra_status spectra_decode_reconstruct_workspace_bytes(const spectra_codec* c, int32_t batch, int64_t max_len,
                                                          size_t* bytes) {
  if (!c || !bytes || batch <= 0 || max_len < 0) return fail(SPECTRA_ERR_INVALID, "bad arguments");
  const int64_t pages = (max_len + c->h.P - 1) / c->h.P;
  const RtPlan p = make_rt_plan(c->h, batch, (int)std::min<int64_t>(std::max<int64_t>(pages, 1), 1 << 30), true);
  *bytes = p.ws_bytes;
  return SPECTRA_OK;
}

spectra_status spectra_decode_attend_reconstruct(const spectra_codec* c, const spectra_cache* cache, const float* q,
                                                 double rope_theta, float* out, void* workspace,
                                                 size_t workspace_bytes, void* stream) {
  if (!c || !q || !out || !workspace) return fail(SPECTRA_ERR_INVALID, "null pointer");
  if (!(rope_theta == 0.0 || (rope_theta > 1.0 && std::isfinite(rope_theta))))
    return fail(SPECTRA_ERR_INVALID, "rope_theta must be 0 (no rotation) or a finite base above 1");
  std::string why;
  if (!rt_supported(c->h, &why)) return fail(SPECTRA_ERR_UNSUPPORTED, why);
  if (!aligned(q, 4) || !aligned(out, 4) || !aligned(workspace, 256))
    return fail(SPECTRA_ERR_INVALID, "misaligned buffer");
  spectra_status s = check_cache(c, cache);
  if (s != SPECTRA_OK) return s;
  s = check_device(c);
  if (s != SPECTRA_OK) return s;
  const RtPlan plan = make_rt_plan(c->h, cache->batch, cache->max_pages_per_seq);
  if (workspace_bytes < plan.ws_bytes) return fail(SPECTRA_ERR_INVALID, "workspace too small");
  CUDA_TRY(launch_decode_reconstruct(c->h, c->d, *cache, q, rope_theta, out, workspace, plan,
                                     static_cast<cudaStream_t>(stream)));
  return SPECTRA_OK;
}

spectra_status spectra_reconstruct(const spectra_codec* c, const spectra_cache* cache, int32_t seq, int64_t t0,
                                   int64_t n, float* K_out, float* V_out, void* stream) {
  if (!c || !K_out || !V_out) return fail(SPECTRA_ERR_INVALID, "null pointer");
  spectra_status s = check_cache(c, cache);
  if (s != SPECTRA_OK) return s;
  if (seq < 0 || seq >= cache->batch) return fail(SPECTRA_ERR_INVALID, "seq out of range");
  if (t0 < 0 || n < 0 || n > ((int64_t)1 << 26)) return fail(SPECTRA_ERR_INVALID, "token range out of range");
  if (!aligned(K_out, 4) || !aligned(V_out, 4)) return fail(SPECTRA_ERR_INVALID, "misaligned buffer");
  s = check_device(c);
  if (s != SPECTRA_OK) return s;
  CUDA_TRY(launch_reconstruct(c->h, c->d, *cache, seq, t0, n, K_out, V_out, static_cast<cudaStream_t>(stream)));
  return SPECTRA_OK;
}

spectra_status spectra_device_status(const spectra_codec* c, void* stream) {
  if (!c) return fail(SPECTRA_ERR_INVALID, "null codec");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUDA_TRY(cudaStreamSynchronize(st));
  int32_t v = 0;
  CUDA_TRY(cudaMemcpy(&v, c->err, 4, cudaMemcpyDeviceToHost));
  CUDA_TRY(cudaMemset(c->err, 0, 4));
  if (v == 0) return SPECTRA_OK;
  return fail(static_cast<spectra_status>(v), "device-side error recorded by a kernel");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode attention without any allocation.
//
// Some callers cannot allocate device memory at all when they run decode: a
// runtime that plans every buffer statically ahead of time, a host process
// whose allocator is owned by another framework, or code that runs where a
// cudaMalloc would stall or be refused.  They still own their inputs and
// outputs, but have nowhere to put the decode's scratch (folded queries and
// the split-K partial records).  This entry point keeps that scratch in one
// file-scope device array of fixed size instead.  The array exists on every
// GPU that loads the library until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = 4u << 20;  // 4 MiB per device
static __device__ __align__(256) uint8_t g_static_decode_scratch[kStaticScratchBytes];

struct StaticScratch {
  std::mutex mu;
  void* ptr[64] = {};
};
StaticScratch g_static_scratch;

}  // namespace

extern "C" spectra_status spectra_decode_attend_noalloc(const spectra_codec* c, const spectra_cache* cache,
                                                        const float* q, float* out, void* stream) {
  if (!c || !q || !out) return fail(SPECTRA_ERR_INVALID, "null pointer");
  if (!c->decode_ok) return fail(SPECTRA_ERR_UNSUPPORTED, c->decode_why);
  if (!aligned(q, 16) || !aligned(out, 16)) return fail(SPECTRA_ERR_INVALID, "misaligned buffer");
  spectra_status s = check_cache(c, cache);
  if (s != SPECTRA_OK) return s;
  s = check_device(c);
  if (s != SPECTRA_OK) return s;
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(SPECTRA_ERR_UNSUPPORTED, "device ordinal above 63");
  void* scratch = nullptr;
  {
    // First call on this device: look up the device address of the static array
    // (the host-side symbol is not a device address).
    std::lock_guard<std::mutex> lock(g_static_scratch.mu);
    if (!g_static_scratch.ptr[dev]) {
      void* p = nullptr;
      CUDA_TRY(cudaGetSymbolAddress(&p, g_static_decode_scratch));
      g_static_scratch.ptr[dev] = p;
    }
    scratch = g_static_scratch.ptr[dev];
  }
  const DecodePlan plan = make_decode_plan(c->h, cache->batch, cache->max_pages_per_seq);
  if (plan.ws_bytes > kStaticScratchBytes)
    return fail(SPECTRA_ERR_CAPACITY, "decode needs " + std::to_string(plan.ws_bytes) +
                                          " bytes of scratch; the static area holds 4 MiB (use "
                                          "spectra_decode_attend with a caller workspace)");
  CUDA_TRY(launch_decode(c->h, c->d, *cache, q, out, scratch, plan, static_cast<cudaStream_t>(stream)));
  return SPECTRA_OK;
}
