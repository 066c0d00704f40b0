// Host-side math of libspectra: grouped bit allocation, reverse water-filling,
// symmetric eigen-decomposition and the page layout.  Plain C++ (fp64), no CUDA.
//
// Follows "SPECTRA: Pushing the KV Cache Beyond the 2-Bit Cliff via Spectral
// Transform Coding", technical summary, "SPECTRA pipeline": stage 1 (the
// eigen-basis of W^T G W, i.e. the right singular vectors of G^{1/2} W), stage 2
// (reverse water-filling on the latent second moments, adjacent coordinates
// grouped under one width, zero bits drop a group).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>
#include <string>
#include <vector>

#include "spectra_internal.h"

namespace spectra {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

spectra_status fail(spectra_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

static const int kWidths[6] = {0, 1, 2, 3, 4, 8};

static int group_cost(int b, int g, bool overhead) {
  return b == 0 ? 0 : g * b + (overhead ? 32 : 0);
}

// Backward dynamic programme over groups j = n-1..0 and remaining budget c:
// best[j][c] = min_b  S_j 4^-b + best[j+1][c - cost(b)], widths tried in
// increasing order with strict improvement (ties keep the smaller width).
int allocate_widths(const double* sigma2, int rank, int group, int budget, bool overhead,
                    int32_t* widths, double* distortion) {
  if (group <= 0 || rank % group != 0 || budget < 0) return 1;
  const int n = rank / group;
  std::vector<double> S(n, 0.0);
  for (int j = 0; j < n; ++j) {
    double acc = 0.0;
    for (int i = j * group; i < (j + 1) * group; ++i) acc += sigma2[i];
    S[j] = acc;
  }
  const int W = budget + 1;
  std::vector<double> best((size_t)(n + 1) * W, 0.0);
  std::vector<int8_t> pick((size_t)n * W, 0);
  for (int j = n - 1; j >= 0; --j) {
    for (int c = 0; c <= budget; ++c) {
      double v_best = std::numeric_limits<double>::infinity();
      int b_best = 0;
      for (int wi = 0; wi < 6; ++wi) {
        const int b = kWidths[wi];
        const int cost = group_cost(b, group, overhead);
        if (cost > c) continue;
        const double d = S[j] * std::ldexp(1.0, -2 * b);
        const double v = d + best[(size_t)(j + 1) * W + (c - cost)];
        if (v < v_best) {
          v_best = v;
          b_best = b;
        }
      }
      best[(size_t)j * W + c] = v_best;
      pick[(size_t)j * W + c] = (int8_t)b_best;
    }
  }
  int c = budget;
  double dist = 0.0;
  for (int j = 0; j < n; ++j) {
    const int b = pick[(size_t)j * W + c];
    widths[j] = b;
    c -= group_cost(b, group, overhead);
  }
  for (int j = n - 1; j >= 0; --j) dist = S[j] * std::ldexp(1.0, -2 * widths[j]) + dist;
  if (distortion) *distortion = dist;
  return 0;
}

// Uniform allocation ("SpectralQuant with uniform allocation" of "Ablation,
// Statistical Inference, and Validation for KV-Cache Compression", practical
// recommendations): every kept group gets the same width b and the kept groups
// are the leading k of the first n_eligible; (k, b) minimises the same model
// sum_j S_j 4^-b_j under the budget (ties: fewer bits, then fewer groups).
int allocate_widths_uniform(const double* sigma2, int rank, int group, int n_eligible, int budget,
                            bool overhead, int32_t* widths, double* distortion) {
  if (group <= 0 || rank % group != 0 || budget < 0) return 1;
  const int n = rank / group;
  n_eligible = std::max(0, std::min(n_eligible, n));
  std::vector<double> S(n, 0.0);
  double total = 0.0;
  for (int j = 0; j < n; ++j) {
    double acc = 0.0;
    for (int i = j * group; i < (j + 1) * group; ++i) acc += sigma2[i];
    S[j] = acc;
  }
  for (int j = n - 1; j >= 0; --j) total = S[j] + total;
  double best = total;
  int best_k = 0, best_b = 0, best_bits = 0;
  for (int wi = 1; wi < 6; ++wi) {
    const int b = kWidths[wi];
    const int cost = group_cost(b, group, overhead);
    double kept = 0.0;  // sum_{j<k} S_j
    for (int k = 1; k <= n_eligible; ++k) {
      if ((int64_t)k * cost > budget) break;
      kept += S[k - 1];
      double rest = 0.0;
      for (int j = n - 1; j >= k; --j) rest = S[j] + rest;
      const double d = kept * std::ldexp(1.0, -2 * b) + rest;
      const int bits = k * cost;
      if (d < best || (d == best && bits < best_bits)) {
        best = d;
        best_k = k;
        best_b = b;
        best_bits = bits;
      }
    }
  }
  for (int j = 0; j < n; ++j) widths[j] = j < best_k ? best_b : 0;
  if (distortion) *distortion = best;
  return 0;
}

// Effective rank ("Spectral-KV: SVD-projection KV cache compression (28x)",
// technical principle 1, spectral profiling): the smallest r with
// sum_{i<r} sigma2_i >= threshold * sum_i sigma2_i (sigma2 descending).
int energy_rank(const double* sigma2, int n, double threshold, int* r) {
  if (n <= 0 || !(threshold > 0.0) || threshold > 1.0) return 1;
  double total = 0.0;
  for (int i = 0; i < n; ++i) total += sigma2[i];
  double acc = 0.0;
  int k = n;
  for (int i = 0; i < n; ++i) {
    acc += sigma2[i];
    if (acc >= threshold * total) {
      k = i + 1;
      break;
    }
  }
  *r = k;
  return 0;
}

// Reverse water-filling in closed form: with the k largest second moments
// active, log theta = (sum_{i<k} log s_i - 2 R ln 2) / k; the right k is the one
// whose theta lies in [s_(k+1), s_k).
int water_fill(const double* sigma2, int n, double rate, double* theta, double* rates) {
  if (n <= 0) return 1;
  std::vector<double> s;
  for (int i = 0; i < n; ++i)
    if (sigma2[i] > 0) s.push_back(sigma2[i]);
  std::sort(s.begin(), s.end(), [](double a, double b) { return a > b; });
  double th = 0.0;
  if (s.empty()) {
    th = 0.0;
  } else if (rate <= 0) {
    th = s[0];
  } else {
    double logsum = 0.0;
    th = s[0];
    for (size_t k = 1; k <= s.size(); ++k) {
      logsum += std::log(s[k - 1]);
      const double t = std::exp((logsum - 2.0 * rate * std::log(2.0)) / (double)k);
      if (t < s[k - 1] && (k == s.size() || t >= s[k])) {
        th = t;
        break;
      }
    }
  }
  if (theta) *theta = th;
  if (rates)
    for (int i = 0; i < n; ++i)
      rates[i] = (sigma2[i] > th && th > 0) ? 0.5 * std::log2(sigma2[i] / th) : 0.0;
  return 0;
}

// Cyclic Jacobi on a symmetric matrix: rotations J(p,q,theta) zero A_pq one at a
// time; V accumulates the product of the rotations (its columns converge to
// eigenvectors).  Then eigenpairs are sorted by decreasing eigenvalue (stable)
// and each vector is signed so that its largest-magnitude entry (lowest index on
// ties) is positive.
int sym_eigen(const double* M, int n, double* vals, double* vecs) {
  if (n <= 0 || n > 512) return 1;
  std::vector<double> A(M, M + (size_t)n * n);
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < i; ++j) {
      const double m = 0.5 * (A[(size_t)i * n + j] + A[(size_t)j * n + i]);
      if (!std::isfinite(m)) return 2;
      A[(size_t)i * n + j] = A[(size_t)j * n + i] = m;
    }
  std::vector<double> V((size_t)n * n, 0.0);
  for (int i = 0; i < n; ++i) V[(size_t)i * n + i] = 1.0;
  double frob = 0.0;
  for (double a : A) frob += a * a;
  bool converged = false;
  for (int sweep = 0; sweep < 64; ++sweep) {
    double off = 0.0;
    for (int p = 0; p < n; ++p)
      for (int q = p + 1; q < n; ++q) off += A[(size_t)p * n + q] * A[(size_t)p * n + q];
    if (off <= 1e-30 * frob || off == 0.0) {
      converged = true;
      break;
    }
    for (int p = 0; p < n - 1; ++p) {
      for (int q = p + 1; q < n; ++q) {
        const double apq = A[(size_t)p * n + q];
        if (apq == 0.0) continue;
        const double app = A[(size_t)p * n + p], aqq = A[(size_t)q * n + q];
        if (sweep > 3 && std::fabs(apq) < 1e-18 * std::fabs(app) &&
            std::fabs(apq) < 1e-18 * std::fabs(aqq)) {
          A[(size_t)p * n + q] = A[(size_t)q * n + p] = 0.0;
          continue;
        }
        const double th = (aqq - app) / (2.0 * apq);
        const double t = (th >= 0 ? 1.0 : -1.0) / (std::fabs(th) + std::sqrt(th * th + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < n; ++k) {  // columns p, q of A J
          const double akp = A[(size_t)k * n + p], akq = A[(size_t)k * n + q];
          A[(size_t)k * n + p] = c * akp - s * akq;
          A[(size_t)k * n + q] = s * akp + c * akq;
        }
        for (int k = 0; k < n; ++k) {  // rows p, q of J^T (A J)
          const double apk = A[(size_t)p * n + k], aqk = A[(size_t)q * n + k];
          A[(size_t)p * n + k] = c * apk - s * aqk;
          A[(size_t)q * n + k] = s * apk + c * aqk;
        }
        A[(size_t)p * n + q] = A[(size_t)q * n + p] = 0.0;
        for (int k = 0; k < n; ++k) {
          const double vkp = V[(size_t)k * n + p], vkq = V[(size_t)k * n + q];
          V[(size_t)k * n + p] = c * vkp - s * vkq;
          V[(size_t)k * n + q] = s * vkp + c * vkq;
        }
      }
    }
  }
  if (!converged) {
    double off = 0.0;
    for (int p = 0; p < n; ++p)
      for (int q = p + 1; q < n; ++q) off += A[(size_t)p * n + q] * A[(size_t)p * n + q];
    if (off > 1e-24 * frob) return 3;
  }
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) {
    return A[(size_t)x * n + x] > A[(size_t)y * n + y];
  });
  for (int c = 0; c < n; ++c) {
    const int src = order[c];
    vals[c] = A[(size_t)src * n + src];
    int imax = 0;
    double vmax = -1.0;
    for (int k = 0; k < n; ++k) {
      const double m = std::fabs(V[(size_t)k * n + src]);
      if (m > vmax) {
        vmax = m;
        imax = k;
      }
    }
    const double sg = V[(size_t)imax * n + src] < 0 ? -1.0 : 1.0;
    for (int k = 0; k < n; ++k) vecs[(size_t)k * n + c] = sg * V[(size_t)k * n + src];
  }
  return 0;
}

bool valid_config(const spectra_config& c, std::string* why) {
  auto bad = [&](const char* m) {
    if (why) *why = m;
    return false;
  };
  if (c.d_model <= 0 || c.d_model % 8 != 0) return bad("d_model must be a positive multiple of 8");
  if (c.n_kv_heads <= 0 || c.n_kv_heads > kMaxKV) return bad("n_kv_heads must be in 1..32");
  if (c.n_q_heads <= 0 || c.n_q_heads % c.n_kv_heads != 0) return bad("n_q_heads must be a multiple of n_kv_heads");
  if (c.n_q_heads / c.n_kv_heads > kMaxGQ) return bad("n_q_heads / n_kv_heads must be <= 8");
  if (c.d_head <= 0 || c.d_head > kMaxDHead || c.d_head % 8 != 0) return bad("d_head must be a multiple of 8 in 8..256");
  if (c.group != 8 && c.group != 16) return bad("group must be 8 or 16");
  if (c.rank <= 0 || c.rank > c.d_head || c.rank % c.group != 0) return bad("rank must be a multiple of group, <= d_head");
  if (c.rank / c.group > kMaxGroups) return bad("too many groups");
  if (c.budget_bits < 0 || c.budget_bits > 65536) return bad("budget_bits out of range");
  if (c.page_tokens < 32 || c.page_tokens > 1024 || c.page_tokens % 32 != 0) return bad("page_tokens must be a multiple of 32 in 32..1024");
  return true;
}

int build_layout(const spectra_config& cfg, const int32_t* widths, CodecDev* cd) {
  const int ng = cfg.rank / cfg.group;
  const int P = cfg.page_tokens, g = cfg.group;
  int64_t off = 0;
  int c_col = 0, wup = 0;
  int max_k = 0, max_v = 0, max_sec = 0;
  for (int a = 0; a < cfg.n_kv_heads; ++a) {
    HeadDev& hd = cd->head[a];
    std::memset(&hd, 0, sizeof(hd));
    hd.sec_off = (int32_t)off;
    for (int s = 0; s < 2; ++s) {
      SideDev& sd = hd.side[s];
      sd.c_col0 = c_col;
      sd.wup_off = wup;
      int kept = 0;
      for (int j = 0; j < ng; ++j) {
        const int b = widths[((size_t)a * 2 + s) * ng + j];
        if (b != 0 && b != 1 && b != 2 && b != 3 && b != 4 && b != 8) return 1;
        if (b == 0) continue;
        GroupDev& gd = sd.grp[sd.n_groups++];
        gd.b = b;
        gd.plane_off = (int32_t)off;
        off += (int64_t)b * P * g / 8;
        gd.sz_off = (int32_t)off;
        off += 4 * P;
        gd.col = kept;
        kept += g;
      }
      sd.n_kept = kept;
      c_col += kept;
      wup += kept * cfg.d_head;
      if (s == 0) max_k = std::max(max_k, kept);
      else max_v = std::max(max_v, kept);
    }
    hd.sec_bytes = (int32_t)(off - hd.sec_off);
    max_sec = std::max(max_sec, hd.sec_bytes);
    static const int kClassOrder[5] = {4, 2, 1, 3, 8};
    for (int s = 0; s < 2; ++s) {
      const SideDev& sd = hd.side[s];
      int n = 0;
      for (int ci = 0; ci < 5; ++ci) {
        hd.dec.cls[s][ci] = n;
        for (int j = 0; j < sd.n_groups && n < kDecMaxGroups; ++j) {
          const GroupDev& gd = sd.grp[j];
          if (gd.b != kClassOrder[ci]) continue;
          hd.dec.ord[s][n][0] = gd.plane_off - hd.sec_off;
          hd.dec.ord[s][n][1] = gd.sz_off - hd.sec_off;
          hd.dec.ord[s][n][2] = j;
          hd.dec.ord[s][n][3] = gd.b;
          ++n;
        }
      }
      for (int ci = 5; ci < 8; ++ci) hd.dec.cls[s][ci] = n;
    }
  }
  // a second copy of each K side's W_up, as rows [n_kept][d_head], after all the
  // per-side blocks (the decode's query fold reads it row by row)
  for (int a = 0; a < cfg.n_kv_heads; ++a) {
    cd->head[a].wupk_rows_off = wup;
    wup += cd->head[a].side[0].n_kept * cfg.d_head;
  }
  if (off > (int64_t)1 << 30) return 2;
  cd->d_model = cfg.d_model;
  cd->n_q = cfg.n_q_heads;
  cd->n_kv = cfg.n_kv_heads;
  cd->gq = cfg.n_q_heads / cfg.n_kv_heads;
  cd->d_h = cfg.d_head;
  cd->group = g;
  cd->P = P;
  cd->n_eff = c_col;
  cd->n_eff_pad = ((c_col + 127) / 128) * 128;
  if (cd->n_eff_pad == 0) cd->n_eff_pad = 128;
  cd->max_kept_k = max_k;
  cd->max_kept_v = max_v;
  cd->max_sec_bytes = max_sec;
  cd->page_bytes = off;
  return 0;
}

uint16_t f32_to_bf16_bits(float x) {
  uint32_t u;
  std::memcpy(&u, &x, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40);  // NaN stays NaN
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

float bf16_bits_to_f32(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float x;
  std::memcpy(&x, &u, 4);
  return x;
}

}  // namespace spectra

using namespace spectra;

extern "C" {

spectra_status spectra_allocate_widths(const double* sigma2, int32_t rank, int32_t group,
                                       int32_t budget_bits, int32_t count_overhead,
                                       int32_t* widths_out, double* distortion_out) {
  if (!sigma2 || !widths_out) return fail(SPECTRA_ERR_INVALID, "null pointer");
  if (group <= 0 || rank <= 0 || rank % group || budget_bits < 0 || budget_bits > (1 << 20))
    return fail(SPECTRA_ERR_INVALID, "bad rank/group/budget");
  for (int i = 0; i < rank; ++i)
    if (!std::isfinite(sigma2[i]) || sigma2[i] < 0) return fail(SPECTRA_ERR_NUMERIC, "sigma2 must be finite and >= 0");
  if (allocate_widths(sigma2, rank, group, budget_bits, count_overhead != 0, widths_out, distortion_out))
    return fail(SPECTRA_ERR_INVALID, "allocation failed");
  return SPECTRA_OK;
}

spectra_status spectra_allocate_widths_uniform(const double* sigma2, int32_t rank, int32_t group,
                                               int32_t n_eligible_groups, int32_t budget_bits,
                                               int32_t count_overhead, int32_t* widths_out,
                                               double* distortion_out) {
  if (!sigma2 || !widths_out) return fail(SPECTRA_ERR_INVALID, "null pointer");
  if (group <= 0 || rank <= 0 || rank % group || budget_bits < 0 || budget_bits > (1 << 20))
    return fail(SPECTRA_ERR_INVALID, "bad rank/group/budget");
  for (int i = 0; i < rank; ++i)
    if (!std::isfinite(sigma2[i]) || sigma2[i] < 0) return fail(SPECTRA_ERR_NUMERIC, "sigma2 must be finite and >= 0");
  if (allocate_widths_uniform(sigma2, rank, group, n_eligible_groups, budget_bits, count_overhead != 0,
                              widths_out, distortion_out))
    return fail(SPECTRA_ERR_INVALID, "allocation failed");
  return SPECTRA_OK;
}

spectra_status spectra_energy_rank(const double* sigma2, int32_t n, double threshold, int32_t* rank_out) {
  if (!sigma2 || !rank_out || n <= 0) return fail(SPECTRA_ERR_INVALID, "bad arguments");
  if (!(threshold > 0.0) || threshold > 1.0) return fail(SPECTRA_ERR_INVALID, "threshold must be in (0, 1]");
  for (int i = 0; i < n; ++i)
    if (!std::isfinite(sigma2[i]) || sigma2[i] < 0) return fail(SPECTRA_ERR_NUMERIC, "sigma2 must be finite and >= 0");
  int r = n;
  energy_rank(sigma2, n, threshold, &r);
  *rank_out = r;
  return SPECTRA_OK;
}

spectra_status spectra_water_fill(const double* sigma2, int32_t n, double rate_bits,
                                  double* theta_out, double* rates_out) {
  if (!sigma2 || !theta_out || n <= 0) return fail(SPECTRA_ERR_INVALID, "bad arguments");
  for (int i = 0; i < n; ++i)
    if (!std::isfinite(sigma2[i]) || sigma2[i] < 0) return fail(SPECTRA_ERR_NUMERIC, "sigma2 must be finite and >= 0");
  if (!std::isfinite(rate_bits)) return fail(SPECTRA_ERR_NUMERIC, "rate must be finite");
  if (water_fill(sigma2, n, rate_bits, theta_out, rates_out)) return fail(SPECTRA_ERR_INVALID, "water-fill failed");
  return SPECTRA_OK;
}

spectra_status spectra_sym_eigen(const double* M, int32_t n, double* vals, double* vecs) {
  if (!M || !vals || !vecs || n <= 0 || n > 512) return fail(SPECTRA_ERR_INVALID, "bad arguments");
  const int rc = sym_eigen(M, n, vals, vecs);
  if (rc == 2) return fail(SPECTRA_ERR_NUMERIC, "matrix has non-finite entries");
  if (rc) return fail(SPECTRA_ERR_NUMERIC, "Jacobi eigen solver did not converge");
  return SPECTRA_OK;
}

spectra_status spectra_page_layout(const spectra_config* cfg, const int32_t* widths,
                                   int64_t* page_bytes, int64_t* offsets) {
  if (!cfg || !widths || !page_bytes) return fail(SPECTRA_ERR_INVALID, "null pointer");
  std::string why;
  if (!valid_config(*cfg, &why)) return fail(SPECTRA_ERR_INVALID, why);
  CodecDev* cd = new CodecDev();
  const int rc = build_layout(*cfg, widths, cd);
  if (rc) {
    delete cd;
    return fail(SPECTRA_ERR_INVALID, rc == 1 ? "width must be one of 0,1,2,3,4,8" : "page too large");
  }
  *page_bytes = cd->page_bytes;
  if (offsets) {
    const int ng = cfg->rank / cfg->group;
    const size_t total = (size_t)cfg->n_kv_heads * 2 * ng;
    for (int a = 0; a < cfg->n_kv_heads; ++a)
      for (int s = 0; s < 2; ++s) {
        int k = 0;
        for (int j = 0; j < ng; ++j) {
          const size_t idx = ((size_t)a * 2 + s) * ng + j;
          if (widths[idx] == 0) {
            offsets[idx] = -1;
            offsets[total + idx] = -1;
          } else {
            offsets[idx] = cd->head[a].side[s].grp[k].plane_off;
            offsets[total + idx] = cd->head[a].side[s].grp[k].sz_off;
            ++k;
          }
        }
      }
  }
  delete cd;
  return SPECTRA_OK;
}

const char* spectra_last_error(void) { return g_last_error.c_str(); }

int32_t spectra_abi_version(void) { return SPECTRA_ABI_VERSION; }

}  // extern "C"
