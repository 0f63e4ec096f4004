// Host-only exports: status strings, S-CAS finalisation and the static
// keep-schedule builder.
//
// [HeatKV] project page, Abstract and Method steps 3-4: head-scale pairs are
// ranked by S-CAS and the lowest-ranked are removed until the user's memory
// budget holds, the early sink scales always retained; the schedule is built
// once, offline, before inference.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <climits>
#include <cstring>
#include <vector>

#include "vark.h"

extern "C" const char* vark_status_string(int status) {
  switch (status) {
    case VARK_OK: return "VARK_OK";
    case VARK_E_ARG: return "VARK_E_ARG: invalid argument";
    case VARK_E_SHAPE: return "VARK_E_SHAPE: unsupported shape";
    case VARK_E_ALIGN: return "VARK_E_ALIGN: pointer or stride not 16-byte aligned";
    case VARK_E_BUDGET: return "VARK_E_BUDGET: sink scales alone exceed the budget";
    case VARK_E_CUDA: return "VARK_E_CUDA: CUDA call failed";
    case VARK_E_TIMEOUT: return "VARK_E_TIMEOUT: a bounded device wait gave up";
    case VARK_E_DEVICE: return "VARK_E_DEVICE: current device is not sm_100";
    default: return "VARK: unknown status";
  }
}

extern "C" int vark_version(void) { return 10000; }

static bool sides_ok(int S, const int32_t* sides, int64_t* T_out) {
  if (S < 1 || S > VARK_MAX_SCALES || sides == nullptr) return false;
  int64_t T = 0;
  for (int s = 0; s < S; ++s) {
    if (sides[s] < 1 || sides[s] > 4096) return false;
    T += int64_t(sides[s]) * sides[s];
  }
  if (T > (int64_t(1) << 30)) return false;
  *T_out = T;
  return true;
}

// The budget test compares kept * 10000 with budget_bp * F in int64, with
// F = (L * H) * T tokens: both sides stay below 2^63 when F <= INT64_MAX / 10000.
static bool budget_fits_int64(int64_t LH, int64_t T) {
  return LH >= 1 && T >= 1 && LH <= INT64_MAX / 10000 / T;
}

extern "C" int vark_scas_finalize(const float* mass, int L, int H, int S, int n_calls, double* scas) {
  if (mass == nullptr || scas == nullptr || n_calls < 1) return VARK_E_ARG;
  if (L < 1 || H < 1 || S < 1 || S > VARK_MAX_SCALES) return VARK_E_SHAPE;
  const double inv = 1.0 / double(n_calls);
  for (int64_t lh = 0; lh < int64_t(L) * H; ++lh) {
    const float* M = mass + lh * S * S;           // [s][k]
    for (int s = 0; s < S; ++s) {
      double acc = 0.0;
      for (int k = s + 1; k < S; ++k) acc += double(M[s * S + k]);
      scas[lh * S + s] = acc * inv;
    }
  }
  return VARK_OK;
}

namespace {
struct Candidate {
  double score;
  int32_t l, h, s;
};
}  // namespace

extern "C" int vark_build_schedule(const double* scas, int L, int H, int S, const int32_t* sides,
                                   uint32_t budget_bp, int n_sinks, uint8_t* keep) {
  if (scas == nullptr || keep == nullptr || sides == nullptr) return VARK_E_ARG;
  if (budget_bp > 10000u || n_sinks < 0) return VARK_E_ARG;
  int64_t T = 0;
  if (L < 1 || H < 1 || !sides_ok(S, sides, &T) || n_sinks > S) return VARK_E_SHAPE;
  if (int64_t(L) * H > (int64_t(1) << 24)) return VARK_E_SHAPE;
  if (!budget_fits_int64(int64_t(L) * H, T)) return VARK_E_SHAPE;
  const int64_t LHS = int64_t(L) * H * S;
  for (int64_t i = 0; i < LHS; ++i)
    if (!std::isfinite(scas[i])) return VARK_E_ARG;

  std::vector<int64_t> n(S);
  int64_t sink_per_head = 0;
  for (int s = 0; s < S; ++s) {
    n[s] = int64_t(sides[s]) * sides[s];
    if (s < n_sinks) sink_per_head += n[s];
  }
  const int64_t F = int64_t(L) * H * T;               // full cache, tokens
  const int64_t budget = int64_t(budget_bp);
  int64_t kept = F;
  if (kept * 10000 <= budget * F) {
    std::memset(keep, 1, size_t(LHS));
    return VARK_OK;
  }
  if (int64_t(L) * H * sink_per_head * 10000 > budget * F) return VARK_E_BUDGET;

  std::vector<Candidate> cand;
  cand.reserve(size_t(int64_t(L) * H * (S - n_sinks)));
  for (int l = 0; l < L; ++l)
    for (int h = 0; h < H; ++h)
      for (int s = n_sinks; s < S; ++s)
        cand.push_back({scas[(int64_t(l) * H + h) * S + s], l, h, s});
  // Ascending (score, l, h, s): the index tie-break makes the order total.
  std::sort(cand.begin(), cand.end(), [](const Candidate& a, const Candidate& b) {
    if (a.score != b.score) return a.score < b.score;
    if (a.l != b.l) return a.l < b.l;
    if (a.h != b.h) return a.h < b.h;
    return a.s < b.s;
  });
  std::memset(keep, 1, size_t(LHS));
  for (const Candidate& c : cand) {
    keep[(int64_t(c.l) * H + c.h) * S + c.s] = 0;
    kept -= n[c.s];
    if (kept * 10000 <= budget * F) break;
  }
  return VARK_OK;
}

extern "C" int vark_cache_size_after_layer(const uint8_t* keep, int L, int H, int S, const int32_t* sides, int B,
                                           int D, int64_t* bytes) {
  if (keep == nullptr || bytes == nullptr || sides == nullptr) return VARK_E_ARG;
  int64_t T = 0;
  if (L < 1 || H < 1 || B < 1 || D < 1 || !sides_ok(S, sides, &T)) return VARK_E_SHAPE;
  // every byte count is at most L * H * T * B * D * 4, which must fit int64
  if (int64_t(L) * H > INT64_MAX / T / (int64_t(B) * D * 4)) return VARK_E_SHAPE;
  int64_t total = 0;
  const int64_t per_token = int64_t(B) * D * 2 * 2;   // K and V, bf16
  for (int k = 0; k < S; ++k) {
    const int64_t n = int64_t(sides[k]) * sides[k];
    for (int l = 0; l < L; ++l) {
      int64_t kept_heads = 0;
      for (int h = 0; h < H; ++h) kept_heads += keep[(int64_t(l) * H + h) * S + k] ? 1 : 0;
      const int64_t add = kept_heads * n * per_token;
      total += add;
      bytes[int64_t(k) * L + l] = total;
    }
  }
  return VARK_OK;
}

// Average ranks (1-based) of v, ties sharing the mean of their positions.
static void average_ranks(const std::vector<double>& v, std::vector<double>& rank) {
  const size_t n = v.size();
  std::vector<size_t> idx(n);
  for (size_t i = 0; i < n; ++i) idx[i] = i;
  std::stable_sort(idx.begin(), idx.end(), [&](size_t a, size_t b) { return v[a] < v[b]; });
  rank.assign(n, 0.0);
  for (size_t i = 0; i < n;) {
    size_t j = i;
    while (j + 1 < n && v[idx[j + 1]] == v[idx[i]]) ++j;
    const double r = 0.5 * double(i + j) + 1.0;
    for (size_t t = i; t <= j; ++t) rank[idx[t]] = r;
    i = j + 1;
  }
}

extern "C" int vark_rank_stability(const double* scas_a, const double* scas_b, int L, int H, int S,
                                   const int32_t* sides, uint32_t budget_bp, int n_sinks, double* spearman,
                                   double* drop_jaccard) {
  if (!scas_a || !scas_b || !sides || !spearman || !drop_jaccard) return VARK_E_ARG;
  int64_t T = 0;
  if (L < 1 || H < 1 || !sides_ok(S, sides, &T) || n_sinks < 0 || n_sinks >= S) return VARK_E_SHAPE;
  if (int64_t(L) * H > (int64_t(1) << 24) || !budget_fits_int64(int64_t(L) * H, T)) return VARK_E_SHAPE;
  std::vector<double> a, b;
  for (int l = 0; l < L; ++l)
    for (int h = 0; h < H; ++h)
      for (int s = n_sinks; s < S; ++s) {
        const int64_t i = (int64_t(l) * H + h) * S + s;
        if (!std::isfinite(scas_a[i]) || !std::isfinite(scas_b[i])) return VARK_E_ARG;
        a.push_back(scas_a[i]);
        b.push_back(scas_b[i]);
      }
  std::vector<double> ra, rb;
  average_ranks(a, ra);
  average_ranks(b, rb);
  const double n = double(ra.size());
  double ma = 0, mb = 0;
  for (size_t i = 0; i < ra.size(); ++i) { ma += ra[i]; mb += rb[i]; }
  ma /= n; mb /= n;
  double sab = 0, saa = 0, sbb = 0;
  for (size_t i = 0; i < ra.size(); ++i) {
    sab += (ra[i] - ma) * (rb[i] - mb);
    saa += (ra[i] - ma) * (ra[i] - ma);
    sbb += (rb[i] - mb) * (rb[i] - mb);
  }
  *spearman = (saa > 0 && sbb > 0) ? sab / std::sqrt(saa * sbb) : 0.0;
  std::vector<uint8_t> ka(size_t(int64_t(L) * H * S)), kb(ka.size());
  int rc = vark_build_schedule(scas_a, L, H, S, sides, budget_bp, n_sinks, ka.data());
  if (rc) return rc;
  rc = vark_build_schedule(scas_b, L, H, S, sides, budget_bp, n_sinks, kb.data());
  if (rc) return rc;
  int64_t inter = 0, uni = 0;
  for (size_t i = 0; i < ka.size(); ++i) {
    const bool da = ka[i] == 0, db = kb[i] == 0;
    inter += (da && db) ? 1 : 0;
    uni += (da || db) ? 1 : 0;
  }
  *drop_jaccard = uni > 0 ? double(inter) / double(uni) : 1.0;
  return VARK_OK;
}

extern "C" int vark_build_early_pruning_schedule(const double* scas, int L, int H, int S, const int32_t* sides,
                                                 uint32_t budget_bp, int n_sinks, int32_t* prefix_len,
                                                 uint8_t* evict_step) {
  if (scas == nullptr || sides == nullptr || prefix_len == nullptr || evict_step == nullptr) return VARK_E_ARG;
  if (budget_bp > 10000u || n_sinks < 0) return VARK_E_ARG;
  int64_t T = 0;
  if (L < 1 || H < 1 || !sides_ok(S, sides, &T) || n_sinks > S || S > 254) return VARK_E_SHAPE;
  // prefix lengths are int32; the budget arithmetic stays in int64
  if (int64_t(L) * H > INT32_MAX || !budget_fits_int64(int64_t(L) * H, T)) return VARK_E_SHAPE;
  const int64_t LH = int64_t(L) * H;
  const int64_t LHS = LH * S;
  for (int64_t i = 0; i < LHS; ++i)
    if (!std::isfinite(scas[i])) return VARK_E_ARG;
  // Absolute budget in tokens: budget_bp / 10000 of the final full cache.
  const int64_t F = LH * T;
  const int64_t budget = int64_t(budget_bp);
  int64_t sink_tokens = 0;
  for (int s = 0; s < n_sinks; ++s) sink_tokens += LH * int64_t(sides[s]) * sides[s];
  if (sink_tokens * 10000 > budget * F) return VARK_E_BUDGET;
  // rank[i][(l, h)] = position of (l, h) in O_i: ascending (scas[l][h][i], l, h)
  std::vector<int64_t> rank(size_t(LH) * S, 0);
  std::vector<int64_t> order(static_cast<size_t>(LH));
  for (int i = n_sinks; i < S; ++i) {
    for (int64_t lh = 0; lh < LH; ++lh) order[size_t(lh)] = lh;
    std::sort(order.begin(), order.end(), [&](int64_t a, int64_t b) {
      const double va = scas[a * S + i], vb = scas[b * S + i];
      if (va != vb) return va < vb;
      return a < b;
    });
    for (int64_t pos = 0; pos < LH; ++pos) rank[size_t(i) * LH + order[size_t(pos)]] = pos;
  }
  // N_k: smallest prefix length (non-decreasing in k) whose retained cache
  // after step k, sinks + (LH - N_k) heads of every non-sink scale <= k, fits.
  int64_t N = 0;
  for (int k = 0; k < S; ++k) {
    int64_t nonsink = 0;
    for (int i = n_sinks; i <= k; ++i) nonsink += int64_t(sides[i]) * sides[i];
    int64_t sinks_k = 0;
    for (int i = 0; i < n_sinks && i <= k; ++i) sinks_k += LH * int64_t(sides[i]) * sides[i];
    while (N < LH && (sinks_k + (LH - N) * nonsink) * 10000 > budget * F) ++N;
    prefix_len[k] = int32_t(nonsink > 0 ? N : 0);
  }
  // evict_step[l][h][i]: first step k >= i with rank_i(l, h) < N_k; 255 = kept to the end
  for (int64_t lh = 0; lh < LH; ++lh)
    for (int i = 0; i < S; ++i) {
      uint8_t e = 255;
      if (i >= n_sinks)
        for (int k = i; k < S; ++k)
          if (rank[size_t(i) * LH + lh] < prefix_len[k]) {
            e = uint8_t(k);
            break;
          }
      evict_step[lh * S + i] = e;
    }
  return VARK_OK;
}
