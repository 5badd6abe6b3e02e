// TokenGate gated-prefill path: plain fp64 CPU oracle.
//
// TEST INFRASTRUCTURE. Only the tests, the smoke check and the bench's CPU
// baseline leg load this library. It shares no code with the CUDA path: no
// header, helper, table or constant comes from there, and the CUDA path never
// calls it.
//
// Sources: "TokenGate: l'attention gérée par des tokens ..." (MarkTechPost, French
// translation), sections "Comment TokenGate a-t-il appris le fonctionnement de la
// réduction des tokens ?" (the three-phase forward pass: gate MLP on the
// post-attention residual at layer L, top-K selector, layers above L see only the
// K kept tokens; only the document may be dropped, never the question),
// "Qu'est-ce que l'attention gérée par des tokens ?" (each kept token's score is
// a bias on the attention logits, with a learnable per-head gain and a learnable
// per-head temperature) and "Comment déployer TokenGate ?" (the {state}
// placeholder marks the droppable document; the budget max_kept_prefill_tokens).
//
// Every function is the plain definition of its step, written out as loops in
// double precision. Readings where the pages are silent:
//   * gate MLP = two layers d -> h -> 1 with biases and exact (erf) GELU;
//   * the score is the raw MLP output, used both for ranking and as the bias;
//   * the temperature divides the q.k term only: z = q.k / (sqrt(dh) tau) + g s;
//   * ties go to the lower position, -0 equals +0, NaN ranks below -inf;
//   * every token outside [doc_begin, doc_end) is kept;
//   * query head hq reads KV head hq / (Hq / Hkv);
//   * key j is visible to query i iff j <= i in the (position-ordered) kept list.
//   * the kept tokens' q/k/v projections use the rotary embedding of the Qwen
//     models the pages evaluate (rotate-half pairing, base given by the caller),
//     applied at each token's original position (the pages do not describe it).
// Parity status: gate, select, gather, attention and the q/k/v projection are each
// pinned by tests (closed forms, brute force, library witnesses, invariants); see
// tests/.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// exact widening of the two input storage types
double load_elem(const void* p, int dtype, int64_t i) {
  if (dtype == 0) return (double)((const float*)p)[i];
  uint32_t u = ((uint32_t)((const uint16_t*)p)[i]) << 16;  // bf16 = top half of an f32
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

double gelu(double u) { return 0.5 * u * (1.0 + std::erf(u / std::sqrt(2.0))); }

// total order used by the selector: larger is better; NaN is the worst value and
// -0 is the same value as +0.
struct ScoreKey {
  bool nan;
  double v;
};
ScoreKey score_key(float f) {
  ScoreKey k;
  k.nan = std::isnan(f);
  k.v = k.nan ? 0.0 : (f == 0.0f ? 0.0 : (double)f);
  return k;
}
bool ranks_higher(const ScoreKey& a, const ScoreKey& b) {  // strictly better
  if (a.nan != b.nan) return b.nan;
  if (a.nan) return false;
  return a.v > b.v;
}

}  // namespace

extern "C" {

int oracle_version() { return 1; }

// Gate MLP scorer (section "Comment TokenGate a-t-il appris ...": a small MLP
// scores every token from its residual at layer L):
//   s_i = b2 + sum_k w2[k] * GELU(b1[k] + sum_c x[i,c] * w1[k,c])
// x [n, d] and w1 [h, d] (out x in) in `dtype` (0 = f32, 1 = bf16 bits), b1, w2
// f32, b2 f32. Writes the fp64 value and its fp32 rounding.
void oracle_gate_score(const void* x, int dtype, int64_t n, int d, const void* w1,
                       const float* b1, const float* w2, float b2, int h, double* s64,
                       float* s32) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    double s = (double)b2;
    for (int k = 0; k < h; ++k) {
      double u = (double)b1[k];
      for (int c = 0; c < d; ++c)
        u += load_elem(x, dtype, i * (int64_t)d + c) * load_elem(w1, dtype, (int64_t)k * d + c);
      s += (double)w2[k] * gelu(u);
    }
    if (s64) s64[i] = s;
    if (s32) s32[i] = (float)s;
  }
}

// Top-K with question protection (sections "Comment TokenGate a-t-il appris ..."
// and "Comment déployer TokenGate ?"): for sequence b with tokens
// [cu_seqlens[b], cu_seqlens[b+1]) and droppable span [doc_begin[b], doc_end[b])
// (local positions), keep the min(k_doc[b], span length) span tokens of highest
// score (ties to the lower position) and every token outside the span. Writes the
// kept tokens' global row ids in ascending order and cu_kept[b+1] = running
// total. Returns the total kept, or -1 on a bad span.
int64_t oracle_select_topk(const float* scores, const int32_t* cu_seqlens,
                           const int32_t* doc_begin, const int32_t* doc_end,
                           const int32_t* k_doc, int batch, int32_t* kept_idx,
                           int32_t* cu_kept) {
  int64_t out = 0;
  if (cu_kept) cu_kept[0] = 0;
  for (int b = 0; b < batch; ++b) {
    const int32_t base = cu_seqlens[b];
    const int32_t len = cu_seqlens[b + 1] - base;
    const int32_t db = doc_begin[b], de = doc_end[b];
    if (db < 0 || de < db || de > len) return -1;
    std::vector<int32_t> doc;
    for (int32_t p = db; p < de; ++p) doc.push_back(p);
    // best first; stable_sort keeps equal scores in ascending position order
    std::stable_sort(doc.begin(), doc.end(), [&](int32_t a, int32_t c) {
      return ranks_higher(score_key(scores[base + a]), score_key(scores[base + c]));
    });
    int64_t take = std::min<int64_t>(std::max<int32_t>(k_doc[b], 0), (int64_t)doc.size());
    std::vector<char> keep(len, 1);
    for (int32_t p = db; p < de; ++p) keep[p] = 0;
    for (int64_t r = 0; r < take; ++r) keep[doc[r]] = 1;
    for (int32_t p = 0; p < len; ++p)
      if (keep[p]) {
        if (kept_idx) kept_idx[out] = base + p;
        ++out;
      }
    if (cu_kept) cu_kept[b + 1] = (int32_t)out;
  }
  return out;
}

// Stable compaction (section "Comment TokenGate a-t-il appris ...": layers above L
// process only the K kept tokens): dst[r] = src[kept_idx[r]], row_bytes bytes per
// row.
void oracle_gather_rows(const void* src, int64_t row_bytes, const int32_t* kept_idx,
                        int64_t n_kept, void* dst) {
  for (int64_t r = 0; r < n_kept; ++r)
    std::memcpy((char*)dst + r * row_bytes, (const char*)src + (int64_t)kept_idx[r] * row_bytes,
                (size_t)row_bytes);
}

// Token-gated causal GQA attention over the kept tokens (section "Qu'est-ce que
// l'attention gérée par des tokens ?"): for sequence b (kept rows
// [cu_kept[b], cu_kept[b+1])), query head hq, kept query row i:
//   z_j = (q_i . k_j) / (sqrt(dh) * tau[hq]) + gain[hq] * s_kept[j],  j <= i
//   O_i = sum_j softmax_j(z) v_j
// q [K, hq, dh], k/v [K, hkv, dh] in `dtype`; KV head = hq / (n_hq / n_hkv).
// `rows` (n_rows global kept rows) restricts the computation to those query rows;
// rows == nullptr computes all. out is [K, hq, dh] fp64; only computed rows are
// written.
void oracle_gated_attention(const void* q, const void* k, const void* v, int dtype,
                            const float* s_kept, const float* gain, const float* tau,
                            const int32_t* cu_kept, int batch, int n_hq, int n_hkv, int dh,
                            const int32_t* rows, int64_t n_rows, double* out) {
  const int64_t total = cu_kept[batch];
  std::vector<int32_t> all;
  if (!rows) {
    for (int64_t r = 0; r < total; ++r) all.push_back((int32_t)r);
    rows = all.data();
    n_rows = total;
  }
  const int group = n_hq / n_hkv;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
  for (int64_t t = 0; t < n_rows; ++t) {
    for (int hq = 0; hq < n_hq; ++hq) {
      const int64_t i = rows[t];
      int b = 0;
      while (cu_kept[b + 1] <= i) ++b;
      const int64_t j0 = cu_kept[b];
      const int kv = hq / group;
      const double scale = 1.0 / (std::sqrt((double)dh) * (double)tau[hq]);
      std::vector<double> z(i - j0 + 1);
      double zmax = -INFINITY;
      for (int64_t j = j0; j <= i; ++j) {
        double dot = 0.0;
        for (int c = 0; c < dh; ++c)
          dot += load_elem(q, dtype, (i * n_hq + hq) * (int64_t)dh + c) *
                 load_elem(k, dtype, (j * n_hkv + kv) * (int64_t)dh + c);
        double zj = dot * scale + (double)gain[hq] * (double)s_kept[j];
        z[j - j0] = zj;
        zmax = std::max(zmax, zj);
      }
      double denom = 0.0;
      std::vector<double> acc(dh, 0.0);
      for (int64_t j = j0; j <= i; ++j) {
        double w = std::exp(z[j - j0] - zmax);
        denom += w;
        for (int c = 0; c < dh; ++c) acc[c] += w * load_elem(v, dtype, (j * n_hkv + kv) * (int64_t)dh + c);
      }
      for (int c = 0; c < dh; ++c) out[(i * n_hq + hq) * (int64_t)dh + c] = acc[c] / denom;
    }
  }
}

// The kept tokens' projections for the layers above the gate layer (only the K
// kept tokens get a KV-cache entry: MarkTechPost page, section "Comment TokenGate
// a-t-il appris le fonctionnement de la réduction des tokens ?"). Plain definition:
//   y[r] = W xc[r]            W = [Wq; Wk; Wv] of shape [(hq + 2 hkv) dh, d]
// split per head into q [n, hq, dh], k [n, hkv, dh], v [n, hkv, dh]; q and k heads
// are rotated at the token's ORIGINAL position p = pos[r] (rotary embedding,
// rotate-half pairing): for i < dh/2, theta_i = base^(-2i/dh), a = p theta_i,
//   out[i]        = y[i] cos a - y[i + dh/2] sin a
//   out[i + dh/2] = y[i + dh/2] cos a + y[i] sin a
// v is not rotated. Rows listed in `rows` (all rows when rows == nullptr) are
// computed; the others are left untouched.
void oracle_qkv_rope(const void* xc, int dtype, int64_t n, int d, const void* w, int hq,
                     int hkv, int dh, double base, const int32_t* pos, const int32_t* rows,
                     int64_t n_sel, double* q, double* k, double* v) {
  const int nh = hq + 2 * hkv;
  const int64_t cnt = rows ? n_sel : n;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t s = 0; s < cnt; ++s) {
    const int64_t r = rows ? rows[s] : s;
    std::vector<double> y((size_t)nh * dh);
    for (int o = 0; o < nh * dh; ++o) {
      double acc = 0.0;
      for (int c = 0; c < d; ++c)
        acc += load_elem(w, dtype, (int64_t)o * d + c) * load_elem(xc, dtype, r * d + c);
      y[o] = acc;
    }
    for (int h = 0; h < nh; ++h) {
      const double* yh = &y[(size_t)h * dh];
      double* out = h < hq ? q + (r * hq + h) * dh
                  : h < hq + hkv ? k + (r * hkv + (h - hq)) * dh
                                 : v + (r * hkv + (h - hq - hkv)) * dh;
      if (h >= hq + hkv) {   // value heads: no rotation
        for (int i = 0; i < dh; ++i) out[i] = yh[i];
        continue;
      }
      const int half = dh / 2;
      for (int i = 0; i < half; ++i) {
        const double theta = std::pow(base, -2.0 * i / dh);
        const double a = (double)pos[r] * theta;
        const double c = std::cos(a), sn = std::sin(a);
        out[i] = yh[i] * c - yh[i + half] * sn;
        out[i + half] = yh[i + half] * c + yh[i] * sn;
      }
    }
  }
}

// Backward of the token-gated attention (MarkTechPost page, section "Qu'est-ce que
// l'attention gérée par des tokens ?": the key score is a logit bias precisely so
// that gradients reach the scorer; the gain and the temperature are learned).
// Given dO = dL/dO for the forward above, for sequence b, query head hq (KV head
// kv), kept rows i and keys j <= i, with c = 1 / (sqrt(dh) tau[hq]):
//   z_ij = c q_i.k_j + gain s_j,  P_ij = softmax_j(z_ij),  dP_ij = dO_i . v_j
//   D_i = sum_j P_ij dP_ij,       dZ_ij = P_ij (dP_ij - D_i)
//   dq_i += c sum_j dZ_ij k_j     dk_j += c dZ_ij q_i      dv_j += P_ij dO_i
//   ds_j += gain dZ_ij            dgain += dZ_ij s_j
//   dtau += dZ_ij dz_ij/dtau = dZ_ij (-(q_i.k_j) / (sqrt(dh) tau^2))
// (dk, dv and ds sum over every query head that reads the key; dgain and dtau are
// per query head). q, k, v, dout in `dtype`; every output fp64 and overwritten.
void oracle_gated_attention_bwd(const void* q, const void* k, const void* v, const void* dout,
                                int dtype, const float* s_kept, const float* gain,
                                const float* tau, const int32_t* cu_kept, int batch, int n_hq,
                                int n_hkv, int dh, double* dq, double* dk, double* dv,
                                double* ds, double* dgain, double* dtau) {
  const int64_t total = cu_kept[batch];
  const int group = n_hq / n_hkv;
  for (int64_t t = 0; t < total * n_hq * dh; ++t) dq[t] = 0.0;
  for (int64_t t = 0; t < total * n_hkv * dh; ++t) dk[t] = dv[t] = 0.0;
  for (int64_t t = 0; t < total; ++t) ds[t] = 0.0;
  for (int h = 0; h < n_hq; ++h) dgain[h] = dtau[h] = 0.0;
  auto at = [&](const void* p, int64_t row, int nh, int h, int c) {
    return load_elem(p, dtype, (row * nh + h) * (int64_t)dh + c);
  };
  for (int b = 0; b < batch; ++b) {
    const int64_t j0 = cu_kept[b], j1 = cu_kept[b + 1];
    for (int hq = 0; hq < n_hq; ++hq) {
      const int kv = hq / group;
      const double g = (double)gain[hq], tq = (double)tau[hq];
      const double c = 1.0 / (std::sqrt((double)dh) * tq);
      for (int64_t i = j0; i < j1; ++i) {
        const int64_t n = i - j0 + 1;
        std::vector<double> qk(n), z(n), p(n), dp(n);
        double zmax = -INFINITY;
        for (int64_t j = j0; j <= i; ++j) {
          double dot = 0.0;
          for (int e = 0; e < dh; ++e) dot += at(q, i, n_hq, hq, e) * at(k, j, n_hkv, kv, e);
          qk[j - j0] = dot;
          z[j - j0] = c * dot + g * (double)s_kept[j];
          zmax = std::max(zmax, z[j - j0]);
        }
        double den = 0.0;
        for (int64_t u = 0; u < n; ++u) den += (p[u] = std::exp(z[u] - zmax));
        for (int64_t u = 0; u < n; ++u) p[u] /= den;
        double D = 0.0;
        for (int64_t j = j0; j <= i; ++j) {
          double dot = 0.0;
          for (int e = 0; e < dh; ++e) dot += at(dout, i, n_hq, hq, e) * at(v, j, n_hkv, kv, e);
          dp[j - j0] = dot;
          D += p[j - j0] * dot;
        }
        for (int64_t j = j0; j <= i; ++j) {
          const int64_t u = j - j0;
          const double dz = p[u] * (dp[u] - D);
          for (int e = 0; e < dh; ++e) {
            dq[(i * n_hq + hq) * dh + e] += c * dz * at(k, j, n_hkv, kv, e);
            dk[(j * n_hkv + kv) * dh + e] += c * dz * at(q, i, n_hq, hq, e);
            dv[(j * n_hkv + kv) * dh + e] += p[u] * at(dout, i, n_hq, hq, e);
          }
          ds[j] += g * dz;
          dgain[hq] += dz * (double)s_kept[j];
          dtau[hq] += dz * (-qk[u] / (std::sqrt((double)dh) * tq * tq));
        }
      }
    }
  }
}

// Gated delta rule over the kept tokens (MarkTechPost page, section "Est-ce que cela
// fonctionne avec les modèles d'attention hybrides ?" and its comparison table: the
// hybrid model's Gated DeltaNet layers are pruned too, i.e. above the gate layer
// they run over the kept tokens only). For each sequence and head, a state
// S in R^{dk x dv} starts at zero and, for the sequence's tokens t in order,
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
//   o_t = S_t^T q_t
// q, k [total, H, dk], v [total, H, dv] in `dtype`; alpha, beta [total, H] f32;
// out [total, H, dv] fp64.
void oracle_gated_delta_rule(const void* q, const void* k, const void* v, int dtype,
                             const float* alpha, const float* beta, const int32_t* cu_seqlens,
                             int batch, int n_heads, int dk, int dv, double* out) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int b = 0; b < batch; ++b) {
    for (int h = 0; h < n_heads; ++h) {
      std::vector<double> S((size_t)dk * dv, 0.0), kt(dk), qt(dk), vt(dv), ks(dv);
      for (int64_t t = cu_seqlens[b]; t < cu_seqlens[b + 1]; ++t) {
        for (int i = 0; i < dk; ++i) {
          kt[i] = load_elem(k, dtype, (t * n_heads + h) * (int64_t)dk + i);
          qt[i] = load_elem(q, dtype, (t * n_heads + h) * (int64_t)dk + i);
        }
        for (int c = 0; c < dv; ++c) vt[c] = load_elem(v, dtype, (t * n_heads + h) * (int64_t)dv + c);
        const double a = alpha[t * n_heads + h], be = beta[t * n_heads + h];
        // ks = k_t^T S_{t-1}
        for (int c = 0; c < dv; ++c) {
          double acc = 0.0;
          for (int i = 0; i < dk; ++i) acc += kt[i] * S[(size_t)i * dv + c];
          ks[c] = acc;
        }
        // S_t = a (S - be k (k^T S)) + be k v^T
        for (int i = 0; i < dk; ++i)
          for (int c = 0; c < dv; ++c)
            S[(size_t)i * dv + c] = a * (S[(size_t)i * dv + c] - be * kt[i] * ks[c]) + be * kt[i] * vt[c];
        // o_t = S_t^T q_t
        for (int c = 0; c < dv; ++c) {
          double acc = 0.0;
          for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + c] * qt[i];
          out[(t * n_heads + h) * (int64_t)dv + c] = acc;
        }
      }
    }
  }
}

// Decode over the compacted cache (MarkTechPost page, section "Comment déployer
// TokenGate ?": generation runs on the cache the pruned prefill left behind, with
// max_kept_prefill_tokens bounding it; section "Qu'est-ce que l'attention gérée
// par des tokens ?" for the logits). One new query row per sequence b attends
// over that sequence's cache rows j < cache_len[b] (the new token's own row is in
// the cache already, so the causal rule "key position <= query position" keeps
// every cached row):
//   z_j = (q_b . k_j) / (sqrt(dh) * tau[hq]) + gain[hq] * s_j,  O_b = sum_j softmax_j(z) v_j
// q [B, hq, dh]; k/v cache [B, cap, hkv, dh] in `dtype`; s cache [B, cap] f32;
// KV head = hq / (n_hq / n_hkv). out [B, hq, dh] fp64. A sequence with an empty
// cache gets zeros.
void oracle_gated_decode(const void* q, const void* kc, const void* vc, int dtype,
                         const float* sc, const int32_t* cache_len, int batch, int cap,
                         int n_hq, int n_hkv, int dh, const float* gain, const float* tau,
                         double* out) {
  const int group = n_hq / n_hkv;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < batch; ++b) {
    for (int hq = 0; hq < n_hq; ++hq) {
      const int kv = hq / group;
      const int64_t n = cache_len[b];
      double* o = out + ((int64_t)b * n_hq + hq) * dh;
      for (int c = 0; c < dh; ++c) o[c] = 0.0;
      if (n <= 0) continue;
      const double scale = 1.0 / (std::sqrt((double)dh) * (double)tau[hq]);
      std::vector<double> z(n);
      double zmax = -INFINITY;
      for (int64_t j = 0; j < n; ++j) {
        const int64_t row = ((int64_t)b * cap + j) * n_hkv + kv;
        double dot = 0.0;
        for (int c = 0; c < dh; ++c)
          dot += load_elem(q, dtype, ((int64_t)b * n_hq + hq) * dh + c) *
                 load_elem(kc, dtype, row * dh + c);
        z[j] = dot * scale + (double)gain[hq] * (double)sc[(int64_t)b * cap + j];
        zmax = std::max(zmax, z[j]);
      }
      double denom = 0.0;
      for (int64_t j = 0; j < n; ++j) {
        const double w = std::exp(z[j] - zmax);
        denom += w;
        const int64_t row = ((int64_t)b * cap + j) * n_hkv + kv;
        for (int c = 0; c < dh; ++c) o[c] += w * load_elem(vc, dtype, row * dh + c);
      }
      for (int c = 0; c < dh; ++c) o[c] /= denom;
    }
  }
}

}  // extern "C"
