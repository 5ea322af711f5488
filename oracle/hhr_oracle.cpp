// TEST INFRASTRUCTURE ONLY -- not part of the product path.
//
// A plain, slow, single-threaded CPU oracle for the decode-time retrieval path
// of "HHR: Hierarchical Hash Retrieval for Efficient LLM Generation"
// (arXiv 2610.01230).  Only the test suite, the package smoke check and the
// benchmark's CPU-baseline / reference arm may load it.  It shares no code,
// header, table or helper with the CUDA library, and the CUDA library never
// loads it.
//
// Conventions
//  * bf16 values arrive as raw uint16 bit patterns and are widened exactly.
//  * Every sum is carried in double, in index order.  A value that the method
//    stores in float32 is rounded once, to nearest even.
//  * Row-vector convention of §3.3.1 Eq. 4: the rotated key is k~ = k R, i.e.
//    k~[j] = sum_i k[i] R[i][j].  Projection of §3.3.2 Eq. 10: z = x W, i.e.
//    z[t] = sum_i x[i] W[i][t].
//  * Page p of a (sequence, KV head) covers tokens [p*S, min((p+1)*S, n)) of
//    the n valid keys (§3.3.1: keys are split into non-overlapping pages).
//
// Readings where the paper leaves a step open (each is restated where used):
//  R1  Page metadata is stored as bf16: the minimum rounded toward -inf, the
//      maximum toward +inf, so that Eq. 3 remains an upper bound.
//  R2  The sign of a projection that is exactly zero is taken as bit 0.
//  R3  W applies to the unrotated key/query (§3.3.2 defines z = x W on keys).
//  R4  GQA: a KV head g serves query heads G(g) = {g*r, ..., g*r + r - 1}; the
//      page score is the max over G(g) of Eq. 3 and the token distance is the
//      min over G(g) of Eq. 2 ("kept if useful to any head of the group").
//  R5  The threshold c_h of §3.3.1 is realised as a fixed page budget P (the
//      paper's "candidate budget", Appendix A); ties go to the lower page index.
//  R6  Token selection keeps the k smallest distances (Top-K ratio of §4.1);
//      ties go to the lower token index.  No sink/local tokens are forced in.
//  R7  Attention over the selected keys is softmax(scale * q.k) V with the
//      original (unrotated) keys; Eq. 4 shows the logits are unchanged by R.
// Variants (flags of the *_v / *_f32 / *_agg entry points):
//  V1  float32 page metadata: l and u kept exactly as the float32 extrema of
//      the rotated keys (no rounding), instead of R1's outward bf16.
//  V2  GQA-sum: the token distance is the sum over G(g) of Eq. 2, instead of
//      R4's min (the paper does not treat grouped heads; both readings fit).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

namespace {

double widen_bf16(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

uint32_t bits_of(float f) {
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  return u;
}

// Largest bf16 value <= f (f finite).  Truncating the low 16 bits moves the
// value toward zero; for a negative inexact value one more bf16 step of
// magnitude is needed to land below f.
uint16_t bf16_toward_neg_inf(float f) {
  const uint32_t u = bits_of(f);
  const uint16_t t = static_cast<uint16_t>(u >> 16);
  if ((u & 0xFFFFu) == 0) return t;
  return (u >> 31) ? static_cast<uint16_t>(t + 1) : t;
}

// Smallest bf16 value >= f (f finite).
uint16_t bf16_toward_pos_inf(float f) {
  const uint32_t u = bits_of(f);
  const uint16_t t = static_cast<uint16_t>(u >> 16);
  if ((u & 0xFFFFu) == 0) return t;
  return (u >> 31) ? t : static_cast<uint16_t>(t + 1);
}

double meta_value(uint16_t h) { return widen_bf16(h); }
double meta_value(float f) { return static_cast<double>(f); }

int bit_count(uint32_t x) {
  int c = 0;
  for (int i = 0; i < 32; ++i) c += (x >> i) & 1u;
  return c;
}

}  // namespace

extern "C" {

// §3.3.1 Eq. 4: out[n][j] = float32( sum_i x[n][i] * R[i][j] ).
void hhro_rotate(const uint16_t* x, int64_t n, int32_t d, const float* R, float* out) {
  std::vector<double> acc(d);
  for (int64_t row = 0; row < n; ++row) {
    std::fill(acc.begin(), acc.end(), 0.0);
    for (int i = 0; i < d; ++i) {
      const double xi = widen_bf16(x[row * d + i]);
      const float* Ri = R + static_cast<int64_t>(i) * d;
      for (int j = 0; j < d; ++j) acc[j] += xi * static_cast<double>(Ri[j]);
    }
    for (int j = 0; j < d; ++j) out[row * d + j] = static_cast<float>(acc[j]);
  }
}

// §3.3.2 Eq. 10 with the inference-time binarisation c = sign(z) (§3.3.2, text
// after Eq. 10) and the binary code of §3.1 Eq. 1.  Bit t of row n is stored in
// word t/32 at bit position t%32 (least significant first); bit = (z > 0)
// (reading R2).  Returns how many projections have |z| < 1e-4 (sign
// ambiguous at float32 precision).  z_out (nullable) receives z in double.
int64_t hhro_project_sign(const uint16_t* x, int64_t n, int32_t d, int32_t bits,
                          const float* W, uint32_t* codes, double* z_out) {
  const int words = bits / 32;
  std::vector<double> z(bits);
  int64_t ambiguous = 0;
  for (int64_t row = 0; row < n; ++row) {
    std::fill(z.begin(), z.end(), 0.0);
    for (int i = 0; i < d; ++i) {
      const double xi = widen_bf16(x[row * d + i]);
      const float* Wi = W + static_cast<int64_t>(i) * bits;
      for (int t = 0; t < bits; ++t) z[t] += xi * static_cast<double>(Wi[t]);
    }
    for (int w = 0; w < words; ++w) {
      uint32_t word = 0;
      for (int b = 0; b < 32; ++b) {
        const double v = z[w * 32 + b];
        if (v > 0.0) word |= (1u << b);
        if (std::fabs(v) < 1e-4) ++ambiguous;
      }
      codes[row * words + w] = word;
    }
    if (z_out)
      for (int t = 0; t < bits; ++t) z_out[row * bits + t] = z[t];
  }
  return ambiguous;
}

// §3.3.1, the definition under Eq. 3: l^j / u^j are the minimum / maximum of
// the (rotated) keys of page p along dimension j.  kt holds rotated keys of
// tokens [t0, n_valid) in row order; pages [p_begin, p_end) are written.
// Storage follows reading R1 (bf16, rounded outward).  Layout of meta per
// page: d lower values, then d upper values.
void hhro_page_meta(const float* kt, int64_t t0, int64_t n_valid, int32_t d, int32_t page,
                    int64_t p_begin, int64_t p_end, uint16_t* meta) {
  for (int64_t p = p_begin; p < p_end; ++p) {
    const int64_t n0 = p * page;
    const int64_t n1 = std::min<int64_t>(n0 + page, n_valid);
    if (n1 <= n0) continue;
    for (int j = 0; j < d; ++j) {
      float lo = std::numeric_limits<float>::infinity();
      float hi = -std::numeric_limits<float>::infinity();
      for (int64_t n = n0; n < n1; ++n) {
        const float v = kt[(n - t0) * d + j];
        lo = std::min(lo, v);
        hi = std::max(hi, v);
      }
      meta[(p * 2 + 0) * d + j] = bf16_toward_neg_inf(lo);
      meta[(p * 2 + 1) * d + j] = bf16_toward_pos_inf(hi);
    }
  }
}

// Variant V1 of the metadata above: the same extrema, kept in float32 as
// computed (no rounding).
void hhro_page_meta_f32(const float* kt, int64_t t0, int64_t n_valid, int32_t d, int32_t page,
                        int64_t p_begin, int64_t p_end, float* meta) {
  for (int64_t p = p_begin; p < p_end; ++p) {
    const int64_t n0 = p * page;
    const int64_t n1 = std::min<int64_t>(n0 + page, n_valid);
    if (n1 <= n0) continue;
    for (int j = 0; j < d; ++j) {
      float lo = std::numeric_limits<float>::infinity();
      float hi = -std::numeric_limits<float>::infinity();
      for (int64_t n = n0; n < n1; ++n) {
        const float v = kt[(n - t0) * d + j];
        lo = std::min(lo, v);
        hi = std::max(hi, v);
      }
      meta[(p * 2 + 0) * d + j] = lo;
      meta[(p * 2 + 1) * d + j] = hi;
    }
  }
}

// Key encoding of one (sequence, KV head) for the keys [n_begin, n_end):
// codes of those keys (Eq. 10 + sign) and the metadata of every page they
// touch, recomputed from all keys [p*S, min((p+1)*S, n_end)) of that page
// (so a page that already held keys before n_begin is re-derived from its
// full key set).  K: [n_cap][d] bf16 bits; codes: [n_cap][bits/32];
// meta: [ceil(n_cap/S)][2][d].  Returns the ambiguous-sign count.
int64_t hhro_encode_unit(const uint16_t* K, int64_t n_begin, int64_t n_end, int32_t d,
                         int32_t bits, int32_t page, const float* R, const float* W,
                         uint32_t* codes, uint16_t* meta) {
  if (n_end <= n_begin) return 0;
  const int64_t p0 = n_begin / page;
  const int64_t p1 = (n_end - 1) / page + 1;
  const int64_t t0 = p0 * page;
  std::vector<float> kt(static_cast<size_t>((n_end - t0) * d));
  hhro_rotate(K + t0 * d, n_end - t0, d, R, kt.data());
  hhro_page_meta(kt.data(), t0, n_end, d, page, p0, p1, meta);
  const int words = bits / 32;
  return hhro_project_sign(K + n_begin * d, n_end - n_begin, d, bits, W,
                           codes + n_begin * words, nullptr);
}

// hhro_encode_unit with float32 metadata (variant V1).
int64_t hhro_encode_unit_f32(const uint16_t* K, int64_t n_begin, int64_t n_end, int32_t d,
                             int32_t bits, int32_t page, const float* R, const float* W,
                             uint32_t* codes, float* meta) {
  if (n_end <= n_begin) return 0;
  const int64_t p0 = n_begin / page;
  const int64_t p1 = (n_end - 1) / page + 1;
  const int64_t t0 = p0 * page;
  std::vector<float> kt(static_cast<size_t>((n_end - t0) * d));
  hhro_rotate(K + t0 * d, n_end - t0, d, R, kt.data());
  hhro_page_meta_f32(kt.data(), t0, n_end, d, page, p0, p1, meta);
  const int words = bits / 32;
  return hhro_project_sign(K + n_begin * d, n_end - n_begin, d, bits, W,
                           codes + n_begin * words, nullptr);
}

// Query side of Eq. 4 (q~ = q R) and of Eq. 10 + sign, for the r query heads
// of one KV group.  Returns the ambiguous-sign count of the query codes.
int64_t hhro_query_prep(const uint16_t* q, int32_t r, int32_t d, int32_t bits,
                        const float* R, const float* W, float* qt, uint32_t* qcode) {
  hhro_rotate(q, r, d, R, qt);
  return hhro_project_sign(q, r, d, bits, W, qcode, nullptr);
}

// §3.3.1 Eq. 3: U_{h,p} = sum_j max(q~_h^j l_p^j, q~_h^j u_p^j), in double from
// the float32 q~ and the widened bf16 bounds; the group score is the max over
// the r heads (reading R4).  Uh (nullable) receives the per-head values
// [r][np].
}  // extern "C"

namespace {
template <typename MetaT>
void page_bounds(const float* qt, int32_t r, int32_t d, const MetaT* meta, int64_t np, double* U,
                 double* Uh) {
  for (int64_t p = 0; p < np; ++p) {
    const MetaT* lo = meta + (p * 2 + 0) * d;
    const MetaT* hi = meta + (p * 2 + 1) * d;
    double best = -std::numeric_limits<double>::infinity();
    for (int h = 0; h < r; ++h) {
      double s = 0.0;
      for (int j = 0; j < d; ++j) {
        const double qj = static_cast<double>(qt[h * d + j]);
        const double a = qj * meta_value(lo[j]);
        const double b = qj * meta_value(hi[j]);
        s += std::max(a, b);
      }
      if (Uh) Uh[h * np + p] = s;
      best = std::max(best, s);
    }
    U[p] = best;
  }
}
}  // namespace

extern "C" {

void hhro_page_bounds(const float* qt, int32_t r, int32_t d, const uint16_t* meta, int64_t np,
                      double* U, double* Uh) {
  page_bounds(qt, r, d, meta, np, U, Uh);
}

// Eq. 3 on float32 metadata (variant V1).
void hhro_page_bounds_f32(const float* qt, int32_t r, int32_t d, const float* meta, int64_t np,
                          double* U, double* Uh) {
  page_bounds(qt, r, d, meta, np, U, Uh);
}

// Page retention (§3.3.1 after Eq. 3, readings R5): indices of the
// min(m, n) largest scores, ties to the lower index, written ascending.
// Returns the count.
int64_t hhro_top_largest(const double* s, int64_t n, int64_t m, int32_t* out) {
  std::vector<int32_t> idx(static_cast<size_t>(n));
  for (int64_t i = 0; i < n; ++i) idx[i] = static_cast<int32_t>(i);
  std::sort(idx.begin(), idx.end(), [s](int32_t a, int32_t b) {
    if (s[a] != s[b]) return s[a] > s[b];
    return a < b;
  });
  const int64_t cnt = std::min(m, n);
  std::sort(idx.begin(), idx.begin() + cnt);
  for (int64_t i = 0; i < cnt; ++i) out[i] = idx[i];
  return cnt;
}

// §3.1 Eq. 2 (Hamming distance = number of differing code bits) between the
// query codes and the code of every valid token of the kept pages; the group
// distance is the min over the r heads (reading R4).  D[slot*S + t] is the
// distance of token pages[slot]*S + t, or -1 where that token is >= n_valid.
// agg = 0: min over the heads (R4); agg = 1: sum over the heads (V2).
void hhro_hamming_agg(const uint32_t* qcode, int32_t r, int32_t words, const uint32_t* codes,
                      const int32_t* pages, int64_t n_pages, int32_t page, int64_t n_valid,
                      int32_t agg, int32_t* D) {
  for (int64_t slot = 0; slot < n_pages; ++slot) {
    for (int t = 0; t < page; ++t) {
      const int64_t n = static_cast<int64_t>(pages[slot]) * page + t;
      if (n >= n_valid) {
        D[slot * page + t] = -1;
        continue;
      }
      int best = std::numeric_limits<int>::max(), total = 0;
      for (int h = 0; h < r; ++h) {
        int dist = 0;
        for (int w = 0; w < words; ++w) dist += bit_count(qcode[h * words + w] ^ codes[n * words + w]);
        best = std::min(best, dist);
        total += dist;
      }
      D[slot * page + t] = agg ? total : best;
    }
  }
}

void hhro_hamming(const uint32_t* qcode, int32_t r, int32_t words, const uint32_t* codes,
                  const int32_t* pages, int64_t n_pages, int32_t page, int64_t n_valid,
                  int32_t* D) {
  hhro_hamming_agg(qcode, r, words, codes, pages, n_pages, page, n_valid, 0, D);
}

// Token selection (§3.3.2 inference + Top-K of §4.1, reading R6): among the
// tokens with D >= 0, the min(k, count) smallest distances, ties to the lower
// token index, written ascending.  Returns the count.
int64_t hhro_top_tokens(const int32_t* D, const int32_t* pages, int64_t n_pages, int32_t page,
                        int64_t k, int32_t* tok) {
  std::vector<std::pair<int32_t, int32_t>> cand;  // (distance, token)
  for (int64_t slot = 0; slot < n_pages; ++slot)
    for (int t = 0; t < page; ++t) {
      const int32_t dist = D[slot * page + t];
      if (dist >= 0) cand.emplace_back(dist, pages[slot] * page + t);
    }
  std::sort(cand.begin(), cand.end());
  const int64_t cnt = std::min<int64_t>(k, static_cast<int64_t>(cand.size()));
  std::vector<int32_t> sel(static_cast<size_t>(cnt));
  for (int64_t i = 0; i < cnt; ++i) sel[i] = cand[i].second;
  std::sort(sel.begin(), sel.end());
  for (int64_t i = 0; i < cnt; ++i) tok[i] = sel[i];
  return cnt;
}

// Selection-quality reference (diagnostic): the m keys among [0, n_valid)
// with the largest exact group logit max_h q_h . k_n (double, from the bf16
// values; the same "any head of the group" reading as R4), ties to the lower
// index, written ascending.  Returns the count.  K: [n_cap][d] bf16 bits.
int64_t hhro_top_logits(const uint16_t* q, int32_t r, int32_t d, const uint16_t* K, int64_t n_valid,
                        int64_t m, int32_t* out) {
  std::vector<double> s(static_cast<size_t>(n_valid));
  for (int64_t n = 0; n < n_valid; ++n) {
    double best = -std::numeric_limits<double>::infinity();
    for (int h = 0; h < r; ++h) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += widen_bf16(q[h * d + j]) * widen_bf16(K[n * d + j]);
      best = std::max(best, acc);
    }
    s[n] = best;
  }
  return hhro_top_largest(s.data(), n_valid, m, out);
}

// Attention over the selected keys (§1: attention is computed on the keys the
// hash retrieval selects; reading R7).  For each of the r heads:
// s_i = scale * q_h . K[idx_i], o = sum_i e^(s_i - max s) V[idx_i] / sum_i e^(s_i - max s).
// K, V: [n_cap][d] bf16 bits of one (sequence, KV head); out: [r][d].
// With no selected key the output is zero.
void hhro_attend(const uint16_t* q, int32_t r, int32_t d, const uint16_t* K, const uint16_t* V,
                 const int32_t* idx, int64_t n_sel, double scale, float* out) {
  std::vector<double> s(static_cast<size_t>(n_sel));
  std::vector<double> o(d);
  for (int h = 0; h < r; ++h) {
    if (n_sel == 0) {
      for (int j = 0; j < d; ++j) out[h * d + j] = 0.0f;
      continue;
    }
    double m = -std::numeric_limits<double>::infinity();
    for (int64_t i = 0; i < n_sel; ++i) {
      const int64_t n = idx[i];
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += widen_bf16(q[h * d + j]) * widen_bf16(K[n * d + j]);
      s[i] = scale * acc;
      m = std::max(m, s[i]);
    }
    double l = 0.0;
    std::fill(o.begin(), o.end(), 0.0);
    for (int64_t i = 0; i < n_sel; ++i) {
      const double p = std::exp(s[i] - m);
      l += p;
      const int64_t n = idx[i];
      for (int j = 0; j < d; ++j) o[j] += p * widen_bf16(V[n * d + j]);
    }
    for (int j = 0; j < d; ++j) out[h * d + j] = static_cast<float>(o[j] / l);
  }
}

// One decode step for one (sequence, KV head): query preparation, page
// bounds, page top-P, Hamming over the kept pages, token top-k and (when out
// is not null) attention.  Outputs are padded with -1 past their counts:
// page_idx [P], tok_idx [k], D [P*S] (nullable), U [ceil(n_valid/S)]
// (nullable).  Returns the number of selected tokens; *q_ambiguous receives
// the ambiguous-sign count of the query codes.
// flags: bit 0 = float32 metadata (V1; meta is float [..][2][d]), bit 1 =
// GQA-sum distances (V2).  hhro_decode_unit is flags = 0.
int64_t hhro_decode_unit_v(const uint16_t* q, int32_t r, int32_t d, int32_t bits, int32_t page,
                           const float* R, const float* W, const uint32_t* codes,
                           const void* meta, const uint16_t* K, const uint16_t* V,
                           int64_t n_valid, int64_t P, int64_t k, double scale, int32_t flags,
                           int32_t* page_idx, int32_t* tok_idx, double* U, int32_t* D,
                           float* out, int64_t* q_ambiguous) {
  const int words = bits / 32;
  std::vector<float> qt(static_cast<size_t>(r) * d);
  std::vector<uint32_t> qcode(static_cast<size_t>(r) * words);
  const int64_t amb = hhro_query_prep(q, r, d, bits, R, W, qt.data(), qcode.data());
  if (q_ambiguous) *q_ambiguous = amb;

  const int64_t np = (n_valid + page - 1) / page;
  std::vector<double> Ubuf(static_cast<size_t>(np));
  if (flags & 1)
    hhro_page_bounds_f32(qt.data(), r, d, static_cast<const float*>(meta), np, Ubuf.data(), nullptr);
  else
    hhro_page_bounds(qt.data(), r, d, static_cast<const uint16_t*>(meta), np, Ubuf.data(), nullptr);
  if (U)
    for (int64_t p = 0; p < np; ++p) U[p] = Ubuf[p];

  std::vector<int32_t> kept(static_cast<size_t>(std::min(P, np)));
  const int64_t n_kept = hhro_top_largest(Ubuf.data(), np, P, kept.data());
  for (int64_t i = 0; i < P; ++i) page_idx[i] = i < n_kept ? kept[i] : -1;

  std::vector<int32_t> Dbuf(static_cast<size_t>(n_kept) * page);
  hhro_hamming_agg(qcode.data(), r, words, codes, kept.data(), n_kept, page, n_valid,
                   (flags & 2) ? 1 : 0, Dbuf.data());
  if (D)
    for (int64_t i = 0; i < P * page; ++i) D[i] = i < n_kept * page ? Dbuf[i] : -1;

  std::vector<int32_t> sel(static_cast<size_t>(k));
  const int64_t n_sel = hhro_top_tokens(Dbuf.data(), kept.data(), n_kept, page, k, sel.data());
  for (int64_t i = 0; i < k; ++i) tok_idx[i] = i < n_sel ? sel[i] : -1;

  if (out) hhro_attend(q, r, d, K, V, sel.data(), n_sel, scale, out);
  return n_sel;
}

int64_t hhro_decode_unit(const uint16_t* q, int32_t r, int32_t d, int32_t bits, int32_t page,
                         const float* R, const float* W, const uint32_t* codes,
                         const uint16_t* meta, const uint16_t* K, const uint16_t* V,
                         int64_t n_valid, int64_t P, int64_t k, double scale,
                         int32_t* page_idx, int32_t* tok_idx, double* U, int32_t* D,
                         float* out, int64_t* q_ambiguous) {
  return hhro_decode_unit_v(q, r, d, bits, page, R, W, codes, meta, K, V, n_valid, P, k, scale,
                            0, page_idx, tok_idx, U, D, out, q_ambiguous);
}

}  // extern "C"
