// CPU oracle of the LSA hot path: indexer -> streaming top-k -> sparse attention.
//
// TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the CPU
// legs of bench.py load this library (through oracle/__init__.py). The product
// path never does, and this file shares no code, header, table or helper with
// the CUDA sources: it includes only the C++ standard library.
//
// Plain, slow, single-threaded C++ per unit of work (one query row, or one
// chunk of one query row's keys), in float64 unless a step fixes another
// precision. A small std::thread harness runs independent units on several
// host cores; every unit's arithmetic is the same whatever the thread count.
//
// What each step computes follows these pages:
//   [LSA]  "LongCat Sparse Attention: Taming the Lightning via Streaming-aware
//          Hierarchical Cross-Layer Indexing" (arXiv 2608.01662, summary page):
//          abstract (1) Streaming-Aware, (2) Cross-Layer, (3) Hierarchical
//          Indexing; key contributions (coarse-to-fine, O(L/P + MP) per query;
//          indexing cost 1/N per layer); limitations (SI gives 50% of the
//          budget to fixed regions).
//   [CARD] "LongCat-Flash-Lite-Sparse" model card: the SI / CLI / HI bullets.
//   [DSA]  "DSA Lightning Indexer" article (Baidu AI Cloud): "Lightweight
//          Scoring Module", "Dynamic Token Selector", "Sparse Attention
//          Calculator", "Quantized computation", "Technical Evolution and
//          Applications".
//
// Readings taken where the pages are silent (each restated where it is used):
//   R1  score[t,s] = sum_h w[t,h] * ReLU(q[t,h] . k[s]) / sqrt(d)  [DSA scoring
//       module shows single-head ReLU(QK^T / sqrt(d)); the head weights are the
//       DSA indexer's as [LSA] recaps it]. ReLU(x)/sqrt(d) = ReLU(x/sqrt(d)).
//   R2  key s is visible to the query at absolute position pos iff s <= pos;
//       the T queries of a length-L sequence sit at pos = L-T .. L-1.
//   R3  sink = [0, min(S, pos+1)); window = the W most recent visible tokens
//       not already in the sink; dynamic candidates = visible tokens in
//       neither; D = k - |sink| - |window| dynamic slots.
//   R4  dynamic order: score descending, equal scores to the lower index.
//   R5  output: sink ascending, window ascending, dynamic ascending, then -1.
//   R6  page p = tokens [pP, pP+P); only full pages pooled; float32 sum in
//       ascending row order, one float32 division by P, bf16 round to nearest
//       even (the stored code is what gets scored).
//   R7  forced pages = pages holding sink or window tokens (they count against
//       M); eligible = full, fully visible pages of only dynamic candidates;
//       recall = forced + the top (M - |forced|) eligible pages by page score
//       (ties to the lower page); fine candidates = dynamic candidates inside
//       the recalled pages; then R3-R5 over them.
//   R8  attention: softmax over the valid (>= 0) indices only; lse = max +
//       ln(sum); no valid index => o = 0, lse = -inf. MLA: V = the first d_v
//       columns of the latent row.
//   R9  cross-layer: one index set from the group's indexer inputs feeds every
//       layer (composed in oracle/__init__.py from the calls below).
//   R10 e4m3 operand = value of its OCP E4M3 code times its float32 row scale.
//   R11 compressed entry e = tokens [e m, e m + m), visible once complete; the
//       query at pos sits at entry position (pos + 1) div m - 1.
//   R12 FP8 page key = float32 mean (R6's order) of the dequantized token keys,
//       stored as e4m3 with page scale amax / 448 (RNE, saturating).
#include <sched.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <limits>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// Element codecs
// ---------------------------------------------------------------------------

// bfloat16 is the upper half of a binary32: widen by appending 16 zero bits.
double bf16_value(uint16_t bits) {
  const uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// binary32 -> bfloat16: keep the upper 16 bits, round the dropped 16 to nearest
// with ties to the even upper half (a carry into the exponent is the correct
// rounding to the next binade or to infinity); NaN stays a quiet NaN.
uint16_t bf16_rne(float x) {
  uint32_t u;
  std::memcpy(&u, &x, 4);
  const uint32_t upper = u >> 16, lower = u & 0xFFFFu;
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return static_cast<uint16_t>(upper | 0x0040u);
  const bool up = lower > 0x8000u || (lower == 0x8000u && (upper & 1u));
  return static_cast<uint16_t>(upper + (up ? 1u : 0u));
}

// OCP FP8 E4M3 ("e4m3fn"): s.eeee.mmm, bias 7. Exponent field 0: subnormal
// m/8 * 2^-6; otherwise (1 + m/8) * 2^(e-7); the codes with all seven low bits
// set are NaN (there is no infinity).
double e4m3_value(uint8_t code) {
  const double sign = (code & 0x80) ? -1.0 : 1.0;
  if ((code & 0x7F) == 0x7F) return std::numeric_limits<double>::quiet_NaN();
  const int e = (code >> 3) & 0xF;
  const int m = code & 0x7;
  const double mag = e == 0 ? (m / 8.0) * std::ldexp(1.0, -6) : (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);
  return sign * mag;
}

// Real value -> e4m3 code: the nearest finite e4m3 value, ties to the even code,
// magnitudes beyond 448 saturate to 448; the sign bit follows x (-0 included).
// Written as a search over the 127 non-negative finite values, not bit tricks.
uint8_t e4m3_rne(double x) {
  const double a = std::min(std::fabs(x), 448.0);
  int best = 0;
  double best_d = std::numeric_limits<double>::infinity();
  for (int c = 0; c < 0x7F; ++c) {
    const double dist = std::fabs(e4m3_value(static_cast<uint8_t>(c)) - a);
    if (dist < best_d || (dist == best_d && (c & 1) == 0)) {
      best_d = dist;
      best = c;
    }
  }
  return static_cast<uint8_t>(best | (std::signbit(x) ? 0x80 : 0));
}

// One stored key or query row, decoded to float64: a bf16 code, or an e4m3
// code times its float32 row scale (R10; the product is exact in float64).
struct Rows {
  const void* codes;
  const float* scale;   // e4m3 only: one scale per row
  bool fp8;
  int64_t width;        // elements per row

  void decode(int64_t row, double* out) const {
    if (fp8) {
      const uint8_t* c = static_cast<const uint8_t*>(codes) + row * width;
      const double s = static_cast<double>(scale[row]);
      for (int64_t i = 0; i < width; ++i) out[i] = e4m3_value(c[i]) * s;
    } else {
      const uint16_t* c = static_cast<const uint16_t*>(codes) + row * width;
      for (int64_t i = 0; i < width; ++i) out[i] = bf16_value(c[i]);
    }
  }
};

// ---------------------------------------------------------------------------
// Thread harness: units 0 .. n-1, each run once by one thread
// ---------------------------------------------------------------------------

int host_threads() {
  cpu_set_t set;
  if (sched_getaffinity(0, sizeof(set), &set) == 0) {
    const int n = CPU_COUNT(&set);
    if (n > 0) return n;
  }
  const unsigned n = std::thread::hardware_concurrency();
  return n ? static_cast<int>(n) : 1;
}

void parallel_for(int64_t n_units, int n_threads, const std::function<void(int64_t)>& unit) {
  if (n_threads <= 0) n_threads = host_threads();
  const int64_t nt = std::max<int64_t>(1, std::min<int64_t>(n_threads, n_units));
  if (nt == 1) {
    for (int64_t u = 0; u < n_units; ++u) unit(u);
    return;
  }
  std::atomic<int64_t> next(0);
  std::vector<std::thread> pool;
  for (int64_t i = 0; i < nt; ++i)
    pool.emplace_back([&] {
      for (int64_t u = next.fetch_add(1); u < n_units; u = next.fetch_add(1)) unit(u);
    });
  for (auto& th : pool) th.join();
}

int clamp_len(int v, int L_max) { return v < 0 ? 0 : (v > L_max ? L_max : v); }

int64_t floor_div(int64_t a, int64_t b) {
  const int64_t q = a / b;
  return (a % b != 0 && ((a < 0) != (b < 0))) ? q - 1 : q;
}

// ---------------------------------------------------------------------------
// Lightning-indexer score ([DSA] "Lightweight Scoring Module"; R1, R2, R10)
// ---------------------------------------------------------------------------

// One query, decoded: its H head vectors stored transposed (qT[i*H + h]) so the
// per-head dot products run side by side, and its head weights.
struct Query {
  int H = 0, d = 0;
  std::vector<double> qT, w;

  void set(const double* q_hd /* [H, d] */, const double* w_h, int H_, int d_) {
    H = H_;
    d = d_;
    qT.assign(static_cast<size_t>(H) * d, 0.0);
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < d; ++i) qT[static_cast<size_t>(i) * H + h] = q_hd[static_cast<size_t>(h) * d + i];
    w.assign(w_h, w_h + H);
  }

  // score = (sum_h w[h] * max(sum_i q[h,i] key[i], 0)) / sqrt(d), in float64,
  // each sum in ascending order, rounded once to float32.
  float score(const double* key, double* dots /* [H] scratch */) const {
    for (int h = 0; h < H; ++h) dots[h] = 0.0;
    for (int i = 0; i < d; ++i) {
      const double ki = key[i];
      const double* qi = &qT[static_cast<size_t>(i) * H];
      for (int h = 0; h < H; ++h) dots[h] += qi[h] * ki;
    }
    double s = 0.0;
    for (int h = 0; h < H; ++h) s += w[h] * (dots[h] > 0.0 ? dots[h] : 0.0);
    return static_cast<float>(s / std::sqrt(static_cast<double>(d)));
  }
};

// Decoded query (b, t) of a [B, T, H, d] tensor.
void load_query(const Rows& q, const float* w, int T, int H, int d, int b, int t, Query* out) {
  std::vector<double> qd(static_cast<size_t>(H) * d), wd(H);
  for (int h = 0; h < H; ++h) {
    const int64_t row = (static_cast<int64_t>(b) * T + t) * H + h;
    q.decode(row, &qd[static_cast<size_t>(h) * d]);
    wd[h] = static_cast<double>(w[row]);
  }
  out->set(qd.data(), wd.data(), H, d);
}

// Scores of keys [s0, s1) of one sequence (row offset key_row0 in `keys`) for
// one query; keys at or beyond n_visible get -inf.
void score_range(const Query& q, const Rows& keys, int64_t key_row0, int64_t s0, int64_t s1, int64_t n_visible,
                 float* out) {
  std::vector<double> key(q.d), dots(q.H);
  for (int64_t s = s0; s < s1; ++s) {
    if (s >= n_visible) {
      out[s - s0] = -std::numeric_limits<float>::infinity();
      continue;
    }
    keys.decode(key_row0 + s, key.data());
    out[s - s0] = q.score(key.data(), dots.data());
  }
}

// ---------------------------------------------------------------------------
// Streaming-aware selection ([LSA] abstract (1), [CARD] "SI"; [DSA] "Dynamic
// Token Selector"; R3, R4, R5)
// ---------------------------------------------------------------------------

struct Regions {
  int64_t sink_end, w_lo, w_hi;   // sink [0, sink_end); window [w_lo, w_hi); candidates [sink_end, w_lo)
};

Regions regions(int64_t pos, int64_t sink, int64_t window) {
  Regions r{0, 0, 0};
  if (pos < 0) return r;
  r.sink_end = std::min(sink, pos + 1);
  r.w_lo = std::max(r.sink_end, pos - window + 1);
  r.w_hi = pos + 1;
  return r;
}

// The n best of the candidates by (score descending, index ascending), kept in
// a bounded heap whose top is the worst kept entry, returned ascending by index.
// Candidates must arrive in ascending index order, so an entry equal in score
// to the worst kept one never displaces it (it has the higher index).
struct Cand {
  double score;
  int64_t index;
};

bool better(const Cand& a, const Cand& b) { return a.score > b.score || (a.score == b.score && a.index < b.index); }

std::vector<int64_t> top_by_score(const std::vector<Cand>& ascending, int64_t n) {
  std::vector<Cand> heap;
  if (n <= 0) return {};
  // std heap functions keep the "largest" element on top; with `better` as the
  // ordering the largest is the worst candidate.
  for (const Cand& c : ascending) {
    if (static_cast<int64_t>(heap.size()) < n) {
      heap.push_back(c);
      std::push_heap(heap.begin(), heap.end(), better);
    } else if (better(c, heap.front())) {
      std::pop_heap(heap.begin(), heap.end(), better);
      heap.back() = c;
      std::push_heap(heap.begin(), heap.end(), better);
    }
  }
  std::vector<int64_t> out;
  out.reserve(heap.size());
  for (const Cand& c : heap) out.push_back(c.index);
  std::sort(out.begin(), out.end());
  return out;
}

// Index row of one query from its float32 scores (R3-R5). Dynamic candidates
// whose score is -inf (invisible) are not candidates. Returns false if the
// sink and window exceed the budget.
bool select_row(const float* scores, int64_t n_scores, int64_t pos, int k, int sink, int window, int32_t* out) {
  for (int i = 0; i < k; ++i) out[i] = -1;
  const Regions r = regions(pos, sink, window);
  const int64_t fixed = r.sink_end + (r.w_hi - r.w_lo);
  const int64_t D = k - fixed;
  if (D < 0) return false;
  int64_t o = 0;
  for (int64_t s = 0; s < r.sink_end; ++s) out[o++] = static_cast<int32_t>(s);
  for (int64_t s = r.w_lo; s < r.w_hi; ++s) out[o++] = static_cast<int32_t>(s);
  std::vector<Cand> cands;
  for (int64_t s = r.sink_end; s < r.w_lo && s < n_scores; ++s)
    if (scores[s] > -std::numeric_limits<float>::infinity()) cands.push_back({static_cast<double>(scores[s]), s});
  for (int64_t s : top_by_score(cands, D)) out[o++] = static_cast<int32_t>(s);
  return true;
}

// ---------------------------------------------------------------------------
// Hierarchical indexing ([LSA] abstract (3), key contributions; [CARD] "HI";
// R6, R7, R12)
// ---------------------------------------------------------------------------

// Forced pages (ascending) and the eligible page range [e_lo, e_hi) (R7).
void page_sets(int64_t pos, int64_t P, int64_t sink, int64_t window, std::vector<int64_t>* forced, int64_t* e_lo,
               int64_t* e_hi) {
  forced->clear();
  *e_lo = *e_hi = 0;
  if (pos < 0) return;
  const Regions r = regions(pos, sink, window);
  const int64_t lo = (r.sink_end + P - 1) / P;   // pages holding sink tokens: [0, ceil(|sink| / P))
  int64_t hi;
  std::vector<int64_t> f;
  for (int64_t p = 0; p < lo; ++p) f.push_back(p);
  if (r.w_hi > r.w_lo) {
    for (int64_t p = r.w_lo / P; p <= pos / P; ++p)
      if (p >= lo) f.push_back(p);
    hi = r.w_lo / P;
  } else {
    hi = (pos + 1) / P;
  }
  *forced = f;
  *e_lo = lo;
  *e_hi = std::max(lo, hi);
}

// Reads row `r` of a key table into out [d] as float64.
using RowFn = std::function<void(int64_t, double*)>;

// Coarse-to-fine selection of one query (R7). key(s) reads this sequence's
// token key s, page(p) its page key p (full pages only). idx [k], recalled [M]
// (ascending, -1 padded). Returns false when M is smaller than the forced pages
// or the sink and window exceed the budget.
bool hier_row(const Query& q, const RowFn& key_row, const RowFn& page_row, int64_t pos, int P, int M, int k,
              int sink, int window, int32_t* idx, int32_t* recalled) {
  for (int i = 0; i < k; ++i) idx[i] = -1;
  for (int i = 0; i < M; ++i) recalled[i] = -1;
  if (pos < 0) return true;
  std::vector<int64_t> forced;
  int64_t e_lo, e_hi;
  page_sets(pos, P, sink, window, &forced, &e_lo, &e_hi);
  const int64_t n_dyn = M - static_cast<int64_t>(forced.size());
  if (n_dyn < 0) return false;
  // page scores of the eligible pages, then their top (M - |forced|)
  std::vector<double> key(q.d), dots(q.H);
  std::vector<Cand> pc;
  for (int64_t p = e_lo; p < e_hi; ++p) {
    page_row(p, key.data());
    pc.push_back({static_cast<double>(q.score(key.data(), dots.data())), p});
  }
  std::vector<int64_t> recall = top_by_score(pc, n_dyn);
  recall.insert(recall.end(), forced.begin(), forced.end());
  std::sort(recall.begin(), recall.end());
  for (size_t i = 0; i < recall.size(); ++i) recalled[i] = static_cast<int32_t>(recall[i]);
  // fine candidates: dynamic candidates inside recalled pages, scored on the token keys
  const Regions r = regions(pos, sink, window);
  const int64_t D = k - (r.sink_end + (r.w_hi - r.w_lo));
  if (D < 0) return false;
  std::vector<char> in_recall(static_cast<size_t>(pos / P + 1), 0);
  for (int64_t p : recall)
    if (p <= pos / P) in_recall[static_cast<size_t>(p)] = 1;
  std::vector<Cand> tc;
  for (int64_t s = r.sink_end; s < r.w_lo; ++s) {
    if (!in_recall[static_cast<size_t>(s / P)]) continue;
    key_row(s, key.data());
    tc.push_back({static_cast<double>(q.score(key.data(), dots.data())), s});
  }
  int64_t o = 0;
  for (int64_t s = 0; s < r.sink_end; ++s) idx[o++] = static_cast<int32_t>(s);
  for (int64_t s = r.w_lo; s < r.w_hi; ++s) idx[o++] = static_cast<int32_t>(s);
  for (int64_t s : top_by_score(tc, D)) idx[o++] = static_cast<int32_t>(s);
  return true;
}

// ---------------------------------------------------------------------------
// Sparse attention ([DSA] "Sparse Attention Calculator"; [LSA] abstract:
// attention reads only the selected entries; R8)
// ---------------------------------------------------------------------------

// One query over the rows named by idx (n entries, -1 skipped). q [Hq, d_qk];
// K row j = krow(j) [d_qk], V row j = vrow(j) [d_v]. o [Hq, d_v], lse [Hq].
void attention_row(const double* q, int Hq, int d_qk, int d_v, const int64_t* idx, int64_t n,
                   const std::function<void(int64_t, double*)>& krow, const std::function<void(int64_t, double*)>& vrow,
                   double scale, double* o, double* lse) {
  std::vector<int64_t> valid;
  for (int64_t j = 0; j < n; ++j)
    if (idx[j] >= 0) valid.push_back(idx[j]);
  for (int64_t i = 0; i < static_cast<int64_t>(Hq) * d_v; ++i) o[i] = 0.0;
  if (valid.empty()) {
    for (int h = 0; h < Hq; ++h) lse[h] = -std::numeric_limits<double>::infinity();
    return;
  }
  const int64_t nv = static_cast<int64_t>(valid.size());
  // transposed q so the Hq dot products of one key row run side by side
  std::vector<double> qT(static_cast<size_t>(d_qk) * Hq);
  for (int h = 0; h < Hq; ++h)
    for (int i = 0; i < d_qk; ++i) qT[static_cast<size_t>(i) * Hq + h] = q[static_cast<size_t>(h) * d_qk + i];
  // logits l[j, h] = scale * sum_i q[h, i] K[j, i]
  std::vector<double> logit(static_cast<size_t>(nv) * Hq, 0.0), krow_buf(d_qk), vrow_buf(d_v);
  for (int64_t j = 0; j < nv; ++j) {
    krow(valid[j], krow_buf.data());
    double* lj = &logit[static_cast<size_t>(j) * Hq];
    for (int i = 0; i < d_qk; ++i) {
      const double ki = krow_buf[i];
      const double* qi = &qT[static_cast<size_t>(i) * Hq];
      for (int h = 0; h < Hq; ++h) lj[h] += qi[h] * ki;
    }
    for (int h = 0; h < Hq; ++h) lj[h] *= scale;
  }
  // m = max_j l; p_j = exp(l_j - m); o = sum_j p_j V_j / sum_j p_j
  std::vector<double> mx(Hq, -std::numeric_limits<double>::infinity()), den(Hq, 0.0);
  for (int64_t j = 0; j < nv; ++j)
    for (int h = 0; h < Hq; ++h) mx[h] = std::max(mx[h], logit[static_cast<size_t>(j) * Hq + h]);
  std::vector<double> p(Hq);
  for (int64_t j = 0; j < nv; ++j) {
    vrow(valid[j], vrow_buf.data());
    for (int h = 0; h < Hq; ++h) {
      p[h] = std::exp(logit[static_cast<size_t>(j) * Hq + h] - mx[h]);
      den[h] += p[h];
    }
    for (int h = 0; h < Hq; ++h) {
      double* oh = o + static_cast<size_t>(h) * d_v;
      const double ph = p[h];
      for (int c = 0; c < d_v; ++c) oh[c] += ph * vrow_buf[c];
    }
  }
  for (int h = 0; h < Hq; ++h) {
    double* oh = o + static_cast<size_t>(h) * d_v;
    for (int c = 0; c < d_v; ++c) oh[c] /= den[h];
    lse[h] = mx[h] + std::log(den[h]);
  }
}

// The (b, t) pairs to compute: the given list, or every row.
std::vector<std::pair<int, int>> row_list(int B, int T, const int32_t* rows, int n_rows) {
  std::vector<std::pair<int, int>> out;
  if (rows) {
    for (int i = 0; i < n_rows; ++i) out.emplace_back(rows[2 * i], rows[2 * i + 1]);
  } else {
    for (int b = 0; b < B; ++b)
      for (int t = 0; t < T; ++t) out.emplace_back(b, t);
  }
  return out;
}

constexpr int64_t kChunk = 8192;   // keys per unit of work in the score harness

}  // namespace

// ===========================================================================
// C entry points (host pointers; every function returns 0 on success, -1 on a
// bad argument). Layouts as the CUDA library's, all dense row-major:
//   q [B,T,H,d] (bf16 codes as uint16, or e4m3 codes as uint8 with q_scale
//   [B,T,H]); w [B,T,H] float32; k [B,L_max,d] (codes, k_scale [B,L_max]);
//   seq_len [B] int32; scores [B,T,L_max] float32; idx [B,T,k] int32.
// n_threads <= 0 means every host core this process may run on.
// ===========================================================================

extern "C" {

int orc_host_threads(void) { return host_threads(); }

void orc_bf16_to_f64(int64_t n, const uint16_t* in, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_value(in[i]);
}

void orc_f32_to_bf16_rne(int64_t n, const float* in, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_rne(in[i]);
}

void orc_e4m3_to_f64(int64_t n, const uint8_t* in, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(in[i]);
}

void orc_f64_to_e4m3_rne(int64_t n, const double* in, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_rne(in[i]);
}

// Scores of one query given as float64: q [H,d], w [H], keys [n,d]; keys at or
// beyond n_visible get -inf. out [n] float32.
int orc_indexer_scores_row(const double* q, const double* w, const double* keys, int H, int d, int64_t n,
                           int64_t n_visible, float* out) {
  if (H < 1 || d < 1 || n < 0) return -1;
  Query qq;
  qq.set(q, w, H, d);
  std::vector<double> dots(H);
  for (int64_t s = 0; s < n; ++s)
    out[s] = s < n_visible ? qq.score(keys + s * d, dots.data()) : -std::numeric_limits<float>::infinity();
  return 0;
}

// Flat indexer scores of the listed rows (pairs (b, t); NULL = every row, in
// (b, t) order), written compactly: out [n_rows, n_keys] float32 where n_keys =
// L_rows (keys per sequence). Key s of row (b, t) is visible iff
// s < (pos + 1) >> vis_shift, pos = clamp(seq_len[b], 0, L_max) - T + t
// (vis_shift 0: tokens; log2 m: entries of m tokens, R11).
int orc_indexer_scores_rows(int B, int T, int H, int d, int L_rows, int L_max, int vis_shift, int fp8,
                            const void* q, const float* q_scale, const float* w, const void* k, const float* k_scale,
                            const int32_t* seq_len, const int32_t* rows, int n_rows, float* out, int n_threads) {
  if (B < 1 || T < 1 || H < 1 || d < 1 || L_rows < 0 || vis_shift < 0) return -1;
  const auto list = row_list(B, T, rows, n_rows);
  for (const auto& r : list)
    if (r.first < 0 || r.first >= B || r.second < 0 || r.second >= T) return -1;
  const Rows qr{q, q_scale, fp8 != 0, d};
  const Rows kr{k, k_scale, fp8 != 0, d};
  const int64_t n_chunks = (L_rows + kChunk - 1) / kChunk;
  const int64_t n_list = static_cast<int64_t>(list.size());
  std::vector<Query> queries(list.size());
  parallel_for(n_list, n_threads, [&](int64_t i) {
    load_query(qr, w, T, H, d, list[i].first, list[i].second, &queries[i]);
  });
  parallel_for(n_list * n_chunks, n_threads, [&](int64_t u) {
    const int64_t i = u / n_chunks, c = u % n_chunks;
    const int b = list[i].first, t = list[i].second;
    const int64_t pos = static_cast<int64_t>(clamp_len(seq_len[b], L_max)) - T + t;
    const int64_t n_vis = pos < 0 ? 0 : ((pos + 1) >> vis_shift);
    const int64_t s0 = c * kChunk, s1 = std::min<int64_t>(L_rows, s0 + kChunk);
    score_range(queries[i], kr, static_cast<int64_t>(b) * L_rows, s0, s1, n_vis, out + i * L_rows + s0);
  });
  return 0;
}

// (sink end, window lo, window hi) of a query at pos: sink [0, out[0]), window
// [out[1], out[2]), dynamic candidates [out[0], out[1]) (R3).
void orc_streaming_regions(int64_t pos, int64_t sink, int64_t window, int64_t* out3) {
  const Regions r = regions(pos, sink, window);
  out3[0] = r.sink_end;
  out3[1] = r.w_lo;
  out3[2] = r.w_hi;
}

// Index row of one query (R3-R5) from n_scores float32 scores.
int orc_select_row(const float* scores, int64_t n_scores, int64_t pos, int k, int sink, int window, int32_t* out) {
  if (k < 1) return -1;
  return select_row(scores, n_scores, pos, k, sink, window, out) ? 0 : -1;
}

// Batch selection: scores [B,T,L_max] -> idx [B,T,k].
int orc_select_streaming(const float* scores, const int32_t* seq_len, int B, int T, int L_max, int k, int sink,
                         int window, int32_t* idx, int n_threads) {
  if (B < 1 || T < 1 || L_max < 1 || k < 1) return -1;
  std::atomic<int> bad(0);
  parallel_for(static_cast<int64_t>(B) * T, n_threads, [&](int64_t r) {
    const int b = static_cast<int>(r / T), t = static_cast<int>(r % T);
    const int64_t pos = static_cast<int64_t>(clamp_len(seq_len[b], L_max)) - T + t;
    if (!select_row(scores + r * L_max, L_max, pos, k, sink, window, idx + r * k)) bad = 1;
  });
  return bad ? -1 : 0;
}

// Forced pages (ascending, at most `cap`) and the eligible range (R7). Returns
// the number of forced pages, or -1 if cap is too small.
int orc_page_sets(int64_t pos, int64_t P, int64_t sink, int64_t window, int64_t* forced, int cap, int64_t* e_range) {
  std::vector<int64_t> f;
  page_sets(pos, P, sink, window, &f, &e_range[0], &e_range[1]);
  if (static_cast<int>(f.size()) > cap) return -1;
  for (size_t i = 0; i < f.size(); ++i) forced[i] = f[i];
  return static_cast<int>(f.size());
}

// Page keys from bf16 token keys (R6): k [B,L_max,d] -> out [B,L_max/P,d];
// page rows that are not full are written as 0.
int orc_pool_pages(const uint16_t* k, const int32_t* seq_len, int B, int L_max, int d, int P, uint16_t* out) {
  if (B < 1 || d < 1 || P < 1) return -1;
  const int64_t n_pages = L_max / P;
  std::memset(out, 0, sizeof(uint16_t) * static_cast<size_t>(B) * n_pages * d);
  for (int b = 0; b < B; ++b) {
    const int64_t n_full = clamp_len(seq_len[b], L_max) / P;
    for (int64_t p = 0; p < n_full; ++p)
      for (int i = 0; i < d; ++i) {
        float acc = 0.0f;
        for (int j = 0; j < P; ++j)
          acc = acc + static_cast<float>(bf16_value(k[(static_cast<int64_t>(b) * L_max + p * P + j) * d + i]));
        const float mean = acc / static_cast<float>(P);
        out[(static_cast<int64_t>(b) * n_pages + p) * d + i] = bf16_rne(mean);
      }
  }
  return 0;
}

// Page keys from e4m3 token keys (R12): k8 [B,L_max,d] codes with k_scale
// [B,L_max] -> codes [B,L_max/P,d], scales [B,L_max/P]. Pages that are not full
// get code 0 and scale 1. Each token element is dequantized in float32
// (code value * scale, rounded to float32), summed as R6, divided by P; the
// page scale is amax / 448 in float32 (1 when amax is 0) and each element is
// encoded as e4m3(mean / scale) with mean / scale rounded to float32.
int orc_pool_pages_e4m3(const uint8_t* k8, const float* k_scale, const int32_t* seq_len, int B, int L_max, int d,
                        int P, uint8_t* codes, float* scales) {
  if (B < 1 || d < 1 || P < 1) return -1;
  const int64_t n_pages = L_max / P;
  std::memset(codes, 0, static_cast<size_t>(B) * n_pages * d);
  for (int64_t i = 0; i < static_cast<int64_t>(B) * n_pages; ++i) scales[i] = 1.0f;
  std::vector<float> mean(d);
  for (int b = 0; b < B; ++b) {
    const int64_t n_full = clamp_len(seq_len[b], L_max) / P;
    for (int64_t p = 0; p < n_full; ++p) {
      float amax = 0.0f;
      for (int i = 0; i < d; ++i) {
        float acc = 0.0f;
        for (int j = 0; j < P; ++j) {
          const int64_t row = static_cast<int64_t>(b) * L_max + p * P + j;
          const float x = static_cast<float>(e4m3_value(k8[row * d + i])) * k_scale[row];
          acc = acc + x;
        }
        mean[i] = acc / static_cast<float>(P);
        amax = std::max(amax, std::fabs(mean[i]));
      }
      const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
      const int64_t prow = static_cast<int64_t>(b) * n_pages + p;
      scales[prow] = sc;
      for (int i = 0; i < d; ++i) codes[prow * d + i] = e4m3_rne(static_cast<double>(mean[i] / sc));
    }
  }
  return 0;
}

// Hierarchical indexing of one query given as float64 (R7): q [H,d], w [H],
// keys [L,d] (this sequence's tokens), page_keys [n_pages,d]. idx [k], pages [M].
int orc_index_hier_row(const double* q, const double* w, int H, int d, const double* keys, int64_t L,
                       const double* page_keys, int64_t n_pages, int64_t pos, int P, int M, int k, int sink,
                       int window, int32_t* idx, int32_t* pages) {
  if (H < 1 || d < 1 || P < 1 || M < 0 || k < 1 || pos >= L || (pos >= 0 && (pos + 1) / P > n_pages)) return -1;
  Query qq;
  qq.set(q, w, H, d);
  const RowFn key_row = [&](int64_t s, double* out) { std::memcpy(out, keys + s * d, sizeof(double) * d); };
  const RowFn page_row = [&](int64_t p, double* out) { std::memcpy(out, page_keys + p * d, sizeof(double) * d); };
  return hier_row(qq, key_row, page_row, pos, P, M, k, sink, window, idx, pages) ? 0 : -1;
}

// Hierarchical indexing of a batch (R7; R12 when fp8): q, w, k as the flat
// indexer's; page_keys [B,L_max/P,d] codes (bf16, or e4m3 with page_scale
// [B,L_max/P]). Rows as orc_indexer_scores_rows (NULL = all); idx [n_rows,k],
// pages [n_rows,M] written compactly in list order.
int orc_index_hier(int B, int T, int H, int d, int L_max, int fp8, const void* q, const float* q_scale,
                   const float* w, const void* k, const float* k_scale, const void* page_keys,
                   const float* page_scale, const int32_t* seq_len, int P, int M, int kb, int sink, int window,
                   const int32_t* rows, int n_rows, int32_t* idx, int32_t* pages, int n_threads) {
  if (B < 1 || T < 1 || H < 1 || d < 1 || P < 1 || M < 0 || kb < 1) return -1;
  const auto list = row_list(B, T, rows, n_rows);
  const Rows qr{q, q_scale, fp8 != 0, d};
  const Rows kr{k, k_scale, fp8 != 0, d};
  const Rows pr{page_keys, page_scale, fp8 != 0, d};
  const int64_t n_pages = L_max / P;
  std::atomic<int> bad(0);
  parallel_for(static_cast<int64_t>(list.size()), n_threads, [&](int64_t i) {
    const int b = list[i].first, t = list[i].second;
    if (b < 0 || b >= B || t < 0 || t >= T) {
      bad = 1;
      return;
    }
    Query qq;
    load_query(qr, w, T, H, d, b, t, &qq);
    const int64_t pos = static_cast<int64_t>(clamp_len(seq_len[b], L_max)) - T + t;
    const RowFn key_row = [&](int64_t s, double* out) { kr.decode(static_cast<int64_t>(b) * L_max + s, out); };
    const RowFn page_row = [&](int64_t p, double* out) { pr.decode(static_cast<int64_t>(b) * n_pages + p, out); };
    if (!hier_row(qq, key_row, page_row, pos, P, M, kb, sink, window, idx + i * kb, pages + i * M)) bad = 1;
  });
  return bad ? -1 : 0;
}

// Compressed-entry indexing (R11): entry_keys [B,n_e,d] codes (k_scale [B,n_e]
// for e4m3); seq_len counts tokens; L_max = n_e * m. scores [B,T,n_e] float32
// (-inf at entries not yet complete), idx [B,T,kb] entry ids.
int orc_index_compressed(int B, int T, int H, int d, int n_e, int m, int fp8, const void* q, const float* q_scale,
                         const float* w, const void* entry_keys, const float* k_scale, const int32_t* seq_len,
                         int kb, int sink, int window, float* scores, int32_t* idx, int n_threads) {
  if (B < 1 || T < 1 || H < 1 || d < 1 || n_e < 1 || m < 1 || kb < 1) return -1;
  const int64_t L_max = static_cast<int64_t>(n_e) * m;
  const Rows qr{q, q_scale, fp8 != 0, d};
  const Rows kr{entry_keys, k_scale, fp8 != 0, d};
  std::atomic<int> bad(0);
  parallel_for(static_cast<int64_t>(B) * T, n_threads, [&](int64_t r) {
    const int b = static_cast<int>(r / T), t = static_cast<int>(r % T);
    float* srow = scores + r * n_e;
    int32_t* irow = idx + r * kb;
    for (int64_t e = 0; e < n_e; ++e) srow[e] = -std::numeric_limits<float>::infinity();
    for (int i = 0; i < kb; ++i) irow[i] = -1;
    const int64_t L = std::min<int64_t>(std::max<int64_t>(seq_len[b], 0), L_max);
    const int64_t pe = floor_div(L - T + t + 1, m) - 1;   // last complete entry
    if (pe < 0) return;
    Query qq;
    load_query(qr, w, T, H, d, b, t, &qq);
    score_range(qq, kr, static_cast<int64_t>(b) * n_e, 0, n_e, pe + 1, srow);
    if (!select_row(srow, n_e, pe, kb, sink, window, irow)) bad = 1;
  });
  return bad ? -1 : 0;
}

// Attention of one query given as float64 (R8): q [Hq,d_qk], K rows [n,d_qk],
// V rows [n,d_v] (this sequence's cache), idx [kk] (-1 skipped). o [Hq,d_v],
// lse [Hq].
int orc_sparse_attention_row(const double* q, const double* k_rows, const double* v_rows, int64_t n_rows, int Hq,
                             int d_qk, int d_v, const int64_t* idx, int64_t kk, double scale, double* o,
                             double* lse) {
  for (int64_t j = 0; j < kk; ++j)
    if (idx[j] >= n_rows) return -1;
  attention_row(
      q, Hq, d_qk, d_v, idx, kk,
      [&](int64_t s, double* out) { std::memcpy(out, k_rows + s * d_qk, sizeof(double) * d_qk); },
      [&](int64_t s, double* out) { std::memcpy(out, v_rows + s * d_v, sizeof(double) * d_v); }, scale, o, lse);
  return 0;
}

// Attention of a batch (R8): qa [B,T,Hq,d_qk] bf16 codes; idx [B,T,kk]; K row s
// of sequence b at k + (b*L_max + s)*k_stride (d_qk bf16 codes), V row at
// v + (b*L_max + s)*v_stride (d_v codes; MLA passes v = k). Rows as
// orc_indexer_scores_rows; o [n_rows,Hq,d_v], lse [n_rows,Hq] float64, compact.
int orc_sparse_attention(int B, int T, int Hq, int d_qk, int d_v, int L_max, const uint16_t* qa, const int32_t* idx,
                         int kk, const uint16_t* k, int64_t k_stride, const uint16_t* v, int64_t v_stride, double scale,
                         const int32_t* rows, int n_rows, double* o, double* lse, int n_threads) {
  if (B < 1 || T < 1 || Hq < 1 || d_qk < 1 || d_v < 1 || kk < 0) return -1;
  const auto list = row_list(B, T, rows, n_rows);
  std::atomic<int> bad(0);
  parallel_for(static_cast<int64_t>(list.size()), n_threads, [&](int64_t i) {
    const int b = list[i].first, t = list[i].second;
    if (b < 0 || b >= B || t < 0 || t >= T) {
      bad = 1;
      return;
    }
    const int64_t r = static_cast<int64_t>(b) * T + t;
    std::vector<int64_t> sel(kk);
    for (int j = 0; j < kk; ++j) {
      sel[j] = idx[r * kk + j];
      if (sel[j] >= L_max) {
        bad = 1;
        return;
      }
    }
    std::vector<double> qd(static_cast<size_t>(Hq) * d_qk);
    for (int64_t e = 0; e < static_cast<int64_t>(Hq) * d_qk; ++e) qd[e] = bf16_value(qa[r * Hq * d_qk + e]);
    attention_row(
        qd.data(), Hq, d_qk, d_v, sel.data(), kk,
        [&](int64_t s, double* out) {
          const uint16_t* src = k + (static_cast<int64_t>(b) * L_max + s) * k_stride;
          for (int c = 0; c < d_qk; ++c) out[c] = bf16_value(src[c]);
        },
        [&](int64_t s, double* out) {
          const uint16_t* src = v + (static_cast<int64_t>(b) * L_max + s) * v_stride;
          for (int c = 0; c < d_v; ++c) out[c] = bf16_value(src[c]);
        },
        scale, o + i * Hq * d_v, lse + i * Hq);
  });
  return bad ? -1 : 0;
}

// Attention over an FP8 latent cache (DSA article, "Quantized computation",
// applied to the KV): row s of sequence b holds d_qk e4m3 codes at
// kv8 + (b*L_max + s)*kv_stride (bytes) and its fp32 scale k_scale[b*L_max + s];
// K = code * scale (all d_qk columns), V = the first d_v columns of K. The
// dequantised rows then enter the same attention as orc_sparse_attention.
int orc_sparse_attention_e4m3(int B, int T, int Hq, int d_qk, int d_v, int L_max, const uint16_t* qa,
                              const int32_t* idx, int kk, const uint8_t* kv8, int64_t kv_stride,
                              const float* k_scale, double scale, const int32_t* rows, int n_rows, double* o,
                              double* lse, int n_threads) {
  if (B < 1 || T < 1 || Hq < 1 || d_qk < 1 || d_v < 1 || d_v > d_qk || kk < 0) return -1;
  const auto list = row_list(B, T, rows, n_rows);
  std::atomic<int> bad(0);
  parallel_for(static_cast<int64_t>(list.size()), n_threads, [&](int64_t i) {
    const int b = list[i].first, t = list[i].second;
    if (b < 0 || b >= B || t < 0 || t >= T) {
      bad = 1;
      return;
    }
    const int64_t r = static_cast<int64_t>(b) * T + t;
    std::vector<int64_t> sel(kk);
    for (int j = 0; j < kk; ++j) {
      sel[j] = idx[r * kk + j];
      if (sel[j] >= L_max) {
        bad = 1;
        return;
      }
    }
    std::vector<double> qd(static_cast<size_t>(Hq) * d_qk);
    for (int64_t e = 0; e < static_cast<int64_t>(Hq) * d_qk; ++e) qd[e] = bf16_value(qa[r * Hq * d_qk + e]);
    auto row_of = [&](int64_t s, int width, double* out) {
      const int64_t tok = static_cast<int64_t>(b) * L_max + s;
      const uint8_t* src = kv8 + tok * kv_stride;
      const double sc = static_cast<double>(k_scale[tok]);
      for (int c = 0; c < width; ++c) out[c] = e4m3_value(src[c]) * sc;
    };
    attention_row(
        qd.data(), Hq, d_qk, d_v, sel.data(), kk, [&](int64_t s, double* out) { row_of(s, d_qk, out); },
        [&](int64_t s, double* out) { row_of(s, d_v, out); }, scale, o + i * Hq * d_v, lse + i * Hq);
  });
  return bad ? -1 : 0;
}

}  // extern "C"
