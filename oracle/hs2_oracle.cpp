// HySparse2 hybrid-block ORACLE -- plain C++17, fp64, std::thread.
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct CPU
// statement of what the hybrid-block hot path computes.  Only the test suite,
// the smoke check and the benchmark's CPU-baseline leg may load it.  It shares
// no code, header, table or helper with the CUDA library; both read the same
// input bytes produced by the seeded generator.
//
// What it follows (HySparse2 pages: "Xiaomi MiMo HySparse2" announcement via
// IT Home, paragraphs on KV Bridging, KV Reuse and token-level selection; the
// toolnavs.com summary, section "HySparse2 がやったこと"; the cnyes.com
// article, section "檢索精確到token"):
//   * KV Bridging: each bridged full-attention layer builds its own K and V
//     from the source layer's input hidden state X with its own projection.
//   * The block's full-attention layer attends densely (causal) over the
//     shared MQA cache and, from its attention scores, picks important
//     positions: 1024 global tokens from outside the window, plus the 128 most
//     recent tokens, which are always selected.
//   * The following sparse layers reuse that KV cache and those indices.
// Readings where the pages are silent (score aggregation = sum over heads of
// the causal softmax probability; ties to the lower index; window = the 128
// positions i-127..i; candidates j <= i-128; scale 1/sqrt(D); E4M3 with a
// per-token fp32 scale) are the ones this library documents for its C-ABI.
//
// Pins (tests marked "not gpu"): E4M3/bf16 codecs against torch's CPU casts;
// the projection against numpy matmul; attention against torch's float64
// softmax; the selection against a stable library sort and a brute-force rank
// count; closed forms (rows of probabilities sum to 1; sparse == dense when
// the context fits the budget; all-equal keys tie to indices 0..k-1).

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------- threads --
int g_threads_override = 0;

int n_threads() {
  if (g_threads_override > 0) return g_threads_override;
  if (const char* e = std::getenv("HS2O_THREADS")) {
    int v = std::atoi(e);
    if (v > 0) return v;
  }
  unsigned h = std::thread::hardware_concurrency();
  return h == 0 ? 1 : (int)h;
}

// Runs fn(i) for i in [0, n) on `threads` threads.  Work items are claimed
// from an atomic counter; every item's arithmetic is independent of which
// thread runs it, so results do not depend on the thread count.
void parallel_for(int64_t n, int threads, const std::function<void(int64_t)>& fn) {
  if (threads <= 1 || n <= 1) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  std::atomic<int64_t> next{0};
  auto worker = [&]() {
    for (;;) {
      int64_t i = next.fetch_add(1);
      if (i >= n) break;
      fn(i);
    }
  };
  int t = (int)std::min<int64_t>(threads, n);
  std::vector<std::thread> pool;
  for (int k = 1; k < t; ++k) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
}

// ------------------------------------------------------------------ codecs --
// bf16: 1 sign, 8 exponent (bias 127), 7 stored mantissa bits; the upper half
// of an IEEE binary32.
double bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// Nearest bf16 value, ties to even.  The spacing of bf16 values with binary
// exponent e (x = m * 2^e, 0.5 <= |m| < 1) is 2^(e-8); below the smallest
// normal (2^-126) it stays 2^-133.
uint16_t f64_to_bf16(double x) {
  if (std::isnan(x)) return 0x7FC0;
  if (x == 0.0) return std::signbit(x) ? 0x8000 : 0x0000;
  int e;
  std::frexp(x, &e);
  double ulp = std::ldexp(1.0, std::max(e, -125) - 8);
  double r = std::nearbyint(x / ulp) * ulp;  // default rounding mode: to nearest, ties to even
  float f = (float)r;                         // exact: r is a bf16 value (or overflows to inf)
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

// OCP 8-bit floating point, E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa.
// Exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there are
// no infinities; the largest finite magnitude is 1.75 * 2^8 = 448.
double e4m3_to_f64(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
  if (e == 15 && m == 7) return std::nan("");
  double mag = (e == 0) ? (m / 8.0) * std::ldexp(1.0, -6) : (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);
  return s ? -mag : mag;
}

// Round to the nearest finite E4M3 value, ties to the even code, saturating
// to +-448 ("satfinite"): searches all 127 non-negative finite codes.
uint8_t f64_to_e4m3(double x) {
  if (std::isnan(x)) return 0x7F;
  double a = std::fabs(x);
  int best = 0;
  double best_d = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double d = std::fabs(e4m3_to_f64((uint8_t)c) - a);
    if (d < best_d || (d == best_d && (c % 2) == 0)) {
      best = c;
      best_d = d;
    }
  }
  if (a > 448.0) best = 0x7E;
  return (uint8_t)(best | (std::signbit(x) ? 0x80 : 0));
}

// ------------------------------------------------------------- KV access --
struct Cache {
  int fp8;                // 0: bf16 bits, 1: E4M3 bytes with per-token scale
  const void* k;          // [B][L][D]
  const void* v;
  const float* k_scale;   // [B][L] (fp8 only)
  const float* v_scale;
  int64_t L;
  int D;

  double at(const void* base, const float* sc, int b, int64_t j, int d) const {
    int64_t off = ((int64_t)b * L + j) * D + d;
    if (fp8) return e4m3_to_f64(((const uint8_t*)base)[off]) * (double)sc[(int64_t)b * L + j];
    return bf16_to_f64(((const uint16_t*)base)[off]);
  }
  double key(int b, int64_t j, int d) const { return at(k, k_scale, b, j, d); }
  double val(int b, int64_t j, int d) const { return at(v, v_scale, b, j, d); }
};

// Selected set of query position i from head-summed scores score[0..i]:
// candidates C = {0 .. i-window}, ordered by (score descending, index
// ascending); the first min(topk, |C|) join the window {max(0,i-window+1) .. i};
// the union is written in ascending order and padded with -1.
void select_row(const double* score, int64_t i, int topk, int window, int32_t* idx_out,
                int32_t* n_sel_out) {
  std::vector<int64_t> cand;
  for (int64_t j = 0; j <= i - window; ++j) cand.push_back(j);
  std::sort(cand.begin(), cand.end(), [&](int64_t a, int64_t b) {
    if (score[a] != score[b]) return score[a] > score[b];
    return a < b;
  });
  std::vector<int64_t> sel(cand.begin(), cand.begin() + std::min<int64_t>(topk, (int64_t)cand.size()));
  for (int64_t j = std::max<int64_t>(0, i - window + 1); j <= i; ++j) sel.push_back(j);
  std::sort(sel.begin(), sel.end());
  int slots = topk + window;
  for (int n = 0; n < slots; ++n) idx_out[n] = n < (int)sel.size() ? (int32_t)sel[n] : -1;
  *n_sel_out = (int32_t)sel.size();
}

// Block-level selection, the granularity of the HySparse generation before
// HySparse2 (dpshk.com explainer, section 03: history chosen in blocks of 64
// tokens, so one useful token takes a whole block of the budget; cnyes.com
// article, section "檢索精確到token": the ablation keeps the same budget and
// compares block-level with token-level choice).  Readings where the pages are
// silent: the candidate positions are the token-level ones, C = {0 .. i-window};
// block b holds positions b*block .. b*block+block-1 and is a candidate when it
// holds a candidate position; its score is the sum of the head-summed scores of
// its candidate positions; blocks are ordered by (score descending, block index
// ascending) and the first min(topk / block, #candidate blocks) are selected;
// S = the candidate positions of the selected blocks, union the window, in
// ascending order, padded with -1 to topk + window slots.
void select_blocks_row(const double* score, int64_t i, int topk, int window, int block,
                       int32_t* idx_out, int32_t* n_sel_out) {
  const int64_t last = i - window;  // last candidate position (none when < 0)
  const int64_t nblk = last < 0 ? 0 : last / block + 1;
  std::vector<double> bsum((size_t)nblk, 0.0);
  for (int64_t j = 0; j <= last; ++j) bsum[(size_t)(j / block)] += score[j];
  std::vector<int64_t> order((size_t)nblk);
  for (int64_t b = 0; b < nblk; ++b) order[(size_t)b] = b;
  std::sort(order.begin(), order.end(), [&](int64_t a, int64_t b) {
    if (bsum[(size_t)a] != bsum[(size_t)b]) return bsum[(size_t)a] > bsum[(size_t)b];
    return b > a;  // equal sums: the lower block first
  });
  const int64_t keep = std::min<int64_t>(topk / block, nblk);
  std::vector<int64_t> sel;
  for (int64_t n = 0; n < keep; ++n) {
    const int64_t b = order[(size_t)n];
    for (int64_t j = b * block; j < std::min<int64_t>((b + 1) * block, last + 1); ++j)
      sel.push_back(j);
  }
  for (int64_t w = std::max<int64_t>(0, i - window + 1); w <= i; ++w) sel.push_back(w);
  std::sort(sel.begin(), sel.end());
  const int slots = topk + window;
  for (int n = 0; n < slots; ++n) idx_out[n] = n < (int)sel.size() ? (int32_t)sel[n] : -1;
  *n_sel_out = (int32_t)sel.size();
}

constexpr int64_t kChunk = 2048;  // fixed work-item size: keeps sums independent of threads

}  // namespace

extern "C" {

void hs2o_set_threads(int t) { g_threads_override = t; }
int hs2o_threads(void) { return n_threads(); }

double hs2o_bf16_to_f64(uint16_t b) { return bf16_to_f64(b); }
uint16_t hs2o_f64_to_bf16(double x) { return f64_to_bf16(x); }
double hs2o_e4m3_to_f64(uint8_t c) { return e4m3_to_f64(c); }
uint8_t hs2o_f64_to_e4m3(double x) { return f64_to_e4m3(x); }

// KV Bridging.  For the given token rows r of X [T][hidden] (bf16) and the
// projection Wt [n_layers*2*D][hidden] (bf16; row c holds output column c,
// with c = l*2D + d for K_l and l*2D + D + d for V_l):
//   Y[r][c]      = sum_k X[r][k] * Wt[c][k]                      (fp64)
//   out_bf16     = bf16 round-to-nearest-even of Y
//   out_fp8      = E4M3(Y / s), s = max_d |Y| / 448 per (token, layer, K|V),
//                  s = 1 when that maximum is 0
// Layouts: Y [n_rows][n_cols]; out_bf16 / out_fp8 [n_layers][2][n_rows][D];
// out_scale [n_layers][2][n_rows].  Any output pointer may be NULL.
int hs2o_bridge(const uint16_t* X, int64_t T, int hidden, const uint16_t* Wt, int n_layers, int D,
                const int64_t* rows, int64_t n_rows, double* Y, uint16_t* out_bf16,
                uint8_t* out_fp8, double* out_scale) {
  if (!X || !Wt || !rows || T < 1 || hidden < 1 || n_layers < 1 || D < 1 || n_rows < 0) return 1;
  const int n_cols = n_layers * 2 * D;
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= T) return 1;
  parallel_for(n_rows, n_threads(), [&](int64_t r) {
    const uint16_t* x = X + rows[r] * (int64_t)hidden;
    std::vector<double> xd(hidden), y(n_cols);
    for (int k = 0; k < hidden; ++k) xd[k] = bf16_to_f64(x[k]);
    for (int c = 0; c < n_cols; ++c) {
      const uint16_t* w = Wt + (int64_t)c * hidden;
      double acc = 0.0;
      for (int k = 0; k < hidden; ++k) acc += xd[k] * bf16_to_f64(w[k]);
      y[c] = acc;
    }
    if (Y) std::memcpy(Y + r * n_cols, y.data(), sizeof(double) * n_cols);
    for (int l = 0; l < n_layers; ++l) {
      for (int kv = 0; kv < 2; ++kv) {
        const double* seg = y.data() + l * 2 * D + kv * D;
        int64_t o = (((int64_t)l * 2 + kv) * n_rows + r) * D;
        if (out_bf16)
          for (int d = 0; d < D; ++d) out_bf16[o + d] = f64_to_bf16(seg[d]);
        double amax = 0.0;
        for (int d = 0; d < D; ++d) amax = std::max(amax, std::fabs(seg[d]));
        double s = amax > 0.0 ? amax / 448.0 : 1.0;
        if (out_scale) out_scale[((int64_t)l * 2 + kv) * n_rows + r] = s;
        if (out_fp8)
          for (int d = 0; d < D; ++d) out_fp8[o + d] = f64_to_e4m3(seg[d] / s);
      }
    }
  });
  return 0;
}

// Full-attention layer of a hybrid block, with token selection.
// Queries: Q [B][T][H][D] bf16; query t of sequence b sits at position
// i = L - T + t of that sequence's cache K, V [B][L][D] (bf16, or E4M3 times a
// per-token scale).  For each listed row r (rows[r] = b*T + t; rows == NULL
// means all B*T rows in order):
//   s_hj  = scale * sum_d q[h][d] * k_j[d]            for j <= i
//   p_hj  = exp(s_hj - m_h) / l_h,  m_h = max_j s_hj,  l_h = sum_j exp(s_hj - m_h)
//   lse_h = m_h + log l_h;  O[h][d] = sum_j p_hj v_j[d]
//   score_j = sum_h p_hj   (j <= i; 0 for j > i)
//   selection: select_row above.
// Layouts: O [n_rows][H][D]; lse [n_rows][H]; score [n_rows][L] (may be NULL);
// idx [n_rows][topk+window]; n_sel [n_rows].
int hs2o_full_attn_select(const uint16_t* Q, int kv_fp8, const void* K, const void* V,
                          const float* k_scale, const float* v_scale, int B, int T, int64_t L,
                          int H, int D, double scale, int topk, int window, const int64_t* rows,
                          int64_t n_rows, double* O, double* lse, double* score, int32_t* idx,
                          int32_t* n_sel) {
  if (!Q || !K || !V || B < 1 || T < 1 || L < T || H < 1 || D < 1 || topk < 0 || window < 1)
    return 1;
  if (kv_fp8 && (!k_scale || !v_scale)) return 1;
  if (!rows) n_rows = (int64_t)B * T;
  const Cache kv{kv_fp8, K, V, k_scale, v_scale, L, D};
  const int nt = n_threads();
  // Many short rows: one row per thread.  Few long rows: split each row.
  const bool row_parallel = n_rows >= 2 * nt && L * (int64_t)H <= (int64_t)1 << 22;
  auto run_row = [&](int64_t r, int inner_threads) {
    int64_t bt = rows ? rows[r] : r;
    int b = (int)(bt / T), t = (int)(bt % T);
    int64_t i = L - T + t, n = i + 1;
    std::vector<double> q((size_t)H * D);
    for (int h = 0; h < H; ++h)
      for (int d = 0; d < D; ++d) q[h * D + d] = bf16_to_f64(Q[((int64_t)bt * H + h) * D + d]);
    std::vector<double> p((size_t)H * n);  // logits, then probabilities, [H][n]
    int64_t nchunks = (n + kChunk - 1) / kChunk;
    parallel_for(nchunks, inner_threads, [&](int64_t c) {
      std::vector<double> kj(D);
      for (int64_t j = c * kChunk; j < std::min(n, (c + 1) * kChunk); ++j) {
        for (int d = 0; d < D; ++d) kj[d] = kv.key(b, j, d);
        for (int h = 0; h < H; ++h) {
          double acc = 0.0;
          for (int d = 0; d < D; ++d) acc += q[h * D + d] * kj[d];
          p[(size_t)h * n + j] = scale * acc;
        }
      }
    });
    std::vector<double> lse_row(H);
    parallel_for(H, inner_threads, [&](int64_t h) {
      double* ph = p.data() + (size_t)h * n;
      double m = -INFINITY;
      for (int64_t j = 0; j < n; ++j) m = std::max(m, ph[j]);
      double l = 0.0;
      for (int64_t j = 0; j < n; ++j) l += std::exp(ph[j] - m);
      for (int64_t j = 0; j < n; ++j) ph[j] = std::exp(ph[j] - m) / l;
      lse_row[h] = m + std::log(l);
    });
    std::vector<double> part((size_t)nchunks * H * D, 0.0);
    std::vector<double> sc(n);
    parallel_for(nchunks, inner_threads, [&](int64_t c) {
      std::vector<double> vj(D);
      double* acc = part.data() + (size_t)c * H * D;
      for (int64_t j = c * kChunk; j < std::min(n, (c + 1) * kChunk); ++j) {
        for (int d = 0; d < D; ++d) vj[d] = kv.val(b, j, d);
        double s = 0.0;
        for (int h = 0; h < H; ++h) {
          double pj = p[(size_t)h * n + j];
          s += pj;
          for (int d = 0; d < D; ++d) acc[h * D + d] += pj * vj[d];
        }
        sc[j] = s;
      }
    });
    if (O)
      for (int h = 0; h < H; ++h)
        for (int d = 0; d < D; ++d) {
          double o = 0.0;
          for (int64_t c = 0; c < nchunks; ++c) o += part[((size_t)c * H + h) * D + d];
          O[((size_t)r * H + h) * D + d] = o;
        }
    if (lse)
      for (int h = 0; h < H; ++h) lse[(size_t)r * H + h] = lse_row[h];
    if (score) {
      double* srow = score + (size_t)r * L;
      for (int64_t j = 0; j < L; ++j) srow[j] = j < n ? sc[j] : 0.0;
    }
    if (idx && n_sel)
      select_row(sc.data(), i, topk, window, idx + (size_t)r * (topk + window), n_sel + r);
  };
  if (row_parallel)
    parallel_for(n_rows, nt, [&](int64_t r) { run_row(r, 1); });
  else
    for (int64_t r = 0; r < n_rows; ++r) run_row(r, nt);
  return 0;
}

// One slice of a context held across several devices (context parallelism of
// the full-attention layer; the pages analyse contexts of a million tokens:
// dpshk.com explainer, section 05).  The slice holds L_slice consecutive
// positions of each sequence; query t sits at slice-relative position
// i = qpos + t (it may lie beyond the slice, or before it).  For each listed
// row (b, t) and head h, over the slice's keys j with 0 <= j < L_slice, j <= i:
//   s_hj = scale * <q_h, k_j>,  lse_h = log sum_j exp(s_hj)  (-inf if no key)
//   O_h  = sum_j exp(s_hj - lse_h) v_j                       (0 if no key)
//   score_j = sum_h exp(s_hj - lse_ref_h) for the slice's candidates
//             j <= i - window, where lse_ref = lse_in (the normaliser over the
//             whole context) when given, else the slice's own lse.
// Layouts as hs2o_full_attn_select: O [n_rows][H][D], lse [n_rows][H],
// score [n_rows][L_slice] (0 for non-candidates); lse_in [B*T][H].  With the
// slice = the whole cache (qpos = L - T) this is hs2o_full_attn_select's
// attention and score.
int hs2o_attn_slice(const uint16_t* Q, int kv_fp8, const void* K, const void* V,
                    const float* k_scale, const float* v_scale, int B, int T, int64_t L_slice,
                    int64_t qpos, int H, int D, double scale, int window, const double* lse_in,
                    const int64_t* rows, int64_t n_rows, double* O, double* lse, double* score) {
  if (!Q || !K || !V || B < 1 || T < 1 || L_slice < 1 || H < 1 || D < 1 || window < 1) return 1;
  if (kv_fp8 && (!k_scale || !v_scale)) return 1;
  if (!rows) n_rows = (int64_t)B * T;
  const Cache kv{kv_fp8, K, V, k_scale, v_scale, L_slice, D};
  parallel_for(n_rows, n_threads(), [&](int64_t r) {
    const int64_t bt = rows ? rows[r] : r;
    const int b = (int)(bt / T), t = (int)(bt % T);
    const int64_t i = qpos + t;
    const int64_t n = std::max<int64_t>(0, std::min<int64_t>(L_slice, i + 1));  // visible keys
    std::vector<double> s((size_t)H * std::max<int64_t>(n, 1));
    for (int64_t j = 0; j < n; ++j)
      for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
          acc += bf16_to_f64(Q[((int64_t)bt * H + h) * D + d]) * kv.key(b, j, d);
        s[(size_t)h * n + j] = scale * acc;
      }
    std::vector<double> lse_row(H, -INFINITY);
    for (int h = 0; h < H; ++h) {
      if (n == 0) continue;
      double m = -INFINITY;
      for (int64_t j = 0; j < n; ++j) m = std::max(m, s[(size_t)h * n + j]);
      double l = 0.0;
      for (int64_t j = 0; j < n; ++j) l += std::exp(s[(size_t)h * n + j] - m);
      lse_row[h] = std::log(l) + m;
    }
    if (lse)
      for (int h = 0; h < H; ++h) lse[(size_t)r * H + h] = lse_row[h];
    if (O)
      for (int h = 0; h < H; ++h)
        for (int d = 0; d < D; ++d) {
          double o = 0.0;
          for (int64_t j = 0; j < n; ++j)
            o += std::exp(s[(size_t)h * n + j] - lse_row[h]) * kv.val(b, j, d);
          O[((size_t)r * H + h) * D + d] = o;
        }
    if (score) {
      double* srow = score + (size_t)r * L_slice;
      for (int64_t j = 0; j < L_slice; ++j) srow[j] = 0.0;
      for (int64_t j = 0; j < n && j <= i - window; ++j) {
        double acc = 0.0;
        for (int h = 0; h < H; ++h) {
          const double ref = lse_in ? lse_in[(size_t)bt * H + h] : lse_row[h];
          acc += std::exp(s[(size_t)h * n + j] - ref);
        }
        srow[j] = acc;
      }
    }
  });
  return 0;
}

// Selection alone, from a caller-supplied score row score[0..i].
int hs2o_select(const double* score, int64_t i, int topk, int window, int32_t* idx,
                int32_t* n_sel) {
  if (!score || !idx || !n_sel || i < 0 || topk < 0 || window < 1) return 1;
  select_row(score, i, topk, window, idx, n_sel);
  return 0;
}

// Block-level selection alone, from a caller-supplied score row score[0..i]
// (select_blocks_row above).  topk must be a multiple of block.
int hs2o_select_blocks(const double* score, int64_t i, int topk, int window, int block,
                       int32_t* idx, int32_t* n_sel) {
  if (!score || !idx || !n_sel || i < 0 || topk < 0 || window < 1 || block < 1 ||
      topk % block != 0)
    return 1;
  select_blocks_row(score, i, topk, window, block, idx, n_sel);
  return 0;
}

// Sparse-attention layer with KV Reuse: attention of this layer's own queries
// Q [B][T][H][D] over the selected positions S = idx[row][0 .. n_sel[row]) of
// the same cache, softmax renormalised over S only:
//   O[h][d] = sum_{j in S} exp(s_hj - m_h) / l_h * v_j[d]
// idx/n_sel are laid out [B*T][slots] / [B*T]; rows as in hs2o_full_attn_select.
int hs2o_sparse_attn(const uint16_t* Q, int kv_fp8, const void* K, const void* V,
                     const float* k_scale, const float* v_scale, int B, int T, int64_t L, int H,
                     int D, double scale, const int32_t* idx, const int32_t* n_sel, int slots,
                     const int64_t* rows, int64_t n_rows, double* O) {
  if (!Q || !K || !V || !idx || !n_sel || !O || B < 1 || T < 1 || L < T || H < 1 || D < 1 ||
      slots < 1)
    return 1;
  if (kv_fp8 && (!k_scale || !v_scale)) return 1;
  if (!rows) n_rows = (int64_t)B * T;
  const Cache kv{kv_fp8, K, V, k_scale, v_scale, L, D};
  std::atomic<int> bad{0};
  parallel_for(n_rows, n_threads(), [&](int64_t r) {
    int64_t bt = rows ? rows[r] : r;
    int b = (int)(bt / T);
    int ns = n_sel[bt];
    const int32_t* sel = idx + bt * slots;
    if (ns < 0 || ns > slots) { bad = 1; return; }
    for (int n = 0; n < ns; ++n)
      if (sel[n] < 0 || sel[n] >= L) { bad = 1; return; }
    std::vector<double> kd((size_t)ns * D), vd((size_t)ns * D);
    for (int n = 0; n < ns; ++n)
      for (int d = 0; d < D; ++d) {
        kd[(size_t)n * D + d] = kv.key(b, sel[n], d);
        vd[(size_t)n * D + d] = kv.val(b, sel[n], d);
      }
    std::vector<double> pr(ns);
    for (int h = 0; h < H; ++h) {
      double m = -INFINITY;
      for (int n = 0; n < ns; ++n) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
          acc += bf16_to_f64(Q[((int64_t)bt * H + h) * D + d]) * kd[(size_t)n * D + d];
        pr[n] = scale * acc;
        m = std::max(m, pr[n]);
      }
      double l = 0.0;
      for (int n = 0; n < ns; ++n) l += std::exp(pr[n] - m);
      for (int n = 0; n < ns; ++n) pr[n] = std::exp(pr[n] - m) / l;
      for (int d = 0; d < D; ++d) {
        double o = 0.0;
        for (int n = 0; n < ns; ++n) o += pr[n] * vd[(size_t)n * D + d];
        O[((size_t)r * H + h) * D + d] = o;
      }
    }
  });
  return bad.load();
}

}  // extern "C"
