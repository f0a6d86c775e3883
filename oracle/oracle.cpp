// oracle.cpp — fp64 CPU reference of split-KV decode attention.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
// benchmark's CPU-baseline leg load this library; the product path never
// does, and this file shares no code, header or constant with the CUDA
// library.  It is plain and slow on purpose: every loop runs in the order of
// the definition it restates, in fp64, with no blocking or fusion.
//
// What it computes ("What is Flash-Decoding, and when does it speed up
// LLMs?", slavadubrov.com: the opening paragraph and the section "Why decode
// needs a different schedule"): the output that attention over the complete
// cached history gives for one new query token.  For query head
// h of sequence b, with KV head kv = floor(h / G), G = Hq / Hkv, and n valid
// cached tokens:
//     s_j = sc * sum_d q_d K_{j,d}            j < n,  sc = (double)scale
//     m   = max_j s_j
//     Z   = sum_j exp(s_j - m)
//     O_d = sum_j exp(s_j - m) V_{j,d} / Z
//     lse = m + ln Z                          (natural log of sum_j exp(s_j))
// n = 0 gives O = 0 and lse = -inf.
//
// oracle_attend_split restates the split schedule of the same page ("Why
// decode needs a different schedule": each unit of the split history yields
// a partial output and a log-sum-exp, and a reduction combines them into
// the full-history result):
//     chunk s covers tokens [s*C, min((s+1)*C, n))
//     O_s, lse_s = the definition above over that chunk (O_s normalised)
//     M = max_s lse_s,  w_s = exp(lse_s - M)
//     O = sum_s w_s O_s / sum_s w_s,   lse = M + ln sum_s w_s
//
// Inputs are bf16 bit patterns (uint16), widened exactly to double, or fp64
// values (dequantised caches whose real values need not be bf16).
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

double bf16_to_double(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

double load(const uint16_t* p, long i) { return bf16_to_double(p[i]); }
double load(const double* p, long i) { return p[i]; }

// One query head against n cached rows.  k and v are row-major [n, D] with
// row stride `ld` elements.
template <class T>
void attend_one_head(long n, int D, const T* q, const T* k, const T* v, long ld, double sc,
                     double* out, double* lse) {
  const double ninf = -std::numeric_limits<double>::infinity();
  if (n <= 0) {
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    *lse = ninf;
    return;
  }
  std::vector<double> s(static_cast<size_t>(n));
  for (long j = 0; j < n; ++j) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += load(q, d) * load(k, j * ld + d);
    s[j] = sc * dot;
  }
  double m = ninf;
  for (long j = 0; j < n; ++j) m = s[j] > m ? s[j] : m;
  double Z = 0.0;
  for (long j = 0; j < n; ++j) Z += std::exp(s[j] - m);
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (long j = 0; j < n; ++j) {
    double p = std::exp(s[j] - m);
    for (int d = 0; d < D; ++d) out[d] += p * load(v, j * ld + d);
  }
  for (int d = 0; d < D; ++d) out[d] /= Z;
  *lse = m + std::log(Z);
}

// Split-then-combine for one query head, chunk length C > 0.
void attend_split_one_head(long n, int D, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, long ld, double sc, long C,
                           double* out, double* lse, double* part_o,
                           double* part_lse, long max_parts) {
  const double ninf = -std::numeric_limits<double>::infinity();
  long S = n > 0 ? (n + C - 1) / C : 0;
  std::vector<double> o_s(static_cast<size_t>(S) * D);
  std::vector<double> l_s(static_cast<size_t>(S));
  for (long s = 0; s < S; ++s) {
    long begin = s * C;
    long end = (s + 1) * C < n ? (s + 1) * C : n;
    attend_one_head(end - begin, D, q, k + begin * ld, v + begin * ld, ld, sc,
                    &o_s[static_cast<size_t>(s) * D], &l_s[s]);
  }
  if (part_o && part_lse) {
    for (long s = 0; s < max_parts; ++s) {
      for (int d = 0; d < D; ++d) part_o[s * D + d] = s < S ? o_s[s * D + d] : 0.0;
      part_lse[s] = s < S ? l_s[s] : ninf;
    }
  }
  double M = ninf;
  for (long s = 0; s < S; ++s) M = l_s[s] > M ? l_s[s] : M;
  if (S == 0 || M == ninf) {
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    *lse = ninf;
    return;
  }
  double W = 0.0;
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (long s = 0; s < S; ++s) {
    double w = std::exp(l_s[s] - M);
    W += w;
    for (int d = 0; d < D; ++d) out[d] += w * o_s[s * D + d];
  }
  for (int d = 0; d < D; ++d) out[d] /= W;
  *lse = M + std::log(W);
}

template <class F>
void parallel_for(long count, int nthreads, F f) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > count) nthreads = static_cast<int>(count > 0 ? count : 1);
  std::atomic<long> next{0};
  auto worker = [&]() {
    for (long i = next.fetch_add(1); i < count; i = next.fetch_add(1)) f(i);
  };
  std::vector<std::thread> pool;
  for (int t = 1; t < nthreads; ++t) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// The same with fp64 inputs and an fp64 scale.
void oracle_attend_f64(long n, int D, int G, const double* q, const double* k,
                       const double* v, long ld, double scale, double* out, double* lse) {
  for (int g = 0; g < G; ++g)
    attend_one_head(n, D, q + static_cast<long>(g) * D, k, v, ld, scale,
                    out + static_cast<long>(g) * D, lse + g);
}

// G query heads that share one KV head: q [G, D]; k, v [n, ld] row-major.
void oracle_attend(long n, int D, int G, const uint16_t* q, const uint16_t* k,
                   const uint16_t* v, long ld, float scale, double* out,
                   double* lse) {
  for (int g = 0; g < G; ++g)
    attend_one_head(n, D, q + static_cast<long>(g) * D, k, v, ld,
                    static_cast<double>(scale), out + static_cast<long>(g) * D,
                    lse + g);
}

// Split-then-combine with chunk C; optional per-split outputs
// part_o [G, max_parts, D] and part_lse [G, max_parts].
void oracle_attend_split(long n, int D, int G, const uint16_t* q,
                         const uint16_t* k, const uint16_t* v, long ld,
                         float scale, long C, double* out, double* lse,
                         double* part_o, double* part_lse, long max_parts) {
  for (int g = 0; g < G; ++g)
    attend_split_one_head(
        n, D, q + static_cast<long>(g) * D, k, v, ld, static_cast<double>(scale), C,
        out + static_cast<long>(g) * D, lse + g,
        part_o ? part_o + static_cast<long>(g) * max_parts * D : nullptr,
        part_lse ? part_lse + static_cast<long>(g) * max_parts : nullptr, max_parts);
}

// Whole batch, contiguous cache: q [B, Hq, D]; k, v [B, Hkv, max_len, D];
// seqlens [B] (NULL: every sequence holds max_len tokens; values are clamped
// to [0, max_len]); out [B, Hq, D]; lse [B, Hq].  Runs (b, h) pairs on
// `nthreads` threads.  Returns 0, or -1 if Hq is not a multiple of Hkv.
int oracle_decode(int B, int Hq, int Hkv, int D, long max_len, const uint16_t* q,
                  const uint16_t* k, const uint16_t* v, const int32_t* seqlens,
                  float scale, double* out, double* lse, int nthreads) {
  if (Hkv <= 0 || Hq % Hkv != 0) return -1;
  const int G = Hq / Hkv;
  parallel_for(static_cast<long>(B) * Hq, nthreads, [&](long i) {
    const long b = i / Hq, h = i % Hq, kv = h / G;
    long n = seqlens ? seqlens[b] : max_len;
    if (n < 0) n = 0;
    if (n > max_len) n = max_len;
    const long base = (b * Hkv + kv) * max_len * D;
    attend_one_head(n, D, q + i * D, k + base, v + base, D,
                    static_cast<double>(scale), out + i * D, lse + i);
  });
  return 0;
}

}  // extern "C"
