// sq_oracle.cpp -- CPU oracle for the SmoothQuant W8A8 INT8 linear layer.
//
// TEST INFRASTRUCTURE ONLY (see sq_oracle.h for who may load it, the page
// sections each function follows and the readings taken where the pages are
// silent).  Plain loops over the definitions; the only liberty taken is
// splitting independent output rows/columns across host threads, which does
// not change any arithmetic.  Build with -ffp-contract=off and without fast
// math so every float operation rounds exactly once, as written.
#include "sq_oracle.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <functional>
#include <thread>
#include <vector>

namespace {

int g_threads = 0;

int thread_count() {
  if (g_threads > 0) return g_threads;
  unsigned h = std::thread::hardware_concurrency();
  return h ? static_cast<int>(h) : 1;
}

// Run body(i) for i in [0, n) over the worker threads, handing out indices
// in small chunks.
void parallel_for(int64_t n, const std::function<void(int64_t)>& body) {
  int nt = thread_count();
  if (n <= 0) return;
  if (nt <= 1 || n == 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  nt = static_cast<int>(std::min<int64_t>(nt, n));
  std::atomic<int64_t> next{0};
  auto worker = [&]() {
    for (;;) {
      int64_t i = next.fetch_add(1);
      if (i >= n) break;
      body(i);
    }
  };
  std::vector<std::thread> pool;
  for (int t = 1; t < nt; ++t) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
}

float bf16_to_f32(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint16_t f32_to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return static_cast<uint16_t>((u >> 16) | 0x40u);
  // Round to nearest, ties to even, on the 16 discarded bits.
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

// Exact rounding of a double to BF16 (8 significant bits), ties to even.
uint16_t f64_to_bf16(double d) {
  if (std::isnan(d)) return 0x7FC0;
  uint16_t sign = std::signbit(d) ? 0x8000 : 0;
  double a = std::fabs(d);
  if (a == 0.0) return sign;
  if (std::isinf(a)) return static_cast<uint16_t>(sign | 0x7F80);
  int e = 0;
  std::frexp(a, &e);            // a = f * 2^e, f in [0.5, 1)
  int qe = e - 8;               // weight of the last kept bit (normals)
  if (qe < -133) qe = -133;     // subnormal BF16 spacing is 2^-133
  double r = std::nearbyint(std::ldexp(a, -qe));   // RNE, exact scaling
  double v = std::ldexp(r, qe);
  if (v >= 0x1p128) return static_cast<uint16_t>(sign | 0x7F80);
  float f = static_cast<float>(v);  // exact: v has <= 8 significant bits
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>(sign | (u >> 16));
}

// Symmetric INT8 code of one value given the fp32 multiplier 127/amax.
int8_t quant_code(float v, float mult) {
  float t = v * mult;                    // one fp32 rounding
  float r = std::nearbyint(t);           // round half to even
  if (r > 127.0f) r = 127.0f;
  if (r < -127.0f) r = -127.0f;
  return static_cast<int8_t>(r);
}

// Quantise n values (already in fp32) with one symmetric scale.
float quant_block(const float* v, int64_t n, int8_t* q) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) amax = std::max(amax, std::fabs(v[i]));
  if (amax == 0.0f) {
    for (int64_t i = 0; i < n; ++i) q[i] = 0;
    return 0.0f;
  }
  float scale = amax / 127.0f;
  float mult = 127.0f / amax;
  for (int64_t i = 0; i < n; ++i) q[i] = quant_code(v[i], mult);
  return scale;
}

int64_t row_of(const int64_t* rows, int64_t r) { return rows ? rows[r] : r; }

bool rows_ok(const int64_t* rows, int64_t nrows, int64_t M) {
  if (nrows < 0) return false;
  if (!rows) return nrows == M;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= M) return false;
  return true;
}

}  // namespace

extern "C" {

uint16_t oracle_f32_to_bf16(float f) { return f32_to_bf16(f); }
uint16_t oracle_f64_to_bf16(double d) { return f64_to_bf16(d); }
float oracle_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }

void oracle_set_threads(int n) { g_threads = n; }
int oracle_get_threads(void) { return thread_count(); }

int oracle_smooth_factors(const uint16_t* x, int64_t M, int64_t K, const uint16_t* w,
                          int64_t N, double cap, double floor_, float* s_out,
                          float* inv_s_out) {
  if (M < 0 || N < 0 || K < 0 || !s_out || !inv_s_out) return -1;
  if ((M && !x) || (N && !w)) return -1;
  parallel_for(K, [&](int64_t j) {
    double mx = 0.0, mw = 0.0;
    for (int64_t m = 0; m < M; ++m) mx = std::max(mx, (double)std::fabs(bf16_to_f32(x[m * K + j])));
    for (int64_t n = 0; n < N; ++n) mw = std::max(mw, (double)std::fabs(bf16_to_f32(w[n * K + j])));
    double s;
    if (mx == 0.0 && mw == 0.0) s = 1.0;
    else if (mw == 0.0) s = cap;
    else s = std::sqrt(mx) / std::sqrt(mw);       // alpha = 1/2
    s = std::min(cap, std::max(floor_, s));
    float sf = static_cast<float>(s);
    s_out[j] = sf;
    inv_s_out[j] = static_cast<float>(1.0 / static_cast<double>(sf));
  });
  return 0;
}

int oracle_fold_weight(const uint16_t* w, int64_t N, int64_t K, const float* s,
                       float* w_folded) {
  if (N < 0 || K < 0 || (N * K && (!w || !w_folded))) return -1;
  parallel_for(N, [&](int64_t n) {
    for (int64_t k = 0; k < K; ++k) {
      float v = bf16_to_f32(w[n * K + k]);
      w_folded[n * K + k] = s ? v * s[k] : v;
    }
  });
  return 0;
}

int oracle_quant_weight(const uint16_t* w, int64_t N, int64_t K, const float* s,
                        int64_t group, int8_t* q, float* scales) {
  if (N < 0 || K < 0 || group < 0) return -1;
  if (group && (K % group)) return -2;
  if (N * K && (!w || !q || !scales)) return -1;
  const int64_t g = group ? group : K;
  const int64_t nblk = (K && g) ? K / g : 0;
  parallel_for(N, [&](int64_t n) {
    std::vector<float> row(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) {
      float v = bf16_to_f32(w[n * K + k]);
      row[k] = s ? v * s[k] : v;
    }
    for (int64_t b = 0; b < nblk; ++b)
      scales[n * nblk + b] = quant_block(row.data() + b * g, g, q + n * K + b * g);
  });
  return 0;
}

int oracle_quant_per_token(const uint16_t* x, int64_t M, int64_t K, const float* inv_s,
                           int8_t* q, float* s_tok) {
  if (M < 0 || K < 0) return -1;
  if (M && (!x || !q || !s_tok)) return -1;
  parallel_for(M, [&](int64_t m) {
    std::vector<float> row(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) {
      float v = bf16_to_f32(x[m * K + k]);
      row[k] = inv_s ? v * inv_s[k] : v;          // the 1/s fold, one rounding
    }
    s_tok[m] = quant_block(row.data(), K, q + m * K);
  });
  return 0;
}

int oracle_mm_i32(const int8_t* q_a, const int8_t* q_w, int64_t M, int64_t N, int64_t K,
                  const int64_t* rows, int64_t nrows, int32_t* acc) {
  if (M < 0 || N < 0 || K < 0 || !rows_ok(rows, nrows, M)) return -1;
  parallel_for(nrows, [&](int64_t r) {
    const int8_t* a = q_a + row_of(rows, r) * K;
    for (int64_t n = 0; n < N; ++n) {
      const int8_t* b = q_w + n * K;
      int32_t sum = 0;
      for (int64_t k = 0; k < K; ++k) sum += static_cast<int32_t>(a[k]) * static_cast<int32_t>(b[k]);
      acc[r * N + n] = sum;
    }
  });
  return 0;
}

int oracle_epilogue_ch(const int32_t* acc, const float* s_tok, const float* s_ch,
                       int64_t nrows, int64_t N, uint16_t* y) {
  if (nrows < 0 || N < 0) return -1;
  parallel_for(nrows, [&](int64_t r) {
    for (int64_t n = 0; n < N; ++n) {
      float v = static_cast<float>(acc[r * N + n]);   // int32 -> f32, RNE
      v = v * s_tok[r];
      v = v * s_ch[n];
      y[r * N + n] = f32_to_bf16(v);
    }
  });
  return 0;
}

int oracle_w8a8_scaled_mm(const int8_t* q_a, const float* s_tok, const int8_t* q_w,
                          const float* s_ch, int64_t M, int64_t N, int64_t K,
                          const int64_t* rows, int64_t nrows, uint16_t* y) {
  if (M < 0 || N < 0 || K < 0 || !rows_ok(rows, nrows, M)) return -1;
  parallel_for(nrows, [&](int64_t r) {
    const int64_t m = row_of(rows, r);
    const int8_t* a = q_a + m * K;
    for (int64_t n = 0; n < N; ++n) {
      const int8_t* b = q_w + n * K;
      int32_t sum = 0;
      for (int64_t k = 0; k < K; ++k) sum += static_cast<int32_t>(a[k]) * static_cast<int32_t>(b[k]);
      float v = static_cast<float>(sum);
      v = v * s_tok[m];
      v = v * s_ch[n];
      y[r * N + n] = f32_to_bf16(v);
    }
  });
  return 0;
}

int oracle_gs128_mm(const int8_t* q_a, const float* s_tok, const int8_t* q_w,
                    const float* s_blk, int64_t M, int64_t N, int64_t K,
                    const int64_t* rows, int64_t nrows, uint16_t* y) {
  const int64_t G = 128;
  if (M < 0 || N < 0 || K < 0 || (K % G) || !rows_ok(rows, nrows, M)) return -1;
  const int64_t nkb = K / G;
  parallel_for(nrows, [&](int64_t r) {
    const int64_t m = row_of(rows, r);
    const int8_t* a = q_a + m * K;
    for (int64_t n = 0; n < N; ++n) {
      const int8_t* b = q_w + n * K;
      float acc = 0.0f;
      for (int64_t kb = 0; kb < nkb; ++kb) {
        int32_t part = 0;                      // exact block partial
        for (int64_t k = kb * G; k < (kb + 1) * G; ++k)
          part += static_cast<int32_t>(a[k]) * static_cast<int32_t>(b[k]);
        acc = std::fmaf(static_cast<float>(part), s_blk[n * nkb + kb], acc);
      }
      y[r * N + n] = f32_to_bf16(acc * s_tok[m]);
    }
  });
  return 0;
}

int oracle_w8a16_mm(const uint16_t* x, const int8_t* q_w, const float* s_ch, int64_t M,
                    int64_t N, int64_t K, const int64_t* rows, int64_t nrows, uint16_t* y,
                    double* abs_out) {
  if (M < 0 || N < 0 || K < 0 || !rows_ok(rows, nrows, M)) return -1;
  parallel_for(nrows, [&](int64_t r) {
    const int64_t m = row_of(rows, r);
    std::vector<double> xr(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) xr[k] = static_cast<double>(bf16_to_f32(x[m * K + k]));
    for (int64_t n = 0; n < N; ++n) {
      const int8_t* b = q_w + n * K;
      double sum = 0.0, mag = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = xr[k] * static_cast<double>(b[k]);   // exact product
        sum += p;
        mag += std::fabs(p);
      }
      const double sc = static_cast<double>(s_ch[n]);
      y[r * N + n] = f64_to_bf16(sum * sc);
      if (abs_out) abs_out[r * N + n] = mag * sc;
    }
  });
  return 0;
}

}  // extern "C"
