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
#include <limits>
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

// ---- exact sum of squares of bf16 values -------------------------------
// A bf16 value is m * 2^e with an integer 0 <= m <= 255 and e in [-133, 120];
// its square m^2 * 2^(2e) has 2e in [-266, 240].  The sum is kept exactly as
// a 576-bit integer A with value A * 2^-266 (9 limbs of 64 bits, limb 0
// lowest), which holds every sum of up to 2^30 squares.
struct SumSq {
  uint64_t limb[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};

  void add_shifted(uint64_t v, int shift) {  // A += v << shift, v < 2^16
    int li = shift / 64, bi = shift % 64;
    unsigned __int128 t = static_cast<unsigned __int128>(v) << bi;
    uint64_t parts[2] = {static_cast<uint64_t>(t), static_cast<uint64_t>(t >> 64)};
    uint64_t carry = 0;
    for (int i = li; i < 9; ++i) {
      uint64_t add = (i - li < 2 ? parts[i - li] : 0);
      unsigned __int128 sum = static_cast<unsigned __int128>(limb[i]) + add + carry;
      limb[i] = static_cast<uint64_t>(sum);
      carry = static_cast<uint64_t>(sum >> 64);
      if (i - li >= 1 && carry == 0) break;
    }
  }

  void add_bf16_square(uint16_t h) {
    const int E = (h >> 7) & 0xFF;
    const uint32_t f = h & 0x7F;
    if (E == 0xFF) return;  // Inf / NaN: outside the defined inputs
    const uint32_t m = E ? (128u + f) : f;
    if (m == 0) return;
    const int e = (E ? E : 1) - 134;
    add_shifted(static_cast<uint64_t>(m) * m, 2 * e + 266);
  }

  int bit(int pos) const { return static_cast<int>((limb[pos / 64] >> (pos % 64)) & 1u); }

  bool any_below(int pos) const {  // any set bit at positions < pos
    for (int i = 0; i < 9 && i * 64 < pos; ++i) {
      const int hi = pos - i * 64;
      const uint64_t mask = hi >= 64 ? ~0ull : ((1ull << hi) - 1);
      if (limb[i] & mask) return true;
    }
    return false;
  }

  // A * 2^-266 rounded to the nearest fp32, ties to even.
  float to_f32() const {
    int top = -1;
    for (int i = 8; i >= 0 && top < 0; --i)
      if (limb[i]) top = i * 64 + 63 - __builtin_clzll(limb[i]);
    if (top < 0) return 0.0f;
    // last kept bit: 24 significant bits, but never below 2^-149 (bit 117)
    const int lsb = std::max(top - 23, 117);
    uint64_t mant = 0;
    for (int pos = top; pos >= lsb; --pos) mant = (mant << 1) | static_cast<uint64_t>(bit(pos));
    const bool round = lsb >= 1 && bit(lsb - 1);
    const bool sticky = lsb >= 2 && any_below(lsb - 1);
    if (round && (sticky || (mant & 1u))) ++mant;
    return std::ldexp(static_cast<float>(mant), lsb - 266);  // exact (or inf)
  }
};

// ---- OCP E4M3 ------------------------------------------------------------
// Finite values: normals (1 + f/8) * 2^(E-7), E = 1..15 (E = 15, f = 7 is
// NaN), subnormals f/8 * 2^-6.  Largest finite 448 = 1.75 * 2^8.
float e4m3_to_f32(uint8_t b) {
  const int sign = (b >> 7) & 1;
  const int E = (b >> 3) & 0xF;
  const int f = b & 7;
  if (E == 15 && f == 7) return std::numeric_limits<float>::quiet_NaN();
  float v = E == 0 ? std::ldexp(static_cast<float>(f), -9)
                   : std::ldexp(static_cast<float>(8 + f), E - 10);
  return sign ? -v : v;
}

uint8_t f32_to_e4m3(float v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t sign = std::signbit(v) ? 0x80 : 0;
  const float a = std::fabs(v);
  if (a >= 448.0f) return static_cast<uint8_t>(sign | 0x7E);   // saturate to 448
  if (a == 0.0f) return sign;
  int e = 0;
  std::frexp(a, &e);                   // a = f * 2^e, f in [0.5, 1)
  int qe = e - 4;                      // weight of the last of 4 significant bits
  if (qe < -9) qe = -9;                // subnormal spacing 2^-9
  const float n = std::nearbyint(std::ldexp(a, -qe));   // exact scaling, RNE
  const float r = std::ldexp(n, qe);                    // the rounded magnitude
  // encode r (exactly representable; r <= 448)
  if (r == 0.0f) return sign;
  int re = 0;
  std::frexp(r, &re);                  // r = f * 2^re
  uint8_t bits;
  if (re - 1 < -6) {                   // subnormal: r = f/8 * 2^-6
    bits = static_cast<uint8_t>(std::ldexp(r, 9));
  } else {
    const int E = re - 1 + 7;
    const int f = static_cast<int>(std::ldexp(r, -(re - 1)) * 8.0f) - 8;
    bits = static_cast<uint8_t>((E << 3) | f);
  }
  return static_cast<uint8_t>(sign | bits);
}

// FP8 codes of n fp32 values with one scale (amax / 448).
float quant_block_fp8(const float* v, int64_t n, uint8_t* q) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) amax = std::max(amax, std::fabs(v[i]));
  if (amax == 0.0f) {
    for (int64_t i = 0; i < n; ++i) q[i] = 0;
    return 0.0f;
  }
  const float scale = amax / 448.0f;
  const float mult = 448.0f / amax;
  for (int64_t i = 0; i < n; ++i) q[i] = f32_to_e4m3(v[i] * mult);
  return scale;
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

// ---------------------------------------------------------------------------
// Fused RMSNorm + fold + quantisation (see the header for the steps).

int oracle_fold_norm_weight(const uint16_t* w, int64_t K, int zero_centered,
                            const float* inv_s, float* gamma) {
  if (K < 0 || (K && (!w || !gamma))) return -1;
  for (int64_t k = 0; k < K; ++k) {
    float g = bf16_to_f32(w[k]);
    if (zero_centered) g = 1.0f + g;
    gamma[k] = inv_s ? g * inv_s[k] : g;
  }
  return 0;
}

float oracle_sumsq_f32(const uint16_t* h, int64_t n) {
  SumSq acc;
  for (int64_t i = 0; i < n; ++i) acc.add_bf16_square(h[i]);
  return acc.to_f32();
}

int oracle_rmsnorm_quant(const uint16_t* h, int64_t M, int64_t K, const float* gamma,
                         float eps, int64_t group, const float* r_in, int8_t* q,
                         float* scales, float* r_out) {
  if (M < 0 || K <= 0 || !(eps > 0.0f)) return -1;
  if (group != K && group != 128) return -1;
  if (K % group) return -2;
  if (M && (!h || !gamma || !q || !scales)) return -1;
  const int64_t nblk = K / group;
  parallel_for(M, [&](int64_t m) {
    const uint16_t* row = h + m * K;
    float r;
    if (r_in) {
      r = r_in[m];
    } else {
      const float ss = oracle_sumsq_f32(row, K);
      const float ms = ss / static_cast<float>(K);
      const float d = std::sqrt(ms + eps);
      r = 1.0f / d;
    }
    if (r_out) r_out[m] = r;
    std::vector<float> v(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) {
      float t = bf16_to_f32(row[k]) * r;
      v[k] = t * gamma[k];
    }
    for (int64_t b = 0; b < nblk; ++b)
      scales[m * nblk + b] = quant_block(v.data() + b * group, group, q + m * K + b * group);
  });
  return 0;
}

// ---------------------------------------------------------------------------
// Per-group (1 x 128) activations with gs128 weights.

int oracle_quant_per_group(const uint16_t* x, int64_t M, int64_t K, const float* inv_s,
                           int8_t* q, float* s_a) {
  const int64_t G = 128;
  if (M < 0 || K < 0 || (K % G)) return -1;
  if (M * K && (!x || !q || !s_a)) return -1;
  const int64_t nblk = K / G;
  parallel_for(M, [&](int64_t m) {
    std::vector<float> v(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) {
      float t = bf16_to_f32(x[m * K + k]);
      v[k] = inv_s ? t * inv_s[k] : t;
    }
    for (int64_t b = 0; b < nblk; ++b)
      s_a[m * nblk + b] = quant_block(v.data() + b * G, G, q + m * K + b * G);
  });
  return 0;
}

int oracle_pg128_mm(const int8_t* q_a, const float* s_a, const int8_t* q_w,
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
        int32_t part = 0;
        for (int64_t k = kb * G; k < (kb + 1) * G; ++k)
          part += static_cast<int32_t>(a[k]) * static_cast<int32_t>(b[k]);
        const float sc = s_a[m * nkb + kb] * s_blk[n * nkb + kb];
        acc = std::fmaf(static_cast<float>(part), sc, acc);
      }
      y[r * N + n] = f32_to_bf16(acc);
    }
  });
  return 0;
}

// ---------------------------------------------------------------------------
// Group-wise W8A16 (reconstructed 16-bit weights).

int oracle_dequant_weight_group(const int8_t* q_w, const float* s_grp, int64_t N, int64_t K,
                                uint16_t* w_hat) {
  const int64_t G = 128;
  if (N < 0 || K < 0 || (K % G)) return -1;
  if (N * K && (!q_w || !s_grp || !w_hat)) return -1;
  const int64_t nkb = K / G;
  parallel_for(N, [&](int64_t n) {
    for (int64_t k = 0; k < K; ++k) {
      const float p = static_cast<float>(q_w[n * K + k]) * s_grp[n * nkb + k / G];
      w_hat[n * K + k] = f32_to_bf16(p);
    }
  });
  return 0;
}

int oracle_w8a16_group_mm(const uint16_t* x, const int8_t* q_w, const float* s_grp,
                          int64_t M, int64_t N, int64_t K, const int64_t* rows,
                          int64_t nrows, uint16_t* y, double* abs_out) {
  const int64_t G = 128;
  if (M < 0 || N < 0 || K < 0 || (K % G) || !rows_ok(rows, nrows, M)) return -1;
  std::vector<uint16_t> w_hat(static_cast<size_t>(N * K));
  if (oracle_dequant_weight_group(q_w, s_grp, N, K, w_hat.data()) != 0) return -1;
  parallel_for(nrows, [&](int64_t r) {
    const int64_t m = row_of(rows, r);
    for (int64_t n = 0; n < N; ++n) {
      double sum = 0.0, mag = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        const double p = static_cast<double>(bf16_to_f32(x[m * K + k])) *
                         static_cast<double>(bf16_to_f32(w_hat[n * K + k]));  // exact
        sum += p;
        mag += std::fabs(p);
      }
      y[r * N + n] = f64_to_bf16(sum);
      if (abs_out) abs_out[r * N + n] = mag;
    }
  });
  return 0;
}

// ---------------------------------------------------------------------------
// FP8 (E4M3) block-scaled weights with per-group activations.

uint8_t oracle_f32_to_e4m3(float v) { return f32_to_e4m3(v); }
float oracle_e4m3_to_f32(uint8_t b) { return e4m3_to_f32(b); }

int oracle_quant_fp8_per_group(const uint16_t* x, int64_t M, int64_t K, const float* inv_s,
                               uint8_t* q, float* s_a) {
  const int64_t G = 128;
  if (M < 0 || K < 0 || (K % G)) return -1;
  if (M * K && (!x || !q || !s_a)) return -1;
  const int64_t nblk = K / G;
  parallel_for(M, [&](int64_t m) {
    std::vector<float> v(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) {
      float t = bf16_to_f32(x[m * K + k]);
      v[k] = inv_s ? t * inv_s[k] : t;
    }
    for (int64_t b = 0; b < nblk; ++b)
      s_a[m * nblk + b] = quant_block_fp8(v.data() + b * G, G, q + m * K + b * G);
  });
  return 0;
}

int oracle_quant_fp8_block(const uint16_t* w, int64_t N, int64_t K, const float* smooth,
                           uint8_t* q, float* s_w) {
  const int64_t G = 128;
  if (N < 0 || K < 0 || (N % G) || (K % G)) return -1;
  if (N * K && (!w || !q || !s_w)) return -1;
  const int64_t nbn = N / G, nbk = K / G;
  parallel_for(nbn * nbk, [&](int64_t blk) {
    const int64_t bn = blk / nbk, bk = blk % nbk;
    std::vector<float> v(static_cast<size_t>(G * G));
    for (int64_t i = 0; i < G; ++i)
      for (int64_t j = 0; j < G; ++j) {
        const int64_t n = bn * G + i, k = bk * G + j;
        float t = bf16_to_f32(w[n * K + k]);
        v[i * G + j] = smooth ? t * smooth[k] : t;
      }
    std::vector<uint8_t> qb(static_cast<size_t>(G * G));
    s_w[bn * nbk + bk] = quant_block_fp8(v.data(), G * G, qb.data());
    for (int64_t i = 0; i < G; ++i)
      for (int64_t j = 0; j < G; ++j) q[(bn * G + i) * K + bk * G + j] = qb[i * G + j];
  });
  return 0;
}

int oracle_fp8_block_mm(const uint8_t* q_a, const float* s_a, const uint8_t* q_w,
                        const float* s_w, int64_t M, int64_t N, int64_t K,
                        const int64_t* rows, int64_t nrows, uint16_t* y, double* abs_out) {
  const int64_t G = 128;
  if (M < 0 || N < 0 || K < 0 || (N % G) || (K % G) || !rows_ok(rows, nrows, M)) return -1;
  const int64_t nkb = K / G;
  // decoded weights (each code's exact value), decoded once
  std::vector<double> wd(static_cast<size_t>(N * K));
  parallel_for(N, [&](int64_t n) {
    for (int64_t k = 0; k < K; ++k) wd[n * K + k] = e4m3_to_f32(q_w[n * K + k]);
  });
  parallel_for(nrows, [&](int64_t r) {
    const int64_t m = row_of(rows, r);
    std::vector<double> a(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) a[k] = e4m3_to_f32(q_a[m * K + k]);
    for (int64_t n = 0; n < N; ++n) {
      double sum = 0.0, mag = 0.0;
      for (int64_t kb = 0; kb < nkb; ++kb) {
        double part = 0.0, pmag = 0.0;   // exact: products have 8 significant bits
        for (int64_t k = kb * G; k < (kb + 1) * G; ++k) {
          const double p = a[k] * wd[n * K + k];
          part += p;
          pmag += std::fabs(p);
        }
        const float sc = s_a[m * nkb + kb] * s_w[(n / G) * nkb + kb];
        sum += part * static_cast<double>(sc);
        mag += pmag * std::fabs(static_cast<double>(sc));
      }
      y[r * N + n] = f64_to_bf16(sum);
      if (abs_out) abs_out[r * N + n] = mag;
    }
  });
  return 0;
}

}  // extern "C"
