// gemv.cuh -- W8A16 for a single token on the CUDA cores.
//
// With one token the W8A16 product is a matrix-vector product: two
// operations per weight byte, well within the CUDA cores, so the weight
// stream is the whole cost and the tensor-core path's set-up, conversion ring
// and split-K reduction are overhead.  Each CTA owns whole output rows (all
// of K), so no partial sums cross CTAs.
//
// Arithmetic: the token is turned once into a 32-bit fixed-point image,
// v_k = rint(x_k * 2^sh) with sh = 157 - e, e the bf16 exponent field of
// max|x| (so |v_k| < 2^31; every x_k within 23 binades of the largest is
// exact, smaller ones are rounded to the nearest 2^-sh).  v_k is split into
// three unsigned bytes and a signed top byte, and each weight row is dotted
// with the four byte planes by dp4a: four signed codes times four bytes into
// an int32, exactly.  The planes' sums are combined exactly in int64 and
// summed over lanes and warps in int64, so the dot product is exact and
// independent of the order; y = bf16(fp64(sum) * s_ch * 2^-sh), two
// roundings (the fp64 product and the bf16 conversion), like the oracle's
// fp64 sum times s_ch rounded to bf16.  One dp4a per four codes and plane,
// so four integer instructions per four codes, against nine for an exact
// int8-to-fp32 conversion with packed fp32 FMAs.  A token holding inf or NaN
// has no fixed-point image: every output is then NaN.
//
// Rows are dealt to the CTAs round-robin (CTA b takes rows b, b + G, b + 2G,
// ...), so at any moment the CTAs read neighbouring rows and the chip sweeps
// the weight matrix front to back.  A producer lane brings two rows per
// shared-memory stage with 1-D bulk copies and keeps about 96 KB in flight
// per SM; each compute warp works on both rows of a stage at once, so the
// two lane reductions overlap (one row per stage measured 1.4 us slower per
// 89 MB call, four rows per stage spill registers).  Compute thread c owns
// four 16-byte chunks of K, c, c + T, c + 2T and c + 3T (T compute
// threads), so a warp's shared-memory reads are contiguous and free of bank
// conflicts, and holds the four byte planes of the matching 64 token values
// in registers.
#pragma once
#include "ptx.cuh"

namespace sq {

struct GemvLayout {
  int S;          // shared-memory stages (kGemvRows weight rows each)
  int nwc;        // compute warps
  int rows_max;   // most rows one CTA owns
  int off_part;   // int64 [rows_max][nwc] warp sums
  int off_ring;   // int8 [S][kGemvRows][K]
  int smem;       // dynamic shared memory bytes
};

constexpr int kGemvChunks = 4;                  // 16-byte chunks of K per compute thread
constexpr int kGemvCodes = 16 * kGemvChunks;    // codes of K per compute thread
constexpr int kGemvMaxThreads = 512;            // up to 15 compute warps: K <= 30720
constexpr int kGemvMaxStages = 16;
constexpr int kGemvRows = 2;                    // weight rows per stage
constexpr int kGemvInFlight = 98304;            // bytes of weights in flight per CTA

// The layout for N rows of K codes over `grid` CTAs, or S = 0 when it does
// not fit (K / 64 compute threads plus the producer warp must fit 512, and
// two stages plus the warp sums must fit shared memory).
inline GemvLayout gemv_layout(int64_t N, int64_t K, int grid) {
  GemvLayout l{};
  if (K <= 0 || K % 128 || grid <= 0) return l;
  const int64_t threads = (K / 16 + kGemvChunks - 1) / kGemvChunks;
  l.nwc = static_cast<int>((threads + 31) / 32);
  l.rows_max = static_cast<int>((N + grid - 1) / grid);
  if (l.nwc * 32 + 32 > kGemvMaxThreads) return l;
  l.off_part = 512;  // barriers and the abort flag first
  const int64_t off_ring =
      (l.off_part + static_cast<int64_t>(l.rows_max) * l.nwc * 8 + 127) / 128 * 128;
  const int64_t cap = 232448 - 128;
  if (off_ring >= cap) return l;
  l.off_ring = static_cast<int>(off_ring);
  const int64_t stage = kGemvRows * K;
  int64_t s = (kGemvInFlight + stage - 1) / stage;
  if (s < 2) s = 2;
  if (s > kGemvMaxStages) s = kGemvMaxStages;
  if (s > (cap - off_ring) / stage) s = (cap - off_ring) / stage;
  l.S = static_cast<int>(s < 2 ? 0 : s);
  l.smem = l.off_ring + l.S * static_cast<int>(stage) + 128;
  return l;
}


// Exact 4-way dot products: signed codes times unsigned or signed bytes.
__device__ __forceinline__ int dp4a_su(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// The K limit of the layout (480 compute threads x 64 codes = 30720) keeps
// |sum| <= K * 127 * 2^31 below 2^53, so the fp64 conversion of the exact
// sum is exact.
static_assert((kGemvMaxThreads - 32) * kGemvCodes * 127.0 * 2147483648.0 < 9007199254740992.0,
              "exact fp64 image of the dot product");

__global__ void __launch_bounds__(kGemvMaxThreads, 1)
    w8a16_gemv_kernel(const __nv_bfloat16* __restrict__ x, const int8_t* __restrict__ q,
                      const float* __restrict__ s_ch, __nv_bfloat16* __restrict__ y, int N, int K,
                      GemvLayout l) {
  extern __shared__ uint8_t gsm_raw[];
  uint8_t* gsm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(gsm_raw) + 127) & ~static_cast<uintptr_t>(127));
  const int S = l.S, nwc = l.nwc;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  uint64_t* full = reinterpret_cast<uint64_t*>(gsm);
  uint64_t* empty = full + kGemvMaxStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + 256);
  unsigned* xmax = reinterpret_cast<unsigned*>(gsm + 260);  // max |x| bf16 bits
  long long* part = reinterpret_cast<long long*>(gsm + l.off_part);
  uint8_t* ring = gsm + l.off_ring;
  const int G = gridDim.x, b = blockIdx.x;
  const int nrows = b < N ? (N - b + G - 1) / G : 0;  // rows b, b + G, ...
  const int nst = (nrows + kGemvRows - 1) / kGemvRows;  // stages this CTA consumes

  griddep_launch_dependents();
  if (t == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, nwc);
    }
    *abort_flag = 0;
    *xmax = 0u;
    fence_mbar_init();
  }
  float sc0 = 1.0f;  // a compute thread's first row scale, used at the end
  __syncthreads();

  if (warp == nwc) {
    // ------------------------------------------------------ weight producer
    // The weights are not written by a preceding kernel (the overlap
    // contract), so they stream before griddep_wait.
    if (lane == 0) {
      int fills = 0, s = 0;
      uint32_t ph = 0;  // phase of stage s's next fill
      for (int it = 0; it < nst; ++it) {
        // a stage is refilled once every compute warp holds its last rows' codes
        if (it >= S && !wait_bounded(empty + s, ph ^ 1u, abort_flag)) break;
        const int rin = nrows - it * kGemvRows < kGemvRows ? nrows - it * kGemvRows : kGemvRows;
        mbar_arrive_expect_tx(full + s, static_cast<uint32_t>(rin * K));
        for (int r = 0; r < rin; ++r)
          bulk_load(ring + (static_cast<size_t>(s) * kGemvRows + r) * K,
                    q + (static_cast<size_t>(b) + static_cast<size_t>(it * kGemvRows + r) * G) * K,
                    static_cast<uint32_t>(K), full + s);
        ++fills;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      // no copy may still be writing shared memory when the CTA exits
      for (int i = fills - S < 0 ? 0 : fills - S; i < fills; ++i)
        wait_drain(full + i % S, static_cast<uint32_t>((i / S) & 1));
    }
  } else {
    // ------------------------------------------------------ compute warps
    griddep_wait();  // the token and the scales may come from the preceding kernel
    if (t < nrows) sc0 = __ldg(s_ch + b + static_cast<size_t>(t) * G);  // requested early
    const int T = nwc * 32;
    const int chunks = K / 16;
    uint4 xr[kGemvChunks][2];  // this thread's 64 token values, bf16
    unsigned m = 0u;
#pragma unroll
    for (int j = 0; j < kGemvChunks; ++j) {
      const int c = j * T + t;
      xr[j][0] = xr[j][1] = make_uint4(0u, 0u, 0u, 0u);
      if (c < chunks) {
        const uint4* xp = reinterpret_cast<const uint4*>(x) + 2 * static_cast<size_t>(c);
        xr[j][0] = __ldg(xp);
        xr[j][1] = __ldg(xp + 1);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t w[4] = {xr[j][h].x, xr[j][h].y, xr[j][h].z, xr[j][h].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          m = max(m, w[e] & 0x7FFFu);
          m = max(m, (w[e] >> 16) & 0x7FFFu);
        }
      }
    }
    m = __reduce_max_sync(0xffffffffu, m);
    if (lane == 0) atomicMax(xmax, m);
    named_bar_sync(1, T);
    const int e_max = static_cast<int>((*xmax >> 7) & 0xFFu);
    const int sh = 157 - e_max;
    // 2^sh built from its fp64 bit pattern (sh lies in [-97, 157])
    const double scale = __longlong_as_double(static_cast<long long>(1023 + sh) << 52);
    // the byte planes: pl[p][4j+e] holds byte p of the fixed-point values of
    // the four token values that meet code word e of chunk j (values 4e ..
    // 4e+3 of the chunk, in bf16 words 2e and 2e+1)
    uint32_t pl[4][4 * kGemvChunks];
#pragma unroll
    for (int j = 0; j < kGemvChunks; ++j) {
      const uint32_t xw[8] = {xr[j][0].x, xr[j][0].y, xr[j][0].z, xr[j][0].w,
                              xr[j][1].x, xr[j][1].y, xr[j][1].z, xr[j][1].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t hv[4] = {xw[2 * e] & 0xFFFFu, xw[2 * e] >> 16, xw[2 * e + 1] & 0xFFFFu,
                                xw[2 * e + 1] >> 16};
        uint32_t planes[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t v = static_cast<uint32_t>(
              __double2int_rn(static_cast<double>(__uint_as_float(hv[u] << 16)) * scale));
#pragma unroll
          for (int p = 0; p < 4; ++p) planes[p] |= ((v >> (8 * p)) & 0xFFu) << (8 * u);
        }
#pragma unroll
        for (int p = 0; p < 4; ++p) pl[p][4 * j + e] = planes[p];
      }
    }
    int s = 0;
    uint32_t ph = 0;
    for (int it = 0; it < nst; ++it) {
      if (!warp_wait_bounded(full + s, ph, abort_flag)) break;
      const uint4* rp = reinterpret_cast<const uint4*>(ring + static_cast<size_t>(s) * kGemvRows * K);
      // codes of the stage's rows (a missing last row reads stale codes and
      // is not stored); codes past K read as 0 (their byte planes are 0 too)
      uint4 v[kGemvRows][kGemvChunks];
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
        for (int j = 0; j < kGemvChunks; ++j) {
          const int c = j * T + t;
          v[r][j] = c < chunks ? rp[r * chunks + c] : make_uint4(0u, 0u, 0u, 0u);
        }
      // the stage is free once every compute warp holds its codes (the
      // arrive orders this warp's loads before it)
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);
      if (++s == S) { s = 0; ph ^= 1u; }
      long long sum[kGemvRows];
#pragma unroll
      for (int r = 0; r < kGemvRows; ++r) {
        int acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};  // two chains per byte plane
#pragma unroll
        for (int j = 0; j < kGemvChunks; ++j) {
          const uint32_t w[4] = {v[r][j].x, v[r][j].y, v[r][j].z, v[r][j].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            int* a = acc[e & 1];
            a[0] = dp4a_su(w[e], pl[0][4 * j + e], a[0]);
            a[1] = dp4a_su(w[e], pl[1][4 * j + e], a[1]);
            a[2] = dp4a_su(w[e], pl[2][4 * j + e], a[2]);
            a[3] = dp4a_ss(w[e], pl[3][4 * j + e], a[3]);
          }
        }
        sum[r] = (static_cast<long long>(acc[0][3] + acc[1][3]) << 24) +
                 (static_cast<long long>(acc[0][2] + acc[1][2]) << 16) +
                 (static_cast<long long>(acc[0][1] + acc[1][1]) << 8) +
                 static_cast<long long>(acc[0][0] + acc[1][0]);
      }
      // the rows' lane sums, reduced side by side
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int r = 0; r < kGemvRows; ++r) sum[r] += __shfl_xor_sync(0xffffffffu, sum[r], off);
      if (lane == 0)
#pragma unroll
        for (int r = 0; r < kGemvRows; ++r)
          if (it * kGemvRows + r < nrows) part[(it * kGemvRows + r) * nwc + warp] = sum[r];
    }
  }
  __syncthreads();
  if (*abort_flag) return;
  const int e_max = static_cast<int>((*xmax >> 7) & 0xFFu);
  const bool finite = e_max != 0xFF;
  const double unscale = __longlong_as_double(static_cast<long long>(1023 - (157 - e_max)) << 52);
  // each row: the exact sum over warps, times s_ch and 2^-sh, rounded once to bf16
  for (int i = t; i < nrows; i += blockDim.x) {
    long long sum = 0;
    for (int w = 0; w < nwc; ++w) sum += part[i * nwc + w];
    const size_t row = static_cast<size_t>(b) + static_cast<size_t>(i) * G;
    const float sc = (i == t && warp < nwc) ? sc0 : __ldg(s_ch + row);
    const double r = static_cast<double>(sum) * static_cast<double>(sc) * unscale;
    y[row] = finite ? __double2bfloat16(r) : __ushort_as_bfloat16(0x7FC0u);
  }
}

}  // namespace sq
