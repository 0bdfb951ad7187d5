// quant.cuh -- HBM-bound kernels: per-token dynamic INT8 quantisation with
// the SmoothQuant 1/s fold, symmetric weight quantisation (per channel or per
// 128-wide K block), SmoothQuant factors from calibration maxima, and the
// exact int8 -> bf16 weight conversion used by the W8A16 path.
//
// Arithmetic (the rounding sequence the oracle states): v = f32(x) * vec[k]
// (one fp32 rounding), amax = max |v|, scale = amax / 127 (IEEE fp32
// division), code = clamp(rint(v * (127 / amax)), -127, 127) with
// round-half-even; amax == 0 gives scale 0 and zero codes.
#pragma once
#include <cuda_fp8.h>

#include "ptx.cuh"

namespace sq {

__device__ __forceinline__ __nv_bfloat162 u32_as_bf162(uint32_t v) {
  __nv_bfloat162 r;
  memcpy(&r, &v, 4);
  return r;
}
__device__ __forceinline__ uint32_t bf162_as_u32(__nv_bfloat162 v) {
  uint32_t r;
  memcpy(&r, &v, 4);
  return r;
}

// Exact conversion of four packed int8 codes to four bf16 values, eight
// instructions for four codes.  A byte b is l - 128 s with l = b & 127 and s
// its sign bit.  The bf16 pattern 0x43 : l reads 2^7 + l (exponent 2^7,
// mantissa l) and 0x43 : (s << 7) reads 2^7 + 2^7 s, so one packed bf16
// subtraction per two codes gives b.  Every operand and result is an integer
// of at most eight significant bits, so the subtraction is exact.
__device__ __forceinline__ void i8x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t l = w & 0x7F7F7F7Fu;
  const uint32_t s = w & 0x80808080u;
  const __nv_bfloat162 a0 = u32_as_bf162(__byte_perm(l, 0x43434343u, 0x4140));
  const __nv_bfloat162 a1 = u32_as_bf162(__byte_perm(l, 0x43434343u, 0x4342));
  const __nv_bfloat162 b0 = u32_as_bf162(__byte_perm(s, 0x43434343u, 0x4140));
  const __nv_bfloat162 b1 = u32_as_bf162(__byte_perm(s, 0x43434343u, 0x4342));
  lo = bf162_as_u32(__hsub2(a0, b0));
  hi = bf162_as_u32(__hsub2(a1, b1));
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ int quant_code(float v, float mult) {
  int c = __float2int_rn(__fmul_rn(v, mult));
  return max(-127, min(127, c));
}

// Low byte of the code rint(v * mult) for |v * mult| < 2^22: adding 1.5 * 2^23
// moves the product into [2^23, 2^24), where the float spacing is 1, so the
// addition itself rounds half-to-even to an integer held in the low mantissa
// bits; the low byte is the two's-complement byte of that integer.  With
// |v| <= amax and mult = fp32(127 / amax), |v * mult| <= 127 * (1 + 2^-24)^2,
// which rounds to at most 127, so no clamp is needed (equal to quant_code).
__device__ __forceinline__ uint32_t quant_byte_bits(float v, float mult) {
  return __float_as_uint(__fadd_rn(__fmul_rn(v, mult), 12582912.0f));
}
// Pack the low bytes of four such patterns into one word (element 0 lowest).
__device__ __forceinline__ uint32_t pack_code_bytes(uint32_t a, uint32_t b, uint32_t c,
                                                    uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Quantise `nseg` segments of `group` contiguous elements of the row-major
// [rows, K] BF16 matrix x, each with its own symmetric scale.  TPR threads
// cooperate on one segment, 16 elements per thread per step (two 128-bit
// loads of x, one 128-bit store of codes).  vec (fp32 [K], optional)
// multiplies element k before quantisation.
template <int TPR, bool HAS_VEC>
__global__ void __launch_bounds__(256) quant_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const float* __restrict__ vec,
                                                         int8_t* __restrict__ q,
                                                         float* __restrict__ scales,
                                                         int64_t nseg, int K, int group) {
  constexpr int SEGS = 256 / TPR;
  __shared__ float red[8];
  const int t = threadIdx.x % TPR;
  const int64_t seg = static_cast<int64_t>(blockIdx.x) * SEGS + threadIdx.x / TPR;
  const bool active = seg < nseg;
  const int64_t base = active ? seg * group : 0;
  const int kofs = static_cast<int>(base % K);

  float amax = 0.0f;
  if (active) {
    for (int c = t * 16; c < group; c += TPR * 16) {
      const uint4* px = reinterpret_cast<const uint4*>(x + base + c);
      float f[16];
      bf16x8_to_f32(__ldg(px), *reinterpret_cast<float(*)[8]>(&f[0]));
      bf16x8_to_f32(__ldg(px + 1), *reinterpret_cast<float(*)[8]>(&f[8]));
      if (HAS_VEC) {
        const float4* pv = reinterpret_cast<const float4*>(vec + kofs + c);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 s = __ldg(pv + j);
          f[4 * j] = __fmul_rn(f[4 * j], s.x);
          f[4 * j + 1] = __fmul_rn(f[4 * j + 1], s.y);
          f[4 * j + 2] = __fmul_rn(f[4 * j + 2], s.z);
          f[4 * j + 3] = __fmul_rn(f[4 * j + 3], s.w);
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(f[j]));
    }
  }
  // reduce over the TPR threads of the segment
#pragma unroll
  for (int off = (TPR < 32 ? TPR : 32) / 2; off > 0; off >>= 1)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (TPR > 32) {
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < TPR / 32; ++w) amax = fmaxf(amax, red[w]);
  }
  if (!active) return;

  const float scale = __fdiv_rn(amax, 127.0f);
  const float mult = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  if (t == 0) scales[seg] = scale;
  for (int c = t * 16; c < group; c += TPR * 16) {
    const uint4* px = reinterpret_cast<const uint4*>(x + base + c);
    float f[16];
    bf16x8_to_f32(__ldg(px), *reinterpret_cast<float(*)[8]>(&f[0]));
    bf16x8_to_f32(__ldg(px + 1), *reinterpret_cast<float(*)[8]>(&f[8]));
    if (HAS_VEC) {
      const float4* pv = reinterpret_cast<const float4*>(vec + kofs + c);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 s = __ldg(pv + j);
        f[4 * j] = __fmul_rn(f[4 * j], s.x);
        f[4 * j + 1] = __fmul_rn(f[4 * j + 1], s.y);
        f[4 * j + 2] = __fmul_rn(f[4 * j + 2], s.z);
        f[4 * j + 3] = __fmul_rn(f[4 * j + 3], s.w);
      }
    }
    uint32_t pk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t b0 = static_cast<uint8_t>(quant_code(f[4 * j], mult));
      const uint32_t b1 = static_cast<uint8_t>(quant_code(f[4 * j + 1], mult));
      const uint32_t b2 = static_cast<uint8_t>(quant_code(f[4 * j + 2], mult));
      const uint32_t b3 = static_cast<uint8_t>(quant_code(f[4 * j + 3], mult));
      pk[j] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    }
    *reinterpret_cast<uint4*>(q + base + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// Modes of the streaming kernel (bit set):
//   QM_NORM  : RMSNorm first.  ss = sum of f32(h)^2 accumulated in fp64 (each
//              square exact) and rounded once to fp32; r = 1 / sqrt(ss/K + eps)
//              with IEEE fp32 division and square root; the value quantised is
//              (f32(h) * r) * vec[k] (vec = the norm weight with 1/s folded in).
//   QM_GROUP : one scale per 128 columns instead of one per row.
//   QM_FP8   : OCP E4M3 codes (scale = amax / 448, saturating RNE conversion)
//              instead of INT8 codes.
enum : int { QM_NORM = 1, QM_GROUP = 2, QM_FP8 = 4 };

// E4M3 codes of two fp32 values (element 0 in the low byte), RNE, saturating.
__device__ __forceinline__ uint32_t e4m3x2_bits(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// Persistent streaming variant.  A row group of TPR threads (1 or 2 warps)
// owns CH chunks of 16 columns per thread, keeps the 1/s factors (or the
// folded norm weight) of those columns in registers for its whole life, and
// streams its rows through a ring of S shared-memory stages filled by 1-D
// bulk copies (one row per stage), so the copy engine keeps S rows per group
// in flight while the threads compute.  Per row: absmax pass and coding pass
// both read the row from shared memory; codes leave in 128-bit stores.  Same
// arithmetic as quant_rows_kernel.  A 128-column group is 8 chunks owned by 8
// adjacent lanes, so per-group maxima need three shuffles.
template <int TPR, int CH, int G, bool HAS_VEC, int MODE = 0>
__global__ void __launch_bounds__(TPR * G) quant_stream_kernel(const __nv_bfloat16* __restrict__ x,
                                                               const float* __restrict__ vec,
                                                               int8_t* __restrict__ q,
                                                               float* __restrict__ scales,
                                                               int64_t nrows, int K, int S,
                                                               float eps = 0.0f,
                                                               float* __restrict__ r_out = nullptr) {
  constexpr int NW = TPR / 32;
  constexpr bool NORM = (MODE & QM_NORM) != 0;
  constexpr bool GROUP = (MODE & QM_GROUP) != 0;
  constexpr bool FP8 = (MODE & QM_FP8) != 0;
  constexpr float QMAX = FP8 ? 448.0f : 127.0f;
  extern __shared__ __align__(128) uint8_t qsm[];
  const int g = threadIdx.x / TPR;            // row group within the block
  const int t = threadIdx.x % TPR;
  const int lane = threadIdx.x & 31;
  const int wig = t >> 5;                     // warp within the group
  const size_t row_bytes = static_cast<size_t>(K) * 2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(qsm);                 // [G][S]
  float* red = reinterpret_cast<float*>(qsm + G * S * 8);            // [G][NW]
  double* red_d = reinterpret_cast<double*>(qsm + 512);              // [G][NW] (NORM)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(qsm + G * S * 8 + G * NW * 4);
  uint8_t* ring = qsm + 1024 + static_cast<size_t>(g) * S * row_bytes;
  uint64_t* full = bars + g * S;
  const int ngrp = K / 128;

  const int64_t group = static_cast<int64_t>(blockIdx.x) * G + g;
  const int64_t ngroups = static_cast<int64_t>(gridDim.x) * G;
  griddep_launch_dependents();  // a dependent GEMM may start its prologue

  if (threadIdx.x == 0) {
    for (int i = 0; i < G * S; ++i) mbar_init(bars + i, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // this thread's 1/s factors (or folded norm weights), kept in registers
  float v[CH][16];
#pragma unroll
  for (int j = 0; j < CH; ++j) {
    const int c = (j * TPR + t) * 16;
#pragma unroll
    for (int i = 0; i < 16; ++i) v[j][i] = 1.0f;
    if (HAS_VEC && c < K) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 s4 = __ldg(reinterpret_cast<const float4*>(vec + c) + i);
        v[j][4 * i] = s4.x;
        v[j][4 * i + 1] = s4.y;
        v[j][4 * i + 2] = s4.z;
        v[j][4 * i + 3] = s4.w;
      }
    }
  }

  // prologue: the first S rows of this group
  int issued = 0;
  if (t == 0) {
    for (int i = 0; i < S; ++i) {
      const int64_t r = group + static_cast<int64_t>(i) * ngroups;
      if (r >= nrows) break;
      mbar_arrive_expect_tx(full + i, static_cast<uint32_t>(row_bytes));
      bulk_load(ring + i * row_bytes, x + r * K, static_cast<uint32_t>(row_bytes), full + i);
      ++issued;
    }
  }
  const int bar_id = 1 + g;
  int stage = 0;
  uint32_t phase = 0;
  for (int64_t r = group, i = 0; r < nrows; r += ngroups, ++i) {
    const bool ok = wait_bounded(full + stage, phase, abort_flag);
    if (named_bar_or(bar_id, TPR, !ok)) break;
    const uint8_t* row = ring + stage * row_bytes;
    // RMSNorm factor of this row (NORM), identical in every thread of the group
    float rn = 1.0f;
    if constexpr (NORM) {
      double ss = 0.0;
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        const int c = (j * TPR + t) * 16;
        if (c < K) {
          float f[16];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + 2 * c), *reinterpret_cast<float(*)[8]>(&f[0]));
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + 2 * c + 16), *reinterpret_cast<float(*)[8]>(&f[8]));
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const double d = static_cast<double>(f[k]);
            ss = __fma_rn(d, d, ss);
          }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (NW > 1) {
        if (lane == 0) red_d[g * NW + wig] = ss;
        named_bar_sync(bar_id, TPR);
        ss = 0.0;
#pragma unroll
        for (int w = 0; w < NW; ++w) ss += red_d[g * NW + w];
      }
      const float ms = __fdiv_rn(__double2float_rn(ss), static_cast<float>(K));
      rn = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
      if (r_out && t == 0) r_out[r] = rn;
    }
    auto value = [&](float h, float vk) {
      if constexpr (NORM) return __fmul_rn(__fmul_rn(h, rn), vk);
      else return HAS_VEC ? __fmul_rn(h, vk) : h;
    };
    // absmax: of the row (per token), or of each chunk's 128-column group
    float amax = 0.0f;
    float gmax[CH];
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int c = (j * TPR + t) * 16;
      float m = 0.0f;
      if (c < K) {
        float f[16];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + 2 * c), *reinterpret_cast<float(*)[8]>(&f[0]));
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + 2 * c + 16), *reinterpret_cast<float(*)[8]>(&f[8]));
#pragma unroll
        for (int k = 0; k < 16; ++k) m = fmaxf(m, fabsf(value(f[k], v[j][k])));
      }
      if constexpr (GROUP) {
        // the 8 lanes 8a .. 8a+7 hold the 8 chunks of one 128-column group
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        gmax[j] = m;
      } else {
        amax = fmaxf(amax, m);
      }
    }
    if constexpr (!GROUP) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if (NW > 1) {
        if (lane == 0) red[g * NW + wig] = amax;
        named_bar_sync(bar_id, TPR);
#pragma unroll
        for (int w = 0; w < NW; ++w) amax = fmaxf(amax, red[g * NW + w]);
      }
      if (t == 0) scales[r] = __fdiv_rn(amax, QMAX);
    }
    int8_t* qr = q + r * K;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int c = (j * TPR + t) * 16;
      if (c < K) {
        const float am = GROUP ? gmax[j] : amax;
        const float mult = am > 0.0f ? __fdiv_rn(QMAX, am) : 0.0f;
        if (GROUP && (t & 7) == 0) scales[r * ngrp + c / 128] = __fdiv_rn(am, QMAX);
        float f[16];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + 2 * c), *reinterpret_cast<float(*)[8]>(&f[0]));
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + 2 * c + 16), *reinterpret_cast<float(*)[8]>(&f[8]));
        uint32_t pk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float xv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) xv[e] = value(f[4 * k + e], v[j][4 * k + e]);
          if constexpr (FP8) {
            const uint32_t lo = e4m3x2_bits(__fmul_rn(xv[0], mult), __fmul_rn(xv[1], mult));
            const uint32_t hi = e4m3x2_bits(__fmul_rn(xv[2], mult), __fmul_rn(xv[3], mult));
            pk[k] = am > 0.0f ? (lo | (hi << 16)) : 0u;  // an all-zero group: zero codes
          } else {
            pk[k] = pack_code_bytes(quant_byte_bits(xv[0], mult), quant_byte_bits(xv[1], mult),
                                    quant_byte_bits(xv[2], mult), quant_byte_bits(xv[3], mult));
          }
        }
        *reinterpret_cast<uint4*>(qr + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
    // every thread of the group is done with this stage (and with red[])
    named_bar_sync(bar_id, TPR);
    if (t == 0) {
      const int64_t rn2 = r + static_cast<int64_t>(S) * ngroups;
      if (rn2 < nrows) {
        mbar_arrive_expect_tx(full + stage, static_cast<uint32_t>(row_bytes));
        bulk_load(ring + stage * row_bytes, x + rn2 * K, static_cast<uint32_t>(row_bytes), full + stage);
        ++issued;
      }
    }
    if (++stage == S) { stage = 0; phase ^= 1u; }
  }
  // no copy may still be writing shared memory when the block exits
  if (t == 0) {
    for (int st = 0; st < S; ++st) {
      const int n = issued / S + (st < issued % S ? 1 : 0);
      if (n > 0) wait_drain(full + st, static_cast<uint32_t>((n - 1) & 1));
    }
  }
}

// Column maxima of |a| (BF16 [rows, K]) folded into out_bits[k] with an
// unsigned atomic max on the fp32 bit pattern (monotonic for values >= 0).
// Thread layout: 8 columns per thread (one 128-bit load), ROWS rows per block.
__global__ void __launch_bounds__(256) colmax_kernel(const __nv_bfloat16* __restrict__ a,
                                                     int64_t rows, int K, int rows_per_block,
                                                     unsigned int* __restrict__ out_bits) {
  const int col8 = blockIdx.x * blockDim.x + threadIdx.x;
  if (col8 * 8 >= K) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_block;
  const int64_t r1 = min(rows, r0 + rows_per_block);
  float m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int64_t r = r0; r < r1; ++r) {
    float f[8];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(a + r * K) + col8), f);
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = fmaxf(m[j], fabsf(f[j]));
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) atomicMax(out_bits + col8 * 8 + j, __float_as_uint(m[j]));
}

// s = clamp(sqrt(mx) / sqrt(mw), floor, cap) in fp64 (both square roots and
// the quotient correctly rounded), with the zero-maximum cases of the
// interface; the maxima arrive as fp32 bit patterns in the output buffers.
__global__ void smooth_finalize_kernel(float* __restrict__ s_out, float* __restrict__ inv_out,
                                       int K, double cap, double floor_) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const double mx = static_cast<double>(__uint_as_float(reinterpret_cast<unsigned*>(s_out)[j]));
  const double mw = static_cast<double>(__uint_as_float(reinterpret_cast<unsigned*>(inv_out)[j]));
  double s;
  if (mx == 0.0 && mw == 0.0) s = 1.0;
  else if (mw == 0.0) s = cap;
  else s = __ddiv_rn(__dsqrt_rn(mx), __dsqrt_rn(mw));
  s = fmin(cap, fmax(floor_, s));
  const float sf = __double2float_rn(s);
  s_out[j] = sf;
  inv_out[j] = __double2float_rn(__ddiv_rn(1.0, static_cast<double>(sf)));
}

// Exact int8 -> bf16 conversion of n codes (n % 16 == 0), 16 per thread-step.
__global__ void __launch_bounds__(256) i8_to_bf16_kernel(const int8_t* __restrict__ q,
                                                         __nv_bfloat16* __restrict__ out,
                                                         int64_t n16) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(q) + i);
    uint4 o0, o1;
    i8x4_to_bf16x4(w.x, o0.x, o0.y);
    i8x4_to_bf16x4(w.y, o0.z, o0.w);
    i8x4_to_bf16x4(w.z, o1.x, o1.y);
    i8x4_to_bf16x4(w.w, o1.z, o1.w);
    uint4* po = reinterpret_cast<uint4*>(out) + 2 * i;
    po[0] = o0;
    po[1] = o1;
  }
}

// Group-scaled reconstruction of four packed int8 codes: bf16(f32(q) * s),
// the fp32 product rounded once, then RNE to bf16 (two roundings).
__device__ __forceinline__ void i8x4_scale_to_bf16x4(uint32_t w, float s, uint32_t& lo,
                                                     uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const float bias = 8388736.0f;  // 2^23 + 128
  const float f0 = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)), bias);
  const float f1 = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541)), bias);
  const float f2 = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)), bias);
  const float f3 = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543)), bias);
  lo = pack_bf16x2(__fmul_rn(f0, s), __fmul_rn(f1, s));
  hi = pack_bf16x2(__fmul_rn(f2, s), __fmul_rn(f3, s));
}

// Group-wise reconstruction of an int8 weight matrix [N, K] into bf16:
// w_hat[n,k] = bf16(f32(q[n,k]) * s_grp[n, k/128]); 16 codes per thread-step.
__global__ void __launch_bounds__(256) i8_to_bf16_group_kernel(const int8_t* __restrict__ q,
                                                               const float* __restrict__ s_grp,
                                                               __nv_bfloat16* __restrict__ out,
                                                               int64_t n16, int K) {
  const int per_row = K / 16, ngrp = K / 128;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / per_row;
    const int c16 = static_cast<int>(i - n * per_row);
    const float sc = __ldg(s_grp + n * ngrp + c16 / 8);
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(q) + i);
    uint4 o0, o1;
    i8x4_scale_to_bf16x4(w.x, sc, o0.x, o0.y);
    i8x4_scale_to_bf16x4(w.y, sc, o0.z, o0.w);
    i8x4_scale_to_bf16x4(w.z, sc, o1.x, o1.y);
    i8x4_scale_to_bf16x4(w.w, sc, o1.z, o1.w);
    uint4* po = reinterpret_cast<uint4*>(out) + 2 * i;
    po[0] = o0;
    po[1] = o1;
  }
}

// FP8 (E4M3) weight quantisation with one scale per [128, 128] block of the
// folded weight f32(w[n,k]) * smooth[k]: one block of 256 threads per weight
// block, thread t owns 64 contiguous elements of row t/2.  scale = amax/448,
// codes e4m3(v * (448/amax)); s_w is [N/128, K/128].
__global__ void __launch_bounds__(256) fp8_block_quant_kernel(const __nv_bfloat16* __restrict__ w,
                                                              const float* __restrict__ smooth,
                                                              uint8_t* __restrict__ q,
                                                              float* __restrict__ s_w, int K) {
  __shared__ float red[8];
  const int bn = blockIdx.y, bk = blockIdx.x;
  const int t = threadIdx.x;
  const int64_t n = static_cast<int64_t>(bn) * 128 + (t >> 1);
  const int k0 = bk * 128 + (t & 1) * 64;
  const __nv_bfloat16* src = w + n * K + k0;
  float v[64];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(src) + i), *reinterpret_cast<float(*)[8]>(&v[8 * i]));
  }
  if (smooth) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float4 s4 = __ldg(reinterpret_cast<const float4*>(smooth + k0) + i);
      v[4 * i] = __fmul_rn(v[4 * i], s4.x);
      v[4 * i + 1] = __fmul_rn(v[4 * i + 1], s4.y);
      v[4 * i + 2] = __fmul_rn(v[4 * i + 2], s4.z);
      v[4 * i + 3] = __fmul_rn(v[4 * i + 3], s4.w);
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((t & 31) == 0) red[t >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  if (t == 0) s_w[static_cast<int64_t>(bn) * (K / 128) + bk] = __fdiv_rn(amax, 448.0f);
  const float mult = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 0.0f;
  uint8_t* dst = q + n * K + k0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t pk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float* f = v + 16 * i + 4 * j;
      const uint32_t lo = e4m3x2_bits(__fmul_rn(f[0], mult), __fmul_rn(f[1], mult));
      const uint32_t hi = e4m3x2_bits(__fmul_rn(f[2], mult), __fmul_rn(f[3], mult));
      pk[j] = amax > 0.0f ? (lo | (hi << 16)) : 0u;
    }
    reinterpret_cast<uint4*>(dst)[i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// gamma[k] = f32(g_k * inv_s[k]) with g_k = 1 + f32(w[k]) (zero-centred norm)
// or f32(w[k]): the norm weight with the SmoothQuant factor 1/s folded in.
__global__ void fold_norm_weight_kernel(const __nv_bfloat16* __restrict__ w, int zero_centered,
                                        const float* __restrict__ inv_s, float* __restrict__ gamma,
                                        int K) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  float g = __bfloat162float(w[k]);
  if (zero_centered) g = __fadd_rn(1.0f, g);
  gamma[k] = inv_s ? __fmul_rn(g, inv_s[k]) : g;
}

}  // namespace sq
