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
#include "ptx.cuh"

namespace sq {

// Exact conversion of four packed int8 codes to four bf16 values.  Each byte
// b is placed in the low mantissa bits of 2^23 after flipping its sign bit,
// which gives the float 2^23 + (q + 128) exactly; subtracting 2^23 + 128 gives
// q exactly, and since |q| <= 128 its fp32 pattern has 16 zero low bits, so
// the bf16 value is the high half.
__device__ __forceinline__ void i8x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const float bias = 8388736.0f;  // 2^23 + 128
  const float f0 = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)), bias);
  const float f1 = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541)), bias);
  const float f2 = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)), bias);
  const float f3 = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543)), bias);
  lo = __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632);
  hi = __byte_perm(__float_as_uint(f2), __float_as_uint(f3), 0x7632);
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

}  // namespace sq
