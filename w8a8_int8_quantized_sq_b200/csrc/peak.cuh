// peak.cuh -- tensor-pipe issue-rate probe: the dense MMA throughput of this
// device in the forms the GEMM kernels use, measured rather than taken from a
// data sheet.  Every CTA pair (one per two SMs) issues back-to-back
// tcgen05.mma cta_group::2 instructions (M = 256, N = 256, K = 32 bytes of
// operands) from shared memory into two alternating tensor-memory
// accumulators.  The operands are pseudo-random bytes (valid INT8 / E4M3 /
// BF16 values), so the tensor core switches as much as in a real GEMM and
// the clock settles where a real GEMM's would.  The caller times the launch
// with events on its stream; the leader's elected thread waits (bounded) for
// the commit of its last MMA, so the kernel ends only when every MMA is done.
#pragma once
#include "gemm3.cuh"

namespace sq {

enum : int { PEAK_I8 = 0, PEAK_F8 = 1, PEAK_BF16 = 2 };

template <int KIND>
__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int iters) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t done;
  __shared__ uint32_t holder;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_ctarank();
  // 16 KB of A (128 rows x 128 bytes) and 16 KB of B per CTA: a 32-bit
  // multiplicative hash of the word index, with each byte's top bits cleared
  // so that every byte is a finite E4M3 / BF16 half (|code| < 64)
  for (int i = threadIdx.x; i < 32768 / 4; i += blockDim.x) {
    const uint32_t h = (static_cast<uint32_t>(i) + 0x9E3779B9u * (blockIdx.x + 1)) * 0x85EBCA6Bu;
    reinterpret_cast<uint32_t*>(smem)[i] = (h ^ (h >> 13)) & 0x3F3F3F3Fu;
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&holder, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = holder;
  if (warp == 1 && rank == 0) {
    const uint32_t idesc = KIND == PEAK_I8 ? idesc_i8_s32_m256(256)
                           : KIND == PEAK_F8 ? idesc_e4m3_f32_m256(256)
                                             : idesc_bf16_f32_m256(256);
    const uint32_t sa = smem_u32(smem), sb = smem_u32(smem + 16384);
    if (elect_one()) {
      for (int i = 0; i < iters; ++i) {
        const uint32_t d = tmem + (i & 1) * 256;
        const uint64_t a = smem_desc_sw128(sa + (i & 3) * 32);
        const uint64_t b = smem_desc_sw128(sb + (i & 3) * 32);
        const uint32_t acc = i >= 2 ? 1u : 0u;
        if constexpr (KIND == PEAK_I8) mma_i8_pair(d, a, b, idesc, acc);
        else if constexpr (KIND == PEAK_F8) mma_f8_pair(d, a, b, idesc, acc);
        else mma_bf16_pair(d, a, b, idesc, acc);
      }
      mma_commit_pair(&done);
      wait_bounded(&done, 0, &abort_flag);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace sq
