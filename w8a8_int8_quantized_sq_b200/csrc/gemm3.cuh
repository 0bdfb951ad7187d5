// gemm3.cuh -- block-scaled GEMMs on CTA pairs (tcgen05 cta_group::2): the
// gs128 variant (one weight scale per 128-wide K block) and the FP8 block
// variant (E4M3 operands, per-group activation scales, [128, 128] weight
// scales).
//
// Both promote every 128-wide K block separately: the K block's MMAs write a
// fresh accumulator in tensor memory and the epilogue warps fold it into fp32
// registers with that block's scale.  The pair tile is 256 MMA rows (128 in
// each CTA's tensor memory) x BN MMA columns, BN = 128 or 256; each CTA
// stages its own 128 A rows and BN / 2 of the B rows per K block.
//   BN = 128: four 128-column accumulators per CTA, 8 epilogue warps.
//   BN = 256: two 256-column accumulators, 16 epilogue warps (64 columns
//          each, loaded 16 at a time to fit 96 registers).  The host picks it
//          when the shape has at least three waves of 256-wide pair tiles.
//
// The operand roles are chosen so that each epilogue thread needs a single
// scale per K block:
//   gs128 (SWAP): A = weights, B = tokens.  A thread owns one output channel
//          n (its tensor-memory lane): acc = fmaf(f32(P), s_blk[n,kb], acc),
//          and y = bf16(acc * s_tok[m]) at the end of the tile.
//   FP8 (not swapped): A = tokens, B = weights.  A thread owns one token m
//          and its 64 channels lie in one 128-channel weight block:
//          acc = fmaf(P, f32(s_a[m,kb] * s_w[n/128,kb]), acc), y = bf16(acc).
// The int32 partials of gs128 become fp32 exactly (|P| <= 128 * 127^2 <
// 2^22): the bits of 1.5 * 2^23 are added, then 1.5 * 2^23 is subtracted, and
// one fmaf per element follows, the oracle's sequence.  With BN = 256 the
// accumulators start at those bits (0x4B400000) and all MMAs of a K block
// accumulate onto them, so the int32 result already is the fp32 pattern of
// 1.5 * 2^23 + P; the epilogue re-arms the bias with a tensor-memory store.
//
// Pace: each K block's accumulator makes a round trip MMA -> commit ->
// epilogue -> release -> MMA warp.  A probe issuing the same pair MMAs with a
// commit per K block and a wait four blocks back ran at two thirds of the
// back-to-back rate with 128-column MMAs and lost nothing with 256-column MMAs
// and two buffers.  Beyond that, a buffer goes back to the MMA only once every
// epilogue warp of both CTAs has released it, and promotion costs two or
// three instructions per element; tensor-memory loads (450 bytes per SM
// clock and more from 16 warps, measured) are not the limit.  Measured
// variants that were slower: packed
// f32x2 promotion; 16 epilogue warps on 128-wide tiles; a 256-thread barrier
// per K block; a cluster-scope releasing arrive (it waited for the
// outstanding scale loads); scale windows staged in shared memory.
//
// Roles per CTA: warp 0 TMA producer, warp 1 tensor-memory allocation (pair)
// and, in the leader CTA, the MMA issuer, the other warps epilogue (NE / 4 per
// tensor-memory lane quadrant, 64 columns each).  No load uses multicast.
#pragma once
#include "gemm2.cuh"

namespace sq {

__host__ __device__ constexpr uint32_t idesc_e4m3_f32_m256(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(256 >> 4) << 24);
}

__device__ __forceinline__ void mma_f8_pair(uint32_t d_tmem, uint64_t a, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Store 16 columns of one value to this warp's 32 tensor-memory lanes (no wait).
__device__ __forceinline__ void tmem_st16_const(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

// BN_: MMA N, the pair tile's B rows (128 or 256).  BIAS_: the int32
// accumulators start at 0x4B400000 (gs128 only), see above.
template <int EPI_, int BN_, bool BIAS_>
struct Gemm3Cfg {
  static constexpr int EPI = EPI_;
  static constexpr bool F8 = EPI == EPI_FP8BLK;
  static constexpr bool SWAP = EPI == EPI_GS128;  // A = weights for gs128
  static constexpr bool BIAS = BIAS_;
  static constexpr int BM = 128;         // A rows per CTA (256 per pair)
  static constexpr int BN = BN_;         // MMA N: B rows per pair tile
  static constexpr int BN_CTA = BN / 2;  // B rows staged by each CTA
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN_CTA * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 6 : 8;
  static constexpr int NE = BN == 256 ? 16 : 8;   // epilogue warps
  static constexpr int CPT = BN / (NE / 4);       // accumulator columns per epilogue thread
  static constexpr int CHUNK = 16;                // columns per tensor-memory load
  static constexpr int THREADS = 64 + NE * 32;
  static constexpr int NACC = 512 / BN;           // accumulator buffers
  static constexpr int TMEM_COLS = 512;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = STAGES * A_BYTES;
  static constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * NACC + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int smem_bytes() { return 1024 + OFF_MISC + 16; }
  static_assert(EPI == EPI_GS128 || EPI == EPI_FP8BLK, "pair block-scaled epilogues");
  static_assert(!BIAS || !F8, "the bias is an int32 bit pattern");
  static_assert(CPT == 64 && CPT % CHUNK == 0, "epilogue layout");
};

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    gemm3_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmArgs g) {
  constexpr int STAGES = Cfg::STAGES, NACC = Cfg::NACC, NE = Cfg::NE, BN = Cfg::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* smA = smem + Cfg::OFF_A;
  uint8_t* smB = smem + Cfg::OFF_B;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* full = bars;                 // leader: the pair's tiles of a stage have landed
  uint64_t* empty = bars + STAGES;       // both: the pair's MMAs are done with a stage
  uint64_t* tfull = bars + 2 * STAGES;   // both: a K block's accumulator is complete
  uint64_t* tempty = tfull + NACC;       // leader: both epilogues have read an accumulator
  uint64_t* drain = tempty + NACC;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int a = 0; a < NACC; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, 2 * NE);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated in both
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      griddep_wait();  // activations and scales may come from the preceding kernel
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      const uint64_t pol = policy_evict_last();  // both operands are re-read by other tiles
      uint32_t stage = 0, phase = 0;
      long long fills = 0;
      bool ok = true;
      for (int t = cluster; ok && t < g.num_tiles; t += nclusters) {
        const int rt = t % g.tiles_r, ct = t / g.tiles_r;
        const int a_row = rt * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM;
        const int b_row = ct * BN + static_cast<int>(rank) * Cfg::BN_CTA;
        for (int kb = 0; kb < g.kb_total; ++kb) {
          if (!wait_bounded(empty + stage, phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(full + stage, 2 * Cfg::STAGE_BYTES);
          tma_load_2d_pair(smA + stage * Cfg::A_BYTES, &tmA, kb * 128, a_row,
                           full_leader + stage * 8, pol);
          tma_load_2d_pair(smB + stage * Cfg::B_BYTES, &tmB, kb * 128, b_row,
                           full_leader + stage * 8, pol);
          ++fills;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (leader) {
        // the pair's copies (both CTAs' bytes count here) have all landed
        for (int st = 0; st < STAGES; ++st) {
          const long long n = fills / STAGES + (st < fills % STAGES ? 1 : 0);
          if (n > 0) wait_drain(full + st, static_cast<uint32_t>((n - 1) & 1));
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------- MMA issuer (leader)
    if (leader) {
      const uint32_t idesc = Cfg::F8 ? idesc_e4m3_f32_m256(BN) : idesc_i8_s32_m256(BN);
      uint32_t stage = 0, phase = 0, local = 0;
      bool ok = true;
      for (int t = cluster; ok && t < g.num_tiles; t += nclusters) {
        for (int kb = 0; kb < g.kb_total; ++kb, ++local) {
          const uint32_t p = local % NACC, u = local / NACC;
          // with the bias a buffer is free once the epilogue has re-armed it
          // (the first time before any MMA); without it a buffer starts free
          const uint32_t par = Cfg::BIAS ? (u & 1u) : ((u & 1u) ^ 1u);
          if (!warp_wait_bounded(tempty + p, par, abort_flag)) { ok = false; break; }
          if (!warp_wait_bounded(full + stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smA + stage * Cfg::A_BYTES);
          const uint32_t sb = smem_u32(smB + stage * Cfg::B_BYTES);
          const uint32_t d = tmem + p * BN;
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {  // a fresh accumulator (or the bias) per K block
              const uint32_t acc = (Cfg::BIAS || k > 0) ? 1u : 0u;
              if constexpr (Cfg::F8)
                mma_f8_pair(d, smem_desc_sw128(sa + k * 32), smem_desc_sw128(sb + k * 32), idesc,
                            acc);
              else
                mma_i8_pair(d, smem_desc_sw128(sa + k * 32), smem_desc_sw128(sb + k * 32), idesc,
                            acc);
            }
            mma_commit_pair_both(empty + stage);
            mma_commit_pair_both(tfull + p);
          }
          __syncwarp();
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (elect_one()) {
        mma_commit_pair(drain);
        wait_drain(drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    griddep_wait();
    const int ew = warp - 2;
    constexpr int CPT = Cfg::CPT, CHUNK = Cfg::CHUNK;
    const int q = warp & 3;                 // tensor-memory lane quadrant
    const int col0 = (ew >> 2) * CPT;       // this thread's accumulator columns
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);
    const int kbt = g.kb_total;
    constexpr uint32_t kBias = 0x4B400000u;  // bits of 1.5 * 2^23
    auto release = [&](uint32_t p) {
      if constexpr (Cfg::BIAS) tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(tempty + p);
        else mbar_arrive_remote(tempty_leader + p * 8);
      }
    };
    if constexpr (Cfg::BIAS) {
      // arm every buffer with the bias before the first MMA
      for (int p = 0; p < NACC; ++p) {
#pragma unroll
        for (int c = 0; c < CPT; c += CHUNK) tmem_st16_const(lane_base + p * BN + col0 + c, kBias);
        release(p);
      }
    }
    uint32_t local = 0;
    bool ok = true;
    for (int t = cluster; ok && t < g.num_tiles; t += nclusters) {
      const int rt = t % g.tiles_r, ct = t / g.tiles_r;
      // this thread's A row (tensor-memory lane): an output channel (gs128)
      // or a token (FP8)
      const int arow = rt * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM + q * 32 + lane;
      const bool row_ok = arow < (Cfg::SWAP ? g.N : g.M);
      const int cbase = ct * BN + col0;     // this thread's first B row (token or channel)
      auto scale_of = [&](int kb) -> float {
        if constexpr (Cfg::SWAP) {
          return row_ok ? __ldg(g.s_blk + static_cast<size_t>(arow) * kbt + kb) : 0.0f;
        } else {
          // the thread's 64 channels lie in one 128-channel weight block
          const float sa = row_ok ? __ldg(g.s_a + static_cast<size_t>(arow) * kbt + kb) : 0.0f;
          const float sw = cbase < g.N ? __ldg(g.s_blk + static_cast<size_t>(cbase >> 7) * kbt + kb)
                                       : 0.0f;
          return __fmul_rn(sa, sw);
        }
      };
      float acc[CPT];
#pragma unroll
      for (int j = 0; j < CPT; ++j) acc[j] = 0.0f;
      // One K block.  Its scale s was loaded two K blocks earlier; the load
      // for two K blocks later overwrites s after its last use.  (A rotating
      // three-register prefetch made each K block wait for the load it had
      // just issued: moving a register whose load is outstanding stalls.)
      auto kblock = [&](int kb, float& s) {
        const uint32_t p = local % NACC, u = local / NACC;
        ++local;
        if (!ok) return;
        if (!warp_wait_bounded(tfull + p, u & 1u, abort_flag)) { ok = false; return; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < CPT; c += CHUNK) {
          uint32_t v[CHUNK];
          tmem_ld16(lane_base + p * BN + col0 + c, v);
          if constexpr (Cfg::BIAS) tmem_st16_const(lane_base + p * BN + col0 + c, kBias);
          if (c + CHUNK == CPT) release(p);  // the whole K block is in registers or consumed
#pragma unroll
          for (int j = 0; j < CHUNK; ++j) {
            float f;
            if constexpr (Cfg::F8) f = __uint_as_float(v[j]);                 // fp32 partial
            else if constexpr (Cfg::BIAS) f = __fsub_rn(__uint_as_float(v[j]), 12582912.0f);
            else f = __fsub_rn(__uint_as_float(v[j] + kBias), 12582912.0f);  // exact f32(P)
            acc[c + j] = __fmaf_rn(f, s, acc[c + j]);
          }
        }
        if (kb + 2 < kbt) s = scale_of(kb + 2);
      };
      float sa = scale_of(0);
      float sb = kbt > 1 ? scale_of(1) : 0.0f;
      for (int kb = 0; kb < kbt; kb += 2) {
        kblock(kb, sa);
        if (kb + 1 < kbt) kblock(kb + 1, sb);
      }
      if (!ok) break;
      // the tile's outputs
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out);
      if constexpr (Cfg::SWAP) {
        // lane = channel n, columns = tokens m; lane j fetches the token
        // scales of columns j and 32 + j (coalesced) and the stores take them
        // from that lane
        const float st_lo = cbase + lane < g.M ? __ldg(g.s_tok + cbase + lane) : 0.0f;
        const float st_hi = cbase + 32 + lane < g.M ? __ldg(g.s_tok + cbase + 32 + lane) : 0.0f;
        __nv_bfloat16* o = out + static_cast<size_t>(cbase) * g.N + arow;  // column j: o + j * N
#pragma unroll
        for (int j = 0; j < CPT; ++j, o += g.N) {
          const float st = __shfl_sync(0xffffffffu, j < 32 ? st_lo : st_hi, j & 31);
          if (row_ok && cbase + j < g.M) *o = __float2bfloat16_rn(__fmul_rn(acc[j], st));
        }
      } else {
        // lane = token m, columns = channels n
        if (row_ok) {
          __nv_bfloat16* orow = out + static_cast<size_t>(arow) * g.N;
#pragma unroll
          for (int j = 0; j < CPT; j += 8) {
            const int n = cbase + j;
            if (n + 8 <= g.N)
              *reinterpret_cast<uint4*>(orow + n) =
                  make_uint4(pack_bf16x2(acc[j], acc[j + 1]), pack_bf16x2(acc[j + 2], acc[j + 3]),
                             pack_bf16x2(acc[j + 4], acc[j + 5]), pack_bf16x2(acc[j + 6], acc[j + 7]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs are done with the pair's tensor memory and barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace sq
