// gemm2.cuh -- W8A8 GEMM on CTA pairs (tcgen05 cta_group::2), for the
// large-token (prefill) shapes.
//
// A cluster of two CTAs on paired SMs computes a 256 x 256 output tile with
// one MMA stream: each CTA stages its own 128 token rows of A and its own
// 128 weight rows (half of the tile's N) of B through a TMA ring, and the
// leader CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32) whose
// accumulator rows land in each CTA's tensor memory.  Against one CTA per
// 128 x 256 tile this halves the B bytes each SM stages per MMA, cutting
// L2->SM traffic by a third and shared-memory traffic per SM, and lets the
// ring hold six stages.  No load uses multicast: every CTA loads its own
// halves; the pair's TMA transaction bytes are counted on the leader's
// barrier and the leader's commits arrive on the barriers of both CTAs.
//
// Roles per CTA: warp 0 TMA producer, warp 1 TMEM allocation (pair) and, in
// the leader only, the MMA issuer, warps 2..5 epilogue (each CTA stores its
// own 128 rows of the tile).  Accumulators are double-buffered (2 x 256
// columns); both CTAs' epilogues release a buffer on the leader's barrier.
#pragma once
#include "gemm.cuh"

namespace sq {

// I8_ = true: W8A8 (kind::i8, int32 accumulators); false: BF16 operands
// (kind::f16, fp32 accumulators), the large-token W8A16 shape after the
// exact int8 -> bf16 weight conversion.
template <int EPI_, int STAGES_, bool I8_ = true>
struct Gemm2Cfg {
  static constexpr bool I8 = I8_;
  static constexpr bool SWAP = false;
  static constexpr int EPI = EPI_;
  static constexpr int STAGES = STAGES_;
  static constexpr int BM = 128;        // token rows per CTA (256 per pair)
  static constexpr int BN = 256;        // output columns per pair tile
  static constexpr int BN_CTA = 128;    // weight rows staged by each CTA
  static constexpr int KB_ELEMS = I8 ? 128 : 64;  // K elements per 128-byte stage row
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN_CTA * 128;
  static constexpr int NE = 4;
  static constexpr int THREADS = 64 + NE * 32;
  static constexpr int NACC = 2;
  static constexpr int TMEM_COLS = 512;
  static constexpr int CW = 32;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = STAGES * A_BYTES;
  static constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * NACC + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int smem_bytes() { return 1024 + OFF_MISC + 16; }
  static_assert(EPI == EPI_SCALE || EPI == EPI_I32, "pair kernel epilogues");
};

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmArgs g) {
  constexpr int STAGES = Cfg::STAGES, NACC = Cfg::NACC, NE = Cfg::NE, BN = Cfg::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* smA = smem + Cfg::OFF_A;
  uint8_t* smB = smem + Cfg::OFF_B;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* full = bars;                 // leader: pair's tiles of a stage have landed
  uint64_t* empty = bars + STAGES;       // both: the pair's MMAs are done with a stage
  uint64_t* tfull = bars + 2 * STAGES;   // both: an accumulator buffer is complete
  uint64_t* tempty = tfull + NACC;       // leader: both epilogues released a buffer
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
  griddep_launch_dependents();  // dependents wait for this grid's completion

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      // activations are re-read by every weight column tile: keep them in L2
      const uint64_t pol_act = policy_evict_last();
      // a weight tile is read by the concurrent clusters of its column, then not again
      const uint64_t pol_wt = policy_evict_normal();
      uint32_t stage = 0, phase = 0;
      long long fills = 0;
      bool ok = true;
      // weights (B) of the first STAGES fills are requested before
      // griddep_wait; their activation tiles follow it
      bool waited = false;
      int pend_kb[STAGES], pend_row[STAGES];
      auto act_load = [&](int st, int kb, int row) {
        tma_load_2d_pair(smA + st * Cfg::A_BYTES, &tmA, kb * Cfg::KB_ELEMS, row,
                         full_leader + st * 8, pol_act);
      };
      auto release_pending = [&]() {
        griddep_wait();
        const int n = fills < STAGES ? static_cast<int>(fills) : STAGES;
        for (int i = 0; i < n; ++i) act_load(i, pend_kb[i], pend_row[i]);
        waited = true;
      };
      for (int t = cluster; ok && t < g.num_tiles; t += nclusters) {
        const int rt = t % g.tiles_r, ct = t / g.tiles_r;
        const int a_row = rt * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM;
        const int b_row = ct * BN + static_cast<int>(rank) * Cfg::BN_CTA;
        for (int kb = 0; kb < g.kb_total; ++kb) {
          if (!waited && fills == STAGES) release_pending();
          if (!wait_bounded(empty + stage, phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(full + stage, 2 * (Cfg::A_BYTES + Cfg::B_BYTES));
          tma_load_2d_pair(smB + stage * Cfg::B_BYTES, &tmB, kb * Cfg::KB_ELEMS, b_row,
                           full_leader + stage * 8, pol_wt);
          if (waited) {
            act_load(stage, kb, a_row);
          } else {
            pend_kb[fills] = kb;
            pend_row[fills] = a_row;
          }
          ++fills;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!waited) release_pending();
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
    // The whole warp runs the loop; one elected lane issues and commits.
    if (leader) {
      const uint32_t idesc = Cfg::I8 ? idesc_i8_s32_m256(BN) : idesc_bf16_f32_m256(BN);
      uint32_t stage = 0, phase = 0, local = 0;
      bool ok = true;
      for (int t = cluster; ok && t < g.num_tiles; t += nclusters, ++local) {
        const uint32_t a = local % NACC, u = local / NACC;
        if (!warp_wait_bounded(tempty + a, (u & 1u) ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + a * BN;
        for (int kb = 0; kb < g.kb_total; ++kb) {
          if (!warp_wait_bounded(full + stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smA + stage * Cfg::A_BYTES);
          const uint32_t sb = smem_u32(smB + stage * Cfg::B_BYTES);
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if constexpr (Cfg::I8)
                mma_i8_pair(d, smem_desc_sw128(sa + k * 32), smem_desc_sw128(sb + k * 32), idesc,
                            (kb > 0 || k > 0) ? 1u : 0u);
              else
                mma_bf16_pair(d, smem_desc_sw128(sa + k * 32), smem_desc_sw128(sb + k * 32),
                              idesc, (kb > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit_pair_both(empty + stage);
          }
          __syncwarp();
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (elect_one()) mma_commit_pair_both(tfull + a);
        __syncwarp();
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
    const uint64_t pol_out = policy_evict_first();  // the output is not re-read here
    const int q = warp & 3;
    const int rr = q * 32 + lane;
    const int nthr = NE * 32;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t local = 0;
    for (int t = cluster; t < g.num_tiles; t += nclusters, ++local) {
      const uint32_t a = local % NACC, u = local / NACC;
      const bool w_ok = wait_bounded(tfull + a, u & 1u, abort_flag);
      if (named_bar_or(1, nthr, !w_ok)) break;
      tc_fence_after();
      const int rt = t % g.tiles_r, ct = t / g.tiles_r;
      const int rt128 = rt * 2 + static_cast<int>(rank);  // this CTA's 128 rows
#pragma unroll 1
      for (int c = 0; c < BN; c += Cfg::CW) {
        uint32_t v[Cfg::CW];
        tmem_ld32(lane_base + a * BN + c, v);
        store_chunk<Cfg>(g, rt128, ct, rr, c, v, pol_out);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(tempty + a);
        else mbar_arrive_cluster(mapa_shared(smem_u32(tempty + a), 0));
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
