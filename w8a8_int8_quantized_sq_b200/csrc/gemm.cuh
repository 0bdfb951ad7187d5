// gemm.cuh -- persistent, warp-specialised tcgen05 GEMM for sm_100a.
//
//   warp 0      : TMA producer (one elected thread) filling a ring of
//                 shared-memory stages, each one 128-byte-wide K block of
//                 A (128 rows) and B (BN rows), 128-byte swizzled.
//   warp 1      : allocates tensor memory; the whole warp runs the issue
//                 loop and one elected lane issues tcgen05.mma (kind::i8
//                 with int32 accumulators, or kind::f16 with BF16 operands
//                 and fp32 accumulators) into TMEM.
//   warps 2..   : epilogue; tcgen05.ld of the accumulators, scale, convert,
//                 store.  Double-buffered accumulators let the epilogue of
//                 one tile overlap the mainloop of the next.
//
// "Rows" are the MMA M dimension (operand A) and "columns" the MMA N
// dimension (operand B).  With SWAP = false A holds the tokens and B the
// output channels; with SWAP = true (small token counts) A holds the weight
// rows and B the tokens, so that the 128-row MMA tile is filled by weights.
//
// Schedules: tile-strided (CTA b takes tiles b, b+G, ...) or stream-K (CTA b
// takes the contiguous range [b*T/G, (b+1)*T/G) of the T = tiles x K-blocks
// iterations).  A tile split across CTAs is combined by the last CTA to
// finish its part: every part is written to a per-CTA slot of the
// workspace, an atomic counter per tile elects the last arrival, which sums
// the parts in CTA order and runs the epilogue, then resets the counter.
// When every CTA owns one K part of one tile (csplit > 1), a tile's CTAs are
// one thread-block cluster instead and the parts meet in rank 0's shared
// memory.
//
// EPI_GS128 (group-size-128 weight scales): every 128-wide K block is MMA'd
// into a fresh int32 TMEM buffer (4 in rotation).  The epilogue warps load a
// buffer's 64 columns per thread at once and release it, then convert each
// block partial P exactly (|P| <= 128 * 127^2 < 2^21: the integer add of the
// bits of 1.5 * 2^23 puts P in the mantissa, one subtraction leaves f32(P))
// and accumulate fmaf(f32(P), s_blk[n, kb], acc) in registers in K-block
// order.
#pragma once
#include "ptx.cuh"
#include "quant.cuh"  // exact int8 -> bf16 conversion

namespace sq {

// Epilogues.  The three block-scaled ones MMA every 128-wide K block into a
// fresh accumulator and promote it in registers:
//   EPI_GS128  : acc = fmaf(f32(P), s_blk[n,kb], acc), y = bf16(acc * s_tok[m])
//   EPI_PG128  : acc = fmaf(f32(P), f32(s_a[m,kb] * s_blk[n,kb]), acc), y = bf16(acc)
//   EPI_FP8BLK : E4M3 operands, fp32 block partials P,
//                acc = fmaf(P, f32(s_a[m,kb] * s_w[n/128,kb]), acc), y = bf16(acc)
// EPI_W16G (group-wise W8A16 on the dequant-on-load path): the converter
// warps reconstruct bf16(f32(q) * s_grp[n, k/128]) and the epilogue stores
// the fp32 sums as they are.
enum : int { EPI_SCALE = 0, EPI_I32 = 1, EPI_GS128 = 2, EPI_PG128 = 3, EPI_FP8BLK = 4,
             EPI_W16G = 5 };

__host__ __device__ constexpr bool is_block_scaled(int epi) {
  return epi == EPI_GS128 || epi == EPI_PG128 || epi == EPI_FP8BLK;
}

struct GemmArgs {
  int R, C;               // MMA rows (A rows) and columns (B rows)
  int kb_total;           // K blocks of 128 bytes
  int tiles_r, tiles_c, num_tiles;
  int stream_k;           // 0: tile-strided, 1: stream-K ranges
  long long total_iters;  // num_tiles * kb_total
  int M, N;               // output y is [M, N] row-major
  const float* s_tok;     // [M] per-token scales (may be null: W8A16)
  const float* s_ch;      // [N] per-channel scales
  const float* s_blk;     // [N, kb_total] block scales (EPI_GS128, EPI_PG128);
                          // [N/128, kb_total] (EPI_FP8BLK)
  const float* s_a;       // [M, kb_total] per-group activation scales
  void* out;              // bf16 [M, N] or int32 [M, N]
  uint32_t* ws;           // stream-K slots [grid][2][128][BN] 32-bit words
  unsigned int* ws_cnt;   // stream-K arrival counters [num_tiles]
  int csplit;             // > 1: the csplit CTAs of a tile form a cluster and
                          // combine their K parts in distributed shared memory
  int pdl;                // launched as a programmatic dependent
};

__host__ __device__ constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

// CONV_ = true (the W8A16 dequant-on-load path): operand A arrives as int8
// weight rows, RK K blocks per raw shared-memory stage (TMA, 128-byte
// swizzle).  Eight converter warps copy a whole raw stage into registers and
// release it, then expand it exactly to bf16 and write it straight into a
// ring of STAGES A tiles in tensor memory (tcgen05.st; 32 columns of two bf16
// per 128-lane row per K block) and wait for their stores once; the MMA reads
// A from tensor memory.  A producer warp of its own loads the K blocks' B tiles into their
// own shared-memory ring.  Everything moves in groups of RK K blocks (one raw
// stage, one A stage, one B stage): one hand-off and one tcgen05.commit per
// 4 x RK MMAs, because short N = 16 MMAs committed one K block at a time keep
// the tensor pipe waiting on each commit.  Keeping A out of shared
// memory leaves 2 bytes of shared-memory traffic per weight byte instead of 6.
template <bool I8_, int BN_, int STAGES_, bool SWAP_, int EPI_, bool CONV_ = false,
          int RSTAGES_ = 0>
struct GemmCfg {
  static constexpr bool I8 = I8_;
  static constexpr int BN = BN_;
  static constexpr int STAGES = STAGES_;
  static constexpr bool SWAP = SWAP_;
  static constexpr int EPI = EPI_;
  static constexpr bool CONV = CONV_;
  static constexpr int RSTAGES = CONV_ ? RSTAGES_ : 0;
  static constexpr int BM = 128;
  static constexpr int KB_BYTES = 128;
  static constexpr int KB_ELEMS = I8 ? 128 : 64;
  static constexpr int A_BYTES = BM * KB_BYTES;
  static constexpr int B_BYTES = BN * KB_BYTES;
  // raw stage: RK K blocks of int8 weight rows, as RK/2 boxes of 128 rows x
  // 128 bytes (two K blocks per row, 128-byte swizzle)
  static constexpr int RK = 4;
  static constexpr int RAW_BOX_BYTES = BM * 128;
  static constexpr int RAW_A_BYTES = (RK / 2) * RAW_BOX_BYTES;
  static constexpr int RAW_BYTES = RAW_A_BYTES;
  static constexpr bool BLK = is_block_scaled(EPI);
  static constexpr bool F8 = EPI == EPI_FP8BLK;          // kind::f8f6f4 (E4M3)
  static constexpr int NE = BLK ? 8 : 4;                 // epilogue warps
  static constexpr int NCV = CONV ? 8 : 0;               // converter warps (2 per row)
  // CONV: one more warp, the producer of the B tiles (warp 2 + NE + NCV)
  static constexpr int THREADS = 64 + NE * 32 + NCV * 32 + (CONV ? 32 : 0);
  static constexpr int NACC = BLK ? 4 : 2;
  // Narrow (swapped, small-token) tiles rotate the K blocks over NSUB
  // independent accumulators, so consecutive tiny MMAs do not wait on each
  // other's result; the epilogue adds them in a fixed order.
  static constexpr int NSUB = (SWAP && !BLK) ? 4 : 1;
  static constexpr int ACC_COLS = NACC * NSUB * BN;
  static constexpr int A_TMEM_COLS = 32;  // one 128 x 64 bf16 A tile in tensor memory
  // CONV: an A stage holds the RK converted K blocks of one raw stage
  static constexpr int TMEM_COLS = CONV ? 512 : pow2_at_least(ACC_COLS);
  static constexpr int CW = BN < 32 ? BN : 32;  // columns per tcgen05.ld
  static constexpr int CPT = BN / (NE / 4);     // columns owned by one epilogue thread
  static constexpr int SBLK_STRIDE = BN + 4;    // floats per K block in the staged s_blk
  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int A_SMEM_BYTES = CONV ? 0 : A_BYTES;  // CONV: A lives in TMEM
  // CONV: the B tiles have their own ring of stages of RK tiles (64 KB), so
  // their loads run ahead of the MMAs instead of following the A stages (a
  // 32 KB ring measured 2 us slower at 16 tokens)
  static constexpr int BSTAGES = CONV ? (65536 / (RK * B_BYTES)) : STAGES;
  static constexpr int B_RING_BYTES = CONV ? BSTAGES * RK * B_BYTES : STAGES * B_BYTES;
  static constexpr int OFF_RAW = 0;
  static constexpr int OFF_A = OFF_RAW + RSTAGES * RAW_BYTES;
  static constexpr int OFF_B = OFF_A + STAGES * A_SMEM_BYTES;
  static constexpr int OFF_BAR = OFF_B + B_RING_BYTES;
  static constexpr int NUM_BARS =
      2 * STAGES + 2 * NACC + 1 + 2 * RSTAGES + (CONV ? 2 * BSTAGES : 0) + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  // EPI_GS128: the tile's block scales; cluster split-K (rank 0 of a tile's
  // cluster): the other ranks' partial sums, [csplit - 1][BM][BN] words
  static constexpr int OFF_SBLK = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr int PART_BYTES = BM * BN * 4;
  static constexpr int smem_bytes(int kb_total, int csplit = 0) {
    return 1024 + OFF_SBLK + ((EPI == EPI_GS128 || EPI == EPI_PG128) ? kb_total * SBLK_STRIDE * 4 : 0) +
           (csplit > 1 ? (csplit - 1) * PART_BYTES : 0);
  }
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M = 128");
  static_assert(!BLK || (I8 && !SWAP && BN == 128), "block-scaled layout");
  static_assert(!CONV || (!I8 && SWAP && (EPI == EPI_SCALE || EPI == EPI_W16G)),
                "dequant-on-load is W8A16, swapped");
  static_assert(EPI != EPI_W16G || CONV, "group-scaled reconstruction happens on load");
  static_assert(!CONV || (RAW_BYTES % 1024 == 0 && B_BYTES % 16 == 0), "raw stage alignment");
  static_assert(!CONV || ACC_COLS + STAGES * RK * A_TMEM_COLS <= 512, "tensor memory A ring");

  static_assert(TMEM_COLS <= 512, "tensor memory");
};

struct Seg {
  int tile, kb0, kb1;
};

__device__ __forceinline__ long long sk_start(long long b, long long G, long long T) {
  return b * T / G;
}
// CTA whose stream-K range contains iteration i.
__device__ __forceinline__ long long sk_owner(long long i, long long G, long long T) {
  return ((i + 1) * G + T - 1) / T - 1;
}

struct SegIter {
  long long pos, end;
  __device__ __forceinline__ void init(const GemmArgs& g) {
    if (g.stream_k) {
      pos = sk_start(blockIdx.x, gridDim.x, g.total_iters);
      end = sk_start(blockIdx.x + 1, gridDim.x, g.total_iters);
    } else {
      pos = blockIdx.x;
      end = g.num_tiles;
    }
  }
  __device__ __forceinline__ bool next(const GemmArgs& g, Seg& s) {
    if (pos >= end) return false;
    if (g.stream_k) {
      s.tile = static_cast<int>(pos / g.kb_total);
      s.kb0 = static_cast<int>(pos % g.kb_total);
      const long long rem = end - pos;
      s.kb1 = static_cast<int>(rem < g.kb_total - s.kb0 ? s.kb0 + rem : g.kb_total);
      pos += s.kb1 - s.kb0;
    } else {
      s.tile = static_cast<int>(pos);
      s.kb0 = 0;
      s.kb1 = g.kb_total;
      pos += gridDim.x;
    }
    return true;
  }
};

// --------------------------------------------------------------- epilogue
// Scale/convert/store CW accumulator columns [c0, c0 + CW) of MMA row rr of
// tile (rt, ct).  v holds int32 (I8) or fp32 bits (BF16) accumulators.
// policy != 0: the 16-byte BF16 output stores carry that L2 eviction hint.
template <class Cfg>
__device__ __forceinline__ void store_chunk(const GemmArgs& g, int rt, int ct, int rr, int c0,
                                            const uint32_t (&v)[Cfg::CW], uint64_t policy = 0,
                                            const float* sc_pre = nullptr,
                                            const float* st_pre = nullptr) {
  constexpr int CW = Cfg::CW;
  const int r = rt * Cfg::BM + rr;
  const int cb = ct * Cfg::BN + c0;
  if constexpr (!Cfg::SWAP) {
    const int m = r;
    if (m >= g.M) return;
    if constexpr (Cfg::EPI == EPI_I32) {
      int32_t* out = static_cast<int32_t*>(g.out) + static_cast<size_t>(m) * g.N;
#pragma unroll
      for (int j = 0; j < CW; j += 4) {
        const int n = cb + j;
        if (n + 4 <= g.N)
          *reinterpret_cast<int4*>(out + n) = make_int4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      }
    } else {
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out) + static_cast<size_t>(m) * g.N;
      const float st = (Cfg::I8 && g.s_tok) ? __ldg(g.s_tok + m) : 1.0f;
#pragma unroll
      for (int j = 0; j < CW; j += 8) {
        const int n = cb + j;
        if (n + 8 > g.N) break;
        float sc[8] = {1.0f, 1.0f, 1.0f, 1.0f, 1.0f, 1.0f, 1.0f, 1.0f};  // no s_ch: unscaled
        if (g.s_ch) {
          const float4 c0v = __ldg(reinterpret_cast<const float4*>(g.s_ch + n));
          const float4 c1v = __ldg(reinterpret_cast<const float4*>(g.s_ch + n) + 1);
          sc[0] = c0v.x; sc[1] = c0v.y; sc[2] = c0v.z; sc[3] = c0v.w;
          sc[4] = c1v.x; sc[5] = c1v.y; sc[6] = c1v.z; sc[7] = c1v.w;
        }
        float f[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if constexpr (Cfg::I8) {
            f[i] = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(v[j + i])), st), sc[i]);
          } else {
            f[i] = __fmul_rn(__uint_as_float(v[j + i]), sc[i]);
          }
        }
        const uint4 o = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                   pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
        if (policy) st_global_v4_hint(out + n, o, policy);
        else *reinterpret_cast<uint4*>(out + n) = o;
      }
    }
  } else {
    const int n = r;
    if (n >= g.N) return;
    if constexpr (Cfg::EPI == EPI_I32) {
      int32_t* out = static_cast<int32_t*>(g.out);
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int m = cb + j;
        if (m < g.M) out[static_cast<size_t>(m) * g.N + n] = static_cast<int32_t>(v[j]);
      }
    } else {
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out);
      const float sc = sc_pre ? *sc_pre : (g.s_ch ? __ldg(g.s_ch + n) : 1.0f);
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int m = cb + j;
        if (m < g.M) {
          float f;
          if constexpr (Cfg::I8) {
            const float st = st_pre ? st_pre[j] : (g.s_tok ? __ldg(g.s_tok + m) : 1.0f);
            f = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(v[j])), st), sc);
          } else {
            f = __fmul_rn(__uint_as_float(v[j]), sc);
          }
          out[static_cast<size_t>(m) * g.N + n] = __float2bfloat16_rn(f);
        }
      }
    }
  }
}

template <class Cfg>
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, uint32_t (&v)[Cfg::CW]) {
  if constexpr (Cfg::CW == 32) tmem_ld32(taddr, v);
  else tmem_ld16(taddr, v);
}

// Columns [c, c + CW) of an accumulator made of `nsub` sub-accumulators
// (BN columns apart), summed in sub-accumulator order.
template <class Cfg>
__device__ __forceinline__ void tmem_ld_acc(uint32_t tb, int c, int nsub,
                                            uint32_t (&v)[Cfg::CW]) {
  tmem_ld_chunk<Cfg>(tb + c, v);
  for (int sub = 1; sub < nsub; ++sub) {
    uint32_t t[Cfg::CW];
    tmem_ld_chunk<Cfg>(tb + sub * Cfg::BN + c, t);
#pragma unroll
    for (int j = 0; j < Cfg::CW; ++j) {
      if constexpr (Cfg::I8)
        v[j] = static_cast<uint32_t>(static_cast<int32_t>(v[j]) + static_cast<int32_t>(t[j]));
      else
        v[j] = __float_as_uint(__fadd_rn(__uint_as_float(v[j]), __uint_as_float(t[j])));
    }
  }
}

// ------------------------------------------------------------------ kernel
template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs g) {
  constexpr int BN = Cfg::BN, STAGES = Cfg::STAGES, NACC = Cfg::NACC, NE = Cfg::NE;
  constexpr int CW = Cfg::CW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* smA = smem + Cfg::OFF_A;
  uint8_t* smB = smem + Cfg::OFF_B;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + NACC;
  uint64_t* drain = tempty + NACC;
  uint64_t* raw_full = drain + 1;             // CONV: producer -> converters
  uint64_t* raw_empty = raw_full + Cfg::RSTAGES;  // CONV: converters -> producer
  uint64_t* b_full = raw_empty + Cfg::RSTAGES;    // CONV: B producer -> MMA
  uint64_t* b_empty = b_full + Cfg::BSTAGES;      // CONV: MMA -> B producer
  uint64_t* red_bar = b_empty + (Cfg::CONV ? Cfg::BSTAGES : 0);  // cluster split-K parts
  uint8_t* smRaw = smem + Cfg::OFF_RAW;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);
  volatile int* sk_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 8);
  float* sblk = reinterpret_cast<float*>(smem + Cfg::OFF_SBLK);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CONV: raw stages thread 0 (the raw-weight producer) issues during set-up.
  // (Doing the same with the weight tiles of the generic producer measured
  // about 1 us slower on the decode shape, so it starts them in its role.)
  long long pre_fills = 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int a = 0; a < NACC; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, NE);
    }
    mbar_init(drain, 1);
    if constexpr (Cfg::CONV) {
      // a converted A stage completes on the converter warps' arrivals
      for (int s = 0; s < STAGES; ++s) mbar_init(full + s, Cfg::NCV);
      for (int s = 0; s < Cfg::RSTAGES; ++s) {
        mbar_init(raw_full + s, 1);
        mbar_init(raw_empty + s, Cfg::NCV);
      }
      for (int s = 0; s < Cfg::BSTAGES; ++s) {
        mbar_init(b_full + s, 1);
        mbar_init(b_empty + s, 1);
      }
    }
    // rank 0 of a split-K cluster: every epilogue thread of the other ranks
    mbar_init(red_bar, (g.csplit > 1 ? g.csplit - 1 : 1) * NE * 32);
    *abort_flag = 0;
    *sk_flag = 0;
    fence_mbar_init();
    if constexpr (Cfg::CONV) {
      // start the weight stream now, while the other warps allocate tensor
      // memory and reach the CTA barrier
      tma_prefetch_desc(&tmA);
      SegIter it;
      it.init(g);
      Seg s;
      while (pre_fills < Cfg::RSTAGES && it.next(g, s)) {
        const int rt = s.tile % g.tiles_r;
        for (int kb = s.kb0; kb < s.kb1 && pre_fills < Cfg::RSTAGES; kb += Cfg::RK) {
          const int n = s.kb1 - kb < Cfg::RK ? s.kb1 - kb : Cfg::RK;
          const int rs = static_cast<int>(pre_fills);
          const int boxes = (n + 1) / 2;
          mbar_arrive_expect_tx(raw_full + rs, boxes * Cfg::RAW_BOX_BYTES);
          for (int b2 = 0; b2 < boxes; ++b2)
            tma_load_2d(smRaw + rs * Cfg::RAW_BYTES + b2 * Cfg::RAW_BOX_BYTES, &tmA,
                        (kb + 2 * b2) * Cfg::KB_ELEMS, rt * Cfg::BM, raw_full + rs);
          ++pre_fills;
        }
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  // split-K clusters: the barriers of every rank are initialised before any
  // rank arrives remotely
  if (g.csplit > 1) cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // a programmatic dependent of this grid may be scheduled now; it waits for
  // this grid's completion before it reads anything this grid writes
  griddep_launch_dependents();

  if ((warp == 0 || warp == 2 + NE + Cfg::NCV) && Cfg::CONV) {
    // ------------------------------- TMA producers: raw int8 weights (warp 0)
    //                          and the K blocks' B tiles (the last warp); one
    //                          warp each, since two spinning lanes of one warp
    //                          take turns and starve each other
    if constexpr (Cfg::CONV) {
      if (warp == 0 && lane == 0) {
        uint32_t rs = 0, rph = 0;
        long long fills = 0;
        SegIter it;
        it.init(g);
        Seg s;
        bool ok = true;
        while (ok && it.next(g, s)) {
          const int rt = s.tile % g.tiles_r;
          for (int kb = s.kb0; kb < s.kb1; kb += Cfg::RK) {
            const int n = s.kb1 - kb < Cfg::RK ? s.kb1 - kb : Cfg::RK;  // K blocks used
            if (fills < pre_fills) {  // issued during set-up
              ++fills;
              if (++rs == Cfg::RSTAGES) { rs = 0; rph ^= 1u; }
              continue;
            }
            if (!wait_bounded(raw_empty + rs, rph ^ 1u, abort_flag)) { ok = false; break; }
            uint8_t* st = smRaw + rs * Cfg::RAW_BYTES;
            const int boxes = (n + 1) / 2;
            mbar_arrive_expect_tx(raw_full + rs, boxes * Cfg::RAW_BOX_BYTES);
            // 128 contiguous weight bytes per row per box, both boxes back to back
            for (int b2 = 0; b2 < boxes; ++b2)
              tma_load_2d(st + b2 * Cfg::RAW_BOX_BYTES, &tmA, (kb + 2 * b2) * Cfg::KB_ELEMS,
                          rt * Cfg::BM, raw_full + rs);
            ++fills;
            if (++rs == Cfg::RSTAGES) { rs = 0; rph ^= 1u; }
          }
        }
        for (int st = 0; st < Cfg::RSTAGES; ++st) {
          const long long n = fills / Cfg::RSTAGES + (st < fills % Cfg::RSTAGES ? 1 : 0);
          if (n > 0) wait_drain(raw_full + st, static_cast<uint32_t>((n - 1) & 1));
        }
      } else if (warp != 0 && lane == 0) {
        tma_prefetch_desc(&tmB);
        griddep_wait();  // the activations may come from the preceding kernel
        uint32_t cs = 0, cph = 0;
        long long bfills = 0;
        SegIter it;
        it.init(g);
        Seg s;
        bool ok = true;
        while (ok && it.next(g, s)) {
          const int ct = s.tile / g.tiles_r;
          for (int kb = s.kb0; kb < s.kb1; kb += Cfg::RK) {
            const int n = s.kb1 - kb < Cfg::RK ? s.kb1 - kb : Cfg::RK;
            if (!wait_bounded(b_empty + cs, cph ^ 1u, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(b_full + cs, n * Cfg::B_BYTES);
            for (int c = 0; c < n; ++c)
              tma_load_2d(smB + (cs * Cfg::RK + c) * Cfg::B_BYTES, &tmB, (kb + c) * Cfg::KB_ELEMS,
                          ct * BN, b_full + cs);
            ++bfills;
            if (++cs == Cfg::BSTAGES) { cs = 0; cph ^= 1u; }
          }
        }
        for (int st = 0; st < Cfg::BSTAGES; ++st) {
          const long long n = bfills / Cfg::BSTAGES + (st < bfills % Cfg::BSTAGES ? 1 : 0);
          if (n > 0) wait_drain(b_full + st, static_cast<uint32_t>((n - 1) & 1));
        }
      }
    }
  } else if (warp >= 2 + NE) {
    // ------------------------------------------- converter warps (CONV only)
    if constexpr (Cfg::CONV) {
      const int q = warp & 3;                  // TMEM lane quadrant of this warp
      const int row = q * 32 + lane;           // weight row of the K block (= TMEM lane)
      const int half = (warp - (2 + NE)) >> 2; // which 32 of its 64 codes
      const uint32_t a_lane = tmem + (static_cast<uint32_t>(q * 32) << 16) + Cfg::ACC_COLS;
      uint32_t rs = 0, rph = 0, cs = 0, cph = 0;
      SegIter it;
      it.init(g);
      Seg s;
      bool ok = true;
      const int ngrp = g.kb_total / 2;  // EPI_W16G: 128-wide groups = two 64-wide K blocks
      while (ok && it.next(g, s)) {
        const int wrow = (s.tile % g.tiles_r) * Cfg::BM + row;  // this thread's weight row
        for (int kb = s.kb0; kb < s.kb1 && ok; kb += Cfg::RK) {
          const int n = s.kb1 - kb < Cfg::RK ? s.kb1 - kb : Cfg::RK;
          float gsc[Cfg::RK];  // EPI_W16G: the group scale of each K block of the stage
          if constexpr (Cfg::EPI == EPI_W16G) {
#pragma unroll
            for (int c = 0; c < Cfg::RK; ++c)
              gsc[c] = (wrow < g.N && c < n)
                           ? __ldg(g.s_blk + static_cast<size_t>(wrow) * ngrp + ((kb + c) >> 1))
                           : 0.0f;
          }
          if (!wait_bounded(raw_full + rs, rph, abort_flag)) { ok = false; break; }
          const uint8_t* raw = smRaw + rs * Cfg::RAW_BYTES;
          // raw row (128-byte swizzle): K block c is chunks 4(c&1)..4(c&1)+3 of
          // its box row, 16-byte chunk j at position j ^ (row & 7).  This
          // thread converts chunks 2*half, 2*half+1 (32 codes -> 32 bf16, two
          // per column, lower K in the low half) into TMEM columns 16*half ..
          // 16*half+15 of the K block's part of the A stage.
          constexpr int CH = 2;
          auto chunk = [&](int c, int jj) {
            return *reinterpret_cast<const uint4*>(
                raw + (c >> 1) * Cfg::RAW_BOX_BYTES + row * 128 +
                (((4 * (c & 1) + 2 * half + jj) ^ (row & 7)) << 4));
          };
          auto convert = [&](const uint4 (&wc)[CH], uint32_t slot) {
            uint32_t o[8 * CH];
#pragma unroll
            for (int j = 0; j < CH; ++j) {
              if constexpr (Cfg::EPI == EPI_W16G) {
                const float sc = gsc[slot];
                i8x4_scale_to_bf16x4(wc[j].x, sc, o[8 * j + 0], o[8 * j + 1]);
                i8x4_scale_to_bf16x4(wc[j].y, sc, o[8 * j + 2], o[8 * j + 3]);
                i8x4_scale_to_bf16x4(wc[j].z, sc, o[8 * j + 4], o[8 * j + 5]);
                i8x4_scale_to_bf16x4(wc[j].w, sc, o[8 * j + 6], o[8 * j + 7]);
              } else {
                i8x4_to_bf16x4(wc[j].x, o[8 * j + 0], o[8 * j + 1]);
                i8x4_to_bf16x4(wc[j].y, o[8 * j + 2], o[8 * j + 3]);
                i8x4_to_bf16x4(wc[j].z, o[8 * j + 4], o[8 * j + 5]);
                i8x4_to_bf16x4(wc[j].w, o[8 * j + 6], o[8 * j + 7]);
              }
            }
            tmem_st16(a_lane + (cs * Cfg::RK + slot) * Cfg::A_TMEM_COLS + half * 16, o);
          };
          // The whole stage's codes go to registers first and the raw stage
          // is released at once (the arrive orders this warp's loads before
          // it), so the next weight load is in flight while this warp waits
          // for its A stage and converts: a raw stage is held for the length
          // of a shared-memory load, not of a conversion.
          uint4 w[Cfg::RK][CH];
#pragma unroll
          for (int c = 0; c < Cfg::RK; ++c) {
            if (c < n) {
#pragma unroll
              for (int j = 0; j < CH; ++j) w[c][j] = chunk(c, j);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(raw_empty + rs);
          // the A stage is free once the MMAs that read it are done
          if (!wait_bounded(empty + cs, cph ^ 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < Cfg::RK; ++c)
            if (c < n) convert(w[c], c);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(full + cs);
          if (++cs == STAGES) { cs = 0; cph ^= 1u; }
          if (++rs == Cfg::RSTAGES) { rs = 0; rph ^= 1u; }
        }
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      uint32_t stage = 0, phase = 0;
      long long fills = 0;
      SegIter it;
      it.init(g);
      Seg s;
      bool ok = true;
      // Under a programmatic launch the weight operand (A when SWAP, else B)
      // of the first STAGES fills is requested before griddep_wait, so that
      // the weight stream starts while the preceding kernel still produces
      // the activations; their activation tiles follow right after the wait.
      // Otherwise every fill requests both at once (so the first stage is
      // not queued behind STAGES weight tiles).
      bool waited = g.pdl == 0;
      int pend_kb[STAGES], pend_row[STAGES];
      auto act_load = [&](int st, int kb, int row) {
        if constexpr (Cfg::SWAP)
          tma_load_2d(smB + st * Cfg::B_BYTES, &tmB, kb * Cfg::KB_ELEMS, row, full + st);
        else
          tma_load_2d(smA + st * Cfg::A_BYTES, &tmA, kb * Cfg::KB_ELEMS, row, full + st);
      };
      auto release_pending = [&]() {
        griddep_wait();
        const int n = fills < STAGES ? static_cast<int>(fills) : STAGES;
        for (int i = 0; i < n; ++i) act_load(i, pend_kb[i], pend_row[i]);
        waited = true;
      };
      while (ok && it.next(g, s)) {
        const int rt = s.tile % g.tiles_r, ct = s.tile / g.tiles_r;
        for (int kb = s.kb0; kb < s.kb1; ++kb) {
          if (!waited && fills == STAGES) release_pending();
          if (!wait_bounded(empty + stage, phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full + stage, Cfg::A_BYTES + Cfg::B_BYTES);
          const int act_row = Cfg::SWAP ? ct * BN : rt * Cfg::BM;
          if constexpr (Cfg::SWAP)
            tma_load_2d(smA + stage * Cfg::A_BYTES, &tmA, kb * Cfg::KB_ELEMS, rt * Cfg::BM,
                        full + stage);
          else
            tma_load_2d(smB + stage * Cfg::B_BYTES, &tmB, kb * Cfg::KB_ELEMS, ct * BN,
                        full + stage);
          if (waited) {
            act_load(stage, kb, act_row);
          } else {
            pend_kb[fills] = kb;
            pend_row[fills] = act_row;
          }
          ++fills;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!waited) release_pending();
      // no copy may still be writing shared memory when the CTA exits
      for (int st = 0; st < STAGES; ++st) {
        const long long n = fills / STAGES + (st < fills % STAGES ? 1 : 0);
        if (n > 0) wait_drain(full + st, static_cast<uint32_t>((n - 1) & 1));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    // The whole warp runs the loop and waits; one elected lane issues the
    // MMAs and commits.
    {
      const uint32_t idesc =
          Cfg::F8 ? idesc_e4m3_f32(BN) : (Cfg::I8 ? idesc_i8_s32(BN) : idesc_bf16_f32(BN));
      uint32_t stage = 0, phase = 0;
      uint32_t bstage = 0, bphase = 0;  // CONV: the separate B ring
      uint32_t local = 0;
      SegIter it;
      it.init(g);
      Seg s;
      bool ok = true;
      while (ok && it.next(g, s)) {
        if constexpr (Cfg::BLK) {
          for (int kb = s.kb0; kb < s.kb1 && ok; ++kb, ++local) {
            const uint32_t p = local % NACC, u = local / NACC;
            if (!warp_wait_bounded(tempty + p, u & 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (!warp_wait_bounded(full + stage, phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smA + stage * Cfg::A_BYTES);
            const uint32_t sb = smem_u32(smB + stage * Cfg::B_BYTES);
            if (elect_one()) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {  // a fresh accumulator per K block
                if constexpr (Cfg::F8)
                  mma_f8(tmem + p * BN, smem_desc_sw128(sa + k * 32), smem_desc_sw128(sb + k * 32),
                         idesc, k > 0 ? 1u : 0u);
                else
                  mma_i8(tmem + p * BN, smem_desc_sw128(sa + k * 32), smem_desc_sw128(sb + k * 32),
                         idesc, k > 0 ? 1u : 0u);
              }
              mma_commit(empty + stage);
              mma_commit(tfull + p);
            }
            __syncwarp();
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
        } else if constexpr (Cfg::CONV) {
          // groups of RK K blocks: A from tensor memory, B from its ring,
          // one commit per group
          const uint32_t a = local % NACC, u = local / NACC;
          if (!warp_wait_bounded(tempty + a, (u & 1u) ^ 1u, abort_flag)) break;
          tc_fence_after();
          int i = 0;  // K block index within the segment
          for (int kb = s.kb0; kb < s.kb1; kb += Cfg::RK) {
            const int n = s.kb1 - kb < Cfg::RK ? s.kb1 - kb : Cfg::RK;
            if (!warp_wait_bounded(full + stage, phase, abort_flag)) { ok = false; break; }
            if (!warp_wait_bounded(b_full + bstage, bphase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_col = tmem + Cfg::ACC_COLS + stage * Cfg::RK * Cfg::A_TMEM_COLS;
            const uint32_t sb0 = smem_u32(smB + bstage * Cfg::RK * Cfg::B_BYTES);
            if (elect_one()) {
              for (int c = 0; c < n; ++c) {
                const uint32_t d = tmem + (a * Cfg::NSUB + (i + c) % Cfg::NSUB) * BN;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  mma_bf16_tmem_a(d, a_col + c * Cfg::A_TMEM_COLS + k * 8,
                                  smem_desc_sw128(sb0 + c * Cfg::B_BYTES + k * 32), idesc,
                                  (i + c >= Cfg::NSUB || k > 0) ? 1u : 0u);
              }
              mma_commit(empty + stage);
              mma_commit(b_empty + bstage);
            }
            __syncwarp();
            i += n;
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            if (++bstage == Cfg::BSTAGES) { bstage = 0; bphase ^= 1u; }
          }
          if (!ok) break;
          if (elect_one()) mma_commit(tfull + a);
          __syncwarp();
          ++local;
        } else {
          const uint32_t a = local % NACC, u = local / NACC;
          if (!warp_wait_bounded(tempty + a, (u & 1u) ^ 1u, abort_flag)) break;
          tc_fence_after();
          for (int kb = s.kb0; kb < s.kb1; ++kb) {
            if (!warp_wait_bounded(full + stage, phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smA + stage * Cfg::A_BYTES);
            const uint32_t sb = smem_u32(smB + stage * Cfg::B_BYTES);
            const int i = kb - s.kb0;
            const uint32_t d = tmem + (a * Cfg::NSUB + i % Cfg::NSUB) * BN;
            if (elect_one()) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint32_t accum = (i >= Cfg::NSUB || k > 0) ? 1u : 0u;
                if constexpr (Cfg::I8)
                  mma_i8(d, smem_desc_sw128(sa + k * 32), smem_desc_sw128(sb + k * 32), idesc,
                         accum);
                else
                  mma_bf16(d, smem_desc_sw128(sa + k * 32), smem_desc_sw128(sb + k * 32), idesc,
                           accum);
              }
              mma_commit(empty + stage);
            }
            __syncwarp();
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          if (elect_one()) mma_commit(tfull + a);
          __syncwarp();
          ++local;
        }
      }
      // every MMA issued by the elected lane has finished before TMEM is freed
      if (elect_one()) {
        mma_commit(drain);
        wait_drain(drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    griddep_wait();  // the scales may come from the preceding kernel
    const int ew = warp - 2;
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int rr = q * 32 + lane;
    const int nthr = NE * 32;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    SegIter it;
    it.init(g);
    Seg s;
    if constexpr (Cfg::BLK) {
      constexpr int CPT = Cfg::CPT;
      constexpr bool COLSCALE = Cfg::EPI == EPI_GS128 || Cfg::EPI == EPI_PG128;
      const int h = ew / 4;
      const int col0 = h * CPT;
      const int et = ew * 32 + lane;
      // every buffer starts free: releasing it completes phase 0
      if (lane == 0)
        for (int p = 0; p < NACC; ++p) mbar_arrive(tempty + p);
      uint32_t local = 0;
      bool ok = true;
      while (ok && it.next(g, s)) {
        const int rt = s.tile % g.tiles_r, ct = s.tile / g.tiles_r;
        const int m = rt * Cfg::BM + rr;
        if constexpr (COLSCALE) {
          // stage this tile's block scales, transposed to [kb][n]; each thread
          // requests a batch of its elements before storing any
          named_bar_sync(1, nthr);
          const int total = g.kb_total * BN;
          for (int base = 0; base < total; base += 8 * nthr) {
            float vals[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int idx = base + i * nthr + et;
              const int j = idx / g.kb_total, kb = idx - j * g.kb_total;
              const int n = ct * BN + j;
              vals[i] = (idx < total && n < g.N)
                            ? __ldg(g.s_blk + static_cast<size_t>(n) * g.kb_total + kb)
                            : 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int idx = base + i * nthr + et;
              const int j = idx / g.kb_total, kb = idx - j * g.kb_total;
              if (idx < total) sblk[kb * Cfg::SBLK_STRIDE + j] = vals[i];
            }
          }
          named_bar_sync(1, nthr);
        }
        // per-group activation scales of this thread's row (0 past the last row)
        const float* sa_row =
            (Cfg::EPI != EPI_GS128 && m < g.M) ? g.s_a + static_cast<size_t>(m) * g.kb_total : nullptr;
        float acc[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) acc[j] = 0.0f;
        // this thread's scalar scale factors of a K block (per-group
        // activations; FP8: times the tile's weight-block scale)
        auto row_scale = [&](int kb) -> float {
          float sa = 0.0f;
          if constexpr (Cfg::EPI != EPI_GS128) sa = sa_row ? __ldg(sa_row + kb) : 0.0f;
          if constexpr (Cfg::F8)
            sa = __fmul_rn(sa, __ldg(g.s_blk + static_cast<size_t>(ct) * g.kb_total + kb));
          return sa;
        };
        float sa_next = row_scale(s.kb0);
        for (int kb = s.kb0; kb < s.kb1; ++kb, ++local) {
          const uint32_t p = local % NACC, u = local / NACC;
          const float sa = sa_next;
          const bool w_ok = wait_bounded(tfull + p, u & 1u, abort_flag);
          if (named_bar_or(1, nthr, !w_ok)) { ok = false; break; }
          tc_fence_after();
          // this K block's partial sums (int32: |sum| <= 128 * 127 * 127 <
          // 2^22; or fp32), then the buffer goes straight back to the MMA
          static_assert(CPT == 64, "one 64-column load per K block");
          uint32_t v[64];
          tmem_ld64(lane_base + p * BN + col0, v);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty + p);
          // the next K block's scales, requested after the release (a
          // releasing arrive would otherwise wait for the load)
          if (kb + 1 < s.kb1) sa_next = row_scale(kb + 1);
          if constexpr (Cfg::F8) {
            const float sc = sa;
#pragma unroll
            for (int j = 0; j < 64; ++j) acc[j] = __fmaf_rn(__uint_as_float(v[j]), sc, acc[j]);
          } else {
            // exact int32 -> fp32: add the bits of 1.5 * 2^23 (the sum lands in
            // the mantissa), subtract 1.5 * 2^23; then one rounding per step
            const float* sk = sblk + kb * Cfg::SBLK_STRIDE + col0;
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
              const float4 s4 = *reinterpret_cast<const float4*>(sk + j);
              float sc[4] = {s4.x, s4.y, s4.z, s4.w};
              if constexpr (Cfg::EPI == EPI_PG128) {
#pragma unroll
                for (int i = 0; i < 4; ++i) sc[i] = __fmul_rn(sa, sc[i]);
              }
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float f = __fsub_rn(__uint_as_float(v[j + i] + 0x4B400000u), 12582912.0f);
                acc[j + i] = __fmaf_rn(f, sc[i], acc[j + i]);
              }
            }
          }
        }
        if (!ok) break;
        if (m < g.M) {
          const float st = Cfg::EPI == EPI_GS128 ? __ldg(g.s_tok + m) : 1.0f;
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out) + static_cast<size_t>(m) * g.N;
#pragma unroll
          for (int j = 0; j < CPT; j += 8) {
            const int n = ct * BN + col0 + j;
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = Cfg::EPI == EPI_GS128 ? __fmul_rn(acc[j + i], st) : acc[j + i];
            if (n + 8 <= g.N)
              *reinterpret_cast<uint4*>(out + n) =
                  make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                             pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
          }
        }
      }
    } else {
      uint32_t local = 0;
      const long long G = gridDim.x, T = g.total_iters;
      const int me = blockIdx.x;
      // Swapped W8A8 tiles hold every token in one chunk (M <= BN): their
      // token scales are read once here, not in the tail of each tile.
      constexpr bool kPreTok =
          Cfg::SWAP && Cfg::I8 && Cfg::EPI == EPI_SCALE && Cfg::CW == Cfg::BN;
      float stok[kPreTok ? Cfg::BN : 1];
      if constexpr (kPreTok) {
#pragma unroll
        for (int j = 0; j < Cfg::BN; ++j)
          stok[j] = (g.s_tok && j < g.M) ? __ldg(g.s_tok + j) : 1.0f;
      }
      while (it.next(g, s)) {
        const uint32_t a = local % NACC, u = local / NACC;
        const int rt = s.tile % g.tiles_r, ct = s.tile / g.tiles_r;
        // the channel scale of this thread's output row, fetched while the
        // MMAs finish (swapped layout: one weight row per thread)
        float sc_pre = 1.0f;  // EPI_W16G: the scales were applied on load
        if constexpr (Cfg::SWAP && Cfg::EPI == EPI_SCALE) {
          const int n = rt * Cfg::BM + rr;
          if (n < g.N) sc_pre = g.s_ch ? __ldg(g.s_ch + n) : 1.0f;
        }
        const float* scp =
            (Cfg::SWAP && (Cfg::EPI == EPI_SCALE || Cfg::EPI == EPI_W16G)) ? &sc_pre : nullptr;
        // swapped W8A8 tiles of one chunk: the token scales in registers
        const float* stp = kPreTok ? stok : nullptr;
        const bool w_ok = wait_bounded(tfull + a, u & 1u, abort_flag);
        if (named_bar_or(1, nthr, !w_ok)) break;
        tc_fence_after();
        const uint32_t tb = lane_base + a * Cfg::NSUB * BN;
        const int nsub = s.kb1 - s.kb0 < Cfg::NSUB ? s.kb1 - s.kb0 : Cfg::NSUB;
        if (s.kb0 == 0 && s.kb1 == g.kb_total) {
#pragma unroll 1
          for (int c = 0; c < BN; c += CW) {
            uint32_t v[CW];
            tmem_ld_acc<Cfg>(tb, c, nsub, v);
            store_chunk<Cfg>(g, rt, ct, rr, c, v, 0, scp, stp);
          }
        } else if (g.csplit > 1) {
          // cluster split-K: the tile's K parts are the ranks of this cluster
          // (rank r = part r); ranks > 0 write their sums into rank 0's shared
          // memory and arrive on its barrier; rank 0 adds them in rank order
          const uint32_t rank = cluster_ctarank();
          uint32_t* red = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_SBLK);
          if (rank != 0) {
            const uint32_t dst = mapa_shared(
                smem_u32(red + (static_cast<size_t>(rank - 1) * Cfg::BM + rr) * BN), 0);
#pragma unroll 1
            for (int c = 0; c < BN; c += CW) {
              uint32_t v[CW];
              tmem_ld_acc<Cfg>(tb, c, nsub, v);
#pragma unroll
              for (int j = 0; j < CW; j += 4)
                st_cluster_v4(dst + (c + j) * 4, v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
            mbar_arrive_cluster(mapa_shared(smem_u32(red_bar), 0));
          } else if (wait_bounded_cluster(red_bar, 0, abort_flag)) {
#pragma unroll 1
            for (int c = 0; c < BN; c += CW) {
              uint32_t v[CW];
              tmem_ld_acc<Cfg>(tb, c, nsub, v);
              for (int r = 1; r < g.csplit; ++r) {
                const uint32_t* prow = red + (static_cast<size_t>(r - 1) * Cfg::BM + rr) * BN + c;
#pragma unroll
                for (int j = 0; j < CW; j += 4) {
                  const uint4 w = *reinterpret_cast<const uint4*>(prow + j);
                  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                  for (int i = 0; i < 4; ++i) {
                    uint32_t& acc = v[j + i];
                    if constexpr (Cfg::I8)
                      acc = static_cast<uint32_t>(static_cast<int32_t>(acc) +
                                                  static_cast<int32_t>(wv[i]));
                    else
                      acc = __float_as_uint(__fadd_rn(__uint_as_float(acc), __uint_as_float(wv[i])));
                  }
                }
              }
              store_chunk<Cfg>(g, rt, ct, rr, c, v, 0, scp, stp);
            }
          }
        } else {
          // stream-K part of a tile: publish, count, and the last arrival reduces
          const long long it0 = static_cast<long long>(s.tile) * g.kb_total;
          const int b_lo = static_cast<int>(sk_owner(it0, G, T));
          const int b_hi = static_cast<int>(sk_owner(it0 + g.kb_total - 1, G, T));
          // slot 0: a CTA's first segment, 1: its last one.  Only the first
          // part of a tile can have started in an earlier tile.
          const int lo_slot = sk_start(b_lo, G, T) < it0 ? 1 : 0;
          const int slot = me == b_lo ? lo_slot : 0;
          uint32_t* wrow = g.ws + (static_cast<size_t>(me * 2 + slot) * Cfg::BM + rr) * BN;
#pragma unroll 1
          for (int c = 0; c < BN; c += CW) {
            uint32_t v[CW];
            tmem_ld_acc<Cfg>(tb, c, nsub, v);
#pragma unroll
            for (int j = 0; j < CW; j += 4)
              *reinterpret_cast<uint4*>(wrow + c + j) = make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          }
          __threadfence();
          named_bar_sync(1, nthr);
          if (ew == 0 && lane == 0) {
            const unsigned prev = atomicAdd(g.ws_cnt + s.tile, 1u);
            const int last = prev == static_cast<unsigned>(b_hi - b_lo);
            if (last) atomicExch(g.ws_cnt + s.tile, 0u);
            *sk_flag = last;
          }
          named_bar_sync(1, nthr);
          if (*sk_flag) {
            __threadfence();
#pragma unroll 1
            for (int c = 0; c < BN; c += CW) {
              uint32_t v[CW];
#pragma unroll
              for (int j = 0; j < CW; ++j) v[j] = 0u;
              // parts are summed in CTA order; up to NB parts' loads in flight
              constexpr int NB = CW >= 32 ? 2 : 4;
              for (int b0 = b_lo; b0 <= b_hi; b0 += NB) {
                int4 w[NB][CW / 4];
#pragma unroll
                for (int u = 0; u < NB; ++u) {
                  const int b = b0 + u;
                  if (b <= b_hi) {
                    const int sl = b == b_lo ? lo_slot : 0;
                    const uint32_t* prow =
                        g.ws + (static_cast<size_t>(b * 2 + sl) * Cfg::BM + rr) * BN + c;
#pragma unroll
                    for (int j = 0; j < CW / 4; ++j) w[u][j] = ld_cg_v4(prow + 4 * j);
                  }
                }
#pragma unroll
                for (int u = 0; u < NB; ++u) {
                  if (b0 + u <= b_hi) {
#pragma unroll
                    for (int j = 0; j < CW / 4; ++j) {
                      const uint32_t wv[4] = {
                          static_cast<uint32_t>(w[u][j].x), static_cast<uint32_t>(w[u][j].y),
                          static_cast<uint32_t>(w[u][j].z), static_cast<uint32_t>(w[u][j].w)};
#pragma unroll
                      for (int i = 0; i < 4; ++i) {
                        uint32_t& acc = v[4 * j + i];
                        if constexpr (Cfg::I8)
                          acc = static_cast<uint32_t>(static_cast<int32_t>(acc) +
                                                      static_cast<int32_t>(wv[i]));
                        else
                          acc = __float_as_uint(__fadd_rn(__uint_as_float(acc),
                                                          __uint_as_float(wv[i])));
                      }
                    }
                  }
                }
              }
              store_chunk<Cfg>(g, rt, ct, rr, c, v, 0, scp, stp);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty + a);
        ++local;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // rank 0 keeps its shared memory until every rank's remote writes are done
  if (g.csplit > 1) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace sq
