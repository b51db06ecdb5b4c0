// Grouped expert GEMM on CTA pairs (tcgen05 cta_group::2) for prefill tiles.
//
// "MoE: dynamism the compiler cannot remove", grouped GEMM section: one launch over
// all experts' rows, each block finding its expert from the per-expert offsets.
// Here a cluster of two CTAs takes a tile of 256 tokens of one expert: the even
// CTA holds token rows m0 .. m0+127, the odd CTA rows m0+128 .. m0+255, and one
// MMA of M = 256 tokens x N = 256 columns covers both.  Each CTA stages its own
// 128 token rows and HALF of the 256 weight columns:
//   GATEUP: the even CTA stages 128 features of W_gate, the odd CTA the same 128
//           features of W_up, so every CTA's accumulator holds [gate | up] for its
//           rows and the SwiGLU stays local;
//   DOWN:   the even CTA stages output features n0 .. n0+127, the odd n0+128 ..
//           n0+255.
// Per 64-deep k-block an SM then moves 32 KB into shared memory and the MMA reads
// 32 KB of it for 128 x 256 x 64 multiply-adds; the single-CTA kernel moves and
// reads 48 KB for the same work: a third fewer staged bytes per flop, and the
// tensor pipe busier (79% against 73.5% of the launch on a V3-shaped batch).  The
// 256-token tiles pad more, though, so pairs pay off only from about 512 rows per
// expert (the host's choice); below that the single CTAs are faster.
//
// Synchronisation (no TMA multicast: each CTA loads only into its own memory):
//   full[s]   (even CTA) stage s of BOTH CTAs: the even producer arms it with both
//             CTAs' bytes, and each CTA's TMA loads complete on it (the pair form
//             of the copy, whose barrier may sit in the peer);
//   empty[s]  (each CTA) stage s consumed: the MMA thread commits to both CTAs;
//   tfull[a]  (each CTA) accumulator a complete: commits to both CTAs;
//   tempty[a] (even CTA) accumulator a drained: 8 epilogue warps of each CTA.
// Every wait is bounded; a CTA that gives up raises its own and its peer's abort
// flag.  After an abort the even CTA drains its issued MMAs and the stages it
// armed (which cover the odd CTA's copies of those stages); the odd CTA, which
// cannot observe its copies on the peer's barrier, waits a fixed 2^21 cycles
// (about a millisecond, orders of magnitude above a copy's latency) for any copy
// of a stage the even CTA did not arm; both then meet at a final cluster barrier
// before the TMEM is released.
#pragma once
#include "gemm_tc.cuh"

namespace moe {

template <int EPI, int WQ = WQ_BF16>
struct PairConfig {
  static constexpr bool QUANT = WQ != WQ_BF16;
  static constexpr int BN = 256;                                   // tokens per pair tile
  static constexpr int TILE_N = EPI == EPI_GATEUP ? 128 : 256;     // features per tile
  static constexpr uint32_t B_HALF = 128 * 64 * 2;   // 128 weight columns x 64 k
  static constexpr uint32_t A_BYTES = 128 * 64 * 2;  // 128 token rows x 64 k
  // quantised weights: this CTA's 128 features x 64 codes, K-contiguous rows, and
  // their 128 bf16 scales in a 1 KB slot
  static constexpr uint32_t RAW_ROW = ByteWeights<WQ>::value ? 64 : WQ == WQ_INT4 ? 32 : 0;
  static constexpr uint32_t RAW_BYTES = 128 * RAW_ROW;
  static constexpr uint32_t SCALE_BYTES = QUANT ? 256 : 0;
  // bf16 stage: [weights | tokens]; quantised stage: [tokens | codes | scales]
  static constexpr uint32_t STAGE_BYTES = QUANT ? A_BYTES + RAW_BYTES + 1024 : B_HALF + A_BYTES;
  static constexpr uint32_t TOKEN_OFF = QUANT ? 0 : B_HALF;
  static constexpr uint32_t RAW_OFF = A_BYTES;
  static constexpr uint32_t SCALE_OFF = A_BYTES + RAW_BYTES;
  // quantised: shared-memory slots of this CTA's expanded weights (the MMA's B
  // half), 128 rows of 128 B, K-major with the 128-byte swizzle
  static constexpr uint32_t W_SLOT_BYTES = QUANT ? 128 * 128 : 0;
  static constexpr int W_SLOTS = 4;   // expansion runs up to four k-blocks ahead
  static constexpr uint32_t W_REGION = W_SLOTS * W_SLOT_BYTES;
  static constexpr int STAGES_RAW = (184 * 1024 - W_REGION) / STAGE_BYTES;
  static constexpr int STAGES = QUANT ? (STAGES_RAW > 8 ? 8 : STAGES_RAW) : 6;
  static constexpr uint32_t ACC_COLS = 256;
  static constexpr uint32_t TMEM_COLS = 512;
  // A = tokens (K-major); B = weights, bf16 MN-major as loaded, expanded K-major;
  // M = 256 tokens, N = 256 columns
  static constexpr uint32_t IDESC = idesc_bf16(256, 256, false, !QUANT);
  // two dequantisation threads per feature of this CTA's half, each for 32 codes
  static constexpr int DEQ_WARPS = QUANT ? 8 : 0;
  static constexpr int THREADS = kTcBaseThreads + 32 * DEQ_WARPS;
  // full, empty, [raw full] per stage; tfull, tempty, drain; [deq, wempty] x 2
  static constexpr uint32_t BAR_BYTES =
      8 * (2 * STAGES + 5 + (QUANT ? STAGES + 3 * W_SLOTS : 0)) + 16 + 4 * STAGES;
  static constexpr uint32_t PREFIX_BYTES = 5 * (kMaxGroups + 1) * 4;
  static constexpr uint32_t EPI_BYTES = kEpiWarps * 32 * 16 * 4;
  static constexpr uint32_t SMEM_BYTES =
      1024 + STAGES * STAGE_BYTES + W_REGION + BAR_BYTES + PREFIX_BYTES + 16 + EPI_BYTES;
  static_assert(SMEM_BYTES + 64 <= 227 * 1024, "shared memory per CTA (dynamic + static)");
  static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 128-byte swizzle alignment");
};

// Bounded wait of a pair kernel: on time-out it also raises the peer's abort flag;
// a patient wait sleeps between polls (see mbar_wait).
MOE_DEV bool pair_wait(uint64_t* bar, uint32_t parity, const TcParams& p, volatile int* abort,
                       uint32_t peer_abort, bool patient = false) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (patient) __nanosleep(128);
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > p.wait_cycles) {
      set_error(p.err, DEV_TIMEOUT);
      *abort = 1;
      st_shared_remote_u32(peer_abort, 1);
      return false;
    }
  }
}

template <int EPI, int WQ = WQ_BF16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairConfig<EPI, WQ>::THREADS, 1)
    k_tc_gemm_pair(const __grid_constant__ TcParams p) {
  using C = PairConfig<EPI, WQ>;
  constexpr int STAGES = C::STAGES;
  constexpr int BN = C::BN;
  constexpr int TN = C::TILE_N;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint8_t* wslots = tiles + STAGES * C::STAGE_BYTES;   // quantised: expanded weights
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(wslots + C::W_REGION);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;   // [2]
  uint64_t* tempty_bar = tfull_bar + 2;       // [2]
  uint64_t* drain_bar = tempty_bar + 2;       // [1]
  // quantised: this CTA's codes landed [STAGES] (local); both CTAs' weight slot a
  // expanded [W_SLOTS] (the even CTA's, counted by both CTAs' dequantisation warps);
  // this CTA's slot a read by the MMAs [W_SLOTS] (local)
  uint64_t* rawfull_bar = drain_bar + 1;
  uint64_t* deq_bar = rawfull_bar + (C::QUANT ? STAGES : 0);
  uint64_t* wempty_bar = deq_bar + (C::QUANT ? C::W_SLOTS : 0);
  // the other CTA: its slot a expanded [W_SLOTS] (local, relayed to deq_bar)
  uint64_t* deq_local = wempty_bar + (C::QUANT ? C::W_SLOTS : 0);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(deq_local + (C::QUANT ? C::W_SLOTS : 0));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* issued = const_cast<int*>(abort_flag) + 2;   // [STAGES] last issued parity + 1
  int* prefix = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full_bar) + C::BAR_BYTES);
  float* stg_all = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(prefix + 5 * (kMaxGroups + 1)) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();   // 0: the CTA that issues the pair's MMAs
  const uint32_t peer = rank ^ 1u;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      issued[s] = 0;
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 2 * kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    if (C::QUANT) {
      for (int s = 0; s < STAGES; ++s) mbar_init(&rawfull_bar[s], 1);
      for (int a = 0; a < C::W_SLOTS; ++a) {
        mbar_init(&deq_local[a], C::DEQ_WARPS);
        mbar_init(&deq_bar[a], 2 * C::DEQ_WARPS);
        mbar_init(&wempty_bar[a], 1);
      }
    }
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    for (int pi = 0; pi < p.n_prob; ++pi) {
      tma_prefetch_desc(&p.prob[pi].tmA);
      if (EPI == EPI_GATEUP) tma_prefetch_desc(&p.prob[pi].tmA2);
      tma_prefetch_desc(&p.prob[pi].tmB);
      if (C::QUANT) {
        tma_prefetch_desc(&p.prob[pi].tmS);
        if (EPI == EPI_GATEUP) tma_prefetch_desc(&p.prob[pi].tmS2);
      }
    }
  }
  // both CTAs' barriers are initialised (and the TMEM allocated) before either
  // CTA signals the other
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t peer_abort = mapa_shared(const_cast<int*>(abort_flag), peer);
  pdl_wait();
  pdl_trigger();
  if (warp >= 2 && warp - 2 < p.n_prob) {
    const TcProblem& P = p.prob[warp - 2];
    group_tile_prefix(P.offsets, P.G, P.uniform_rows, BN, prefix + (warp - 2) * (kMaxGroups + 1),
                      warp == 2 && P.offsets ? prefix + 4 * (kMaxGroups + 1) : nullptr);
  }
  if (warp == 4 && p.interleave)
    group_class_prefix(p.prob[0].offsets, p.prob[0].G, BN, prefix + 2 * (kMaxGroups + 1),
                       prefix + 3 * (kMaxGroups + 1));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = total_tiles(p, prefix, TN);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    const uint32_t full_even = mapa_shared(full_bar, 0);
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        TileInfo ti;
        decode_tile(p, prefix, BN, TN, tile, ti);
        const TcProblem& P = p.prob[ti.prob];
        // this CTA's half of the weight columns: GATEUP gate (even) / up (odd) at the
        // tile's features; DOWN features n0 + 128 * rank
        const void* wmap = (EPI == EPI_GATEUP && rank == 1) ? (const void*)&P.tmA2
                                                             : (const void*)&P.tmA;
        const int wn = (EPI == EPI_GATEUP) ? ti.n0 : ti.n0 + 128 * (int)rank;
        const int brow = ti.b_row + 128 * (int)rank;
        const int kbl = P.K / 64;
        for (int kb = 0; kb < kbl; ++kb) {
          if (!pair_wait(&empty_bar[stage], phase ^ 1, p, abort_flag, peer_abort)) {
            ok = false;
            break;
          }
          uint8_t* st = tiles + stage * C::STAGE_BYTES;
          issued[stage] = (int)phase + 1;
          const uint32_t fb = full_even + stage * 8;
          if (!C::QUANT) {
            // the even CTA arms the stage for both CTAs' bytes
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * C::STAGE_BYTES);
            tma_load_3d_pair(st, wmap, fb, wn, kb * 64, ti.g);
            tma_load_3d_pair(st + 8192, wmap, fb, wn + 64, kb * 64, ti.g);
          } else {
            // tokens of both CTAs complete on the even CTA's barrier; this CTA's
            // codes and scales on its own, where its dequantisation warps wait.
            // Codes stored K-contiguous [G][N][K bytes] (x: the k-block's byte
            // offset in a feature's row, y: the first feature); scales int8 / fp8
            // [G][N], int4 [G][K/128][N]
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * C::A_BYTES);
            mbar_arrive_expect_tx(&rawfull_bar[stage], C::RAW_BYTES + C::SCALE_BYTES);
            const void* smap = (EPI == EPI_GATEUP && rank == 1) ? (const void*)&P.tmS2
                                                                 : (const void*)&P.tmS;
            tma_load_3d(st + C::RAW_OFF, wmap, &rawfull_bar[stage], kb * (int)C::RAW_ROW, wn, ti.g);
            if (WQ != WQ_INT4)
              tma_load_3d(st + C::SCALE_OFF, smap, &rawfull_bar[stage], wn, ti.g, 0);
            else
              tma_load_3d(st + C::SCALE_OFF, smap, &rawfull_bar[stage], wn, kb / 2, ti.g);
          }
          tma_load_2d_pair(st + C::TOKEN_OFF, &P.tmB, fb, kb * 64, brow);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // -------------------------------------------------- MMA issuer (even CTA)
      const uint32_t empty_peer = mapa_shared(empty_bar, peer);
      const uint32_t tfull_peer = mapa_shared(tfull_bar, peer);
      const uint32_t wempty_peer = mapa_shared(wempty_bar, peer);
      int stage = 0;
      uint32_t phase = 0;
      int aslot = 0;
      uint32_t aphase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        TileInfo ti;
        decode_tile(p, prefix, BN, TN, tile, ti);
        const int kbl = p.prob[ti.prob].K / 64;
        if (!pair_wait(&tempty_bar[acc], acc_phase ^ 1, p, abort_flag, peer_abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < kbl; ++kb) {
          if (!pair_wait(&full_bar[stage], phase, p, abort_flag, peer_abort)) {
            ok = false;
            break;
          }
          if (C::QUANT && !pair_wait(&deq_bar[aslot], aphase, p, abort_flag, peer_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st_addr = smem_u32(tiles + stage * C::STAGE_BYTES);
          const uint32_t w_addr = smem_u32(wslots + aslot * C::W_SLOT_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // tokens: K-major SW128, 16 k = 32 B per step, 8-row groups 1 KB apart;
            // bf16 weights: MN-major SW128, 16 k-rows of 128 B per step, the two
            // 64-column halves 8 KB apart, 8-row groups 1 KB apart; expanded
            // weights: K-major SW128 like the tokens (each CTA's slot at the same
            // offset holds its 128 of the 256 columns)
            const uint64_t ad = sw128_desc(st_addr + C::TOKEN_OFF + kk * 32, 16, 1024);
            const uint64_t bd = C::QUANT ? sw128_desc(w_addr + kk * 32, 16, 1024)
                                         : sw128_desc(st_addr + kk * 2048, 8192, 1024);
            tc2_mma_f16(d_tmem, ad, bd, C::IDESC, (kb != 0 || kk != 0) ? 1u : 0u);
          }
          // stage s (and weight slot a) of both CTAs are free once these MMAs have
          // read them
          tc2_commit(smem_u32(&empty_bar[stage]));
          tc2_commit(empty_peer + stage * 8);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
          if (C::QUANT) {
            tc2_commit(smem_u32(&wempty_bar[aslot]));
            tc2_commit(wempty_peer + aslot * 8);
            if (++aslot == C::W_SLOTS) { aslot = 0; aphase ^= 1; }
          }
        }
        if (!ok) break;
        tc2_commit(smem_u32(&tfull_bar[acc]));
        tc2_commit(tfull_peer + acc * 8);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // every MMA issued above completes before TMEM or the peer's memory is released
      tc2_commit(smem_u32(drain_bar));
      const long long t0 = clock64();
      while (!mbar_try_wait(drain_bar, 0) && clock64() - t0 < kWaitCycles) {}
    } else if (C::QUANT && lane == 0 && rank == 1) {
      // ------------------------------------------ expansion relay (other CTA)
      // once this CTA's eight dequantisation warps have filled weight slot a, count
      // them on the issuing CTA's barrier with one cluster-scope release
      const uint32_t deq_even = mapa_shared(deq_bar, 0);
      int aslot = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        TileInfo ti;
        decode_tile(p, prefix, BN, TN, tile, ti);
        const int kbl = p.prob[ti.prob].K / 64;
        for (int kb = 0; kb < kbl; ++kb) {
          if (!pair_wait(&deq_local[aslot], aphase, p, abort_flag, peer_abort)) {
            ok = false;
            break;
          }
          mbar_arrive_release_cluster(deq_even + aslot * 8, C::DEQ_WARPS);
          if (++aslot == C::W_SLOTS) { aslot = 0; aphase ^= 1; }
        }
      }
    }
    __syncwarp();
  } else if (warp >= 2 + kEpiWarps) {
    if (C::QUANT) {
      // -------------------------------------------------- dequantisation
      // warp w (10..17) expands codes [32 sub, 32 sub + 32) of the k-block, sub =
      // ((w - 10) / 4) % 2, for the 32 features of quadrant w % 4 of this CTA's 128,
      // into row `feature` of the weight slot (16-byte chunk c at c ^ (row & 7)),
      // then counts on the even CTA's expansion barrier with a cluster-scope release
      const int dw = warp - 2 - kEpiWarps;
      const int sub = (dw >> 2) & 1;
      const int feat = (warp & 3) * 32 + lane;
      int stage = 0;
      uint32_t phase = 0;
      int aslot = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        TileInfo ti;
        decode_tile(p, prefix, BN, TN, tile, ti);
        const int kbl = p.prob[ti.prob].K / 64;
        for (int kb = 0; kb < kbl; ++kb) {
          if (!pair_wait(&rawfull_bar[stage], phase, p, abort_flag, peer_abort) ||
              !pair_wait(&wempty_bar[aslot], aphase ^ 1, p, abort_flag, peer_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* st = tiles + stage * C::STAGE_BYTES;
          const __nv_bfloat16 sc = reinterpret_cast<const __nv_bfloat16*>(st + C::SCALE_OFF)[feat];
          uint32_t w[16];
          dequant_row<WQ, 32>(st + C::RAW_OFF + feat * C::RAW_ROW + sub * (C::RAW_ROW / 2), sc,
                              lane, w);
          uint8_t* dst = wslots + aslot * C::W_SLOT_BYTES + feat * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(dst + 16 * ((4 * sub + c) ^ (feat & 7))) =
                make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
          fence_proxy_async_shared();   // the tensor core reads them through the async proxy
          tc_fence_before();
          __syncwarp();
          // the issuing CTA's warps count on its barrier; the other CTA's on a local
          // one, which one relay thread hands over with a single cluster-scope release
          if (lane == 0) mbar_arrive(rank == 0 ? &deq_bar[aslot] : &deq_local[aslot]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
          if (++aslot == C::W_SLOTS) { aslot = 0; aphase ^= 1; }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int half = (warp - 2) >> 2;       // which half of the columns it drains
    float* stg = stg_all + (warp - 2) * (32 * 16);
    const uint32_t tempty_even = mapa_shared(tempty_bar, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total; tile += npairs) {
      TileInfo ti;
      decode_tile(p, prefix, BN, TN, tile, ti);
      const TcProblem& P = p.prob[ti.prob];
      const uint32_t t_base = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      int r;
      float sc;
      direct_row<EPI>(P, ti, 128 * (int)rank + q * 32 + lane, r, sc);
      if (!pair_wait(&tfull_bar[acc], acc_phase, p, abort_flag, peer_abort, true)) break;
      tc_fence_after();
      direct_store<EPI, TN>(P, ti, r, sc, t_base, half, lane, stg);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_even + acc * 8);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    if (rank == 0) {
      // the stages this CTA armed (both CTAs' copies): wait (bounded) for the
      // last phase of each
      for (int s = 0; s < STAGES; ++s) {
        if (issued[s]) {
          const long long t0 = clock64();
          while (!mbar_try_wait_cluster(&full_bar[s], (uint32_t)(issued[s] - 1)) &&
                 clock64() - t0 < kWaitCycles) {}
        }
      }
    } else {
      // copies of this CTA complete on the peer's barrier: give any still in
      // flight a fixed, generous time to land
      const long long t0 = clock64();
      while (clock64() - t0 < (1ll << 21)) {}
    }
    // quantised: this CTA's codes and scales complete on its own barriers
    if (C::QUANT) {
      for (int s = 0; s < STAGES; ++s) {
        if (issued[s]) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&rawfull_bar[s], (uint32_t)(issued[s] - 1)) &&
                 clock64() - t0 < kWaitCycles) {}
        }
      }
    }
  }
  // neither CTA leaves while the pair's MMAs may still read its memory or write its
  // TMEM (the even CTA drained them above)
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace moe
