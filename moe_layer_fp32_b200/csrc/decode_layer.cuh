// The whole layer in one launch for decode batches (T <= 32 tokens, bf16 experts).
//
// "MoE: dynamism the compiler cannot remove", batch-1 section, and the picx.dev
// summary of the moe-ceilings study, Practical Implications: at small batches the
// MoE layer is launch bound -- a chain of small kernels spends more time starting
// and draining than moving the touched experts' weights.  Here one cooperative
// launch (one CTA per SM, all resident at once) runs every step, separated by
// grid-wide barriers:
//   1. RMSNorm, one token per CTA;
//   2. the router's K-sliced partial logits, (8 tokens x 128 rows) per work item;
//   3. routing (one token per CTA and a barrier; or, for small problems, every
//      token by every CTA), then -- without a barrier -- the counting-sort
//      permutation, built by every CTA (it is small);
//   4. the grouped gate/up GEMM over the routed rows (tcgen05, 16 or 32 token
//      tiles, rows gathered by the GEMM's own TMA; split along K when the tiles
//      fill at most half the SMs);
//   5. the grouped down GEMM (gated bf16 rows of every assignment);
//   6. the combine, element groups spread over all CTAs.
// The TMEM is allocated once for both GEMMs.  Every barrier wait is bounded: a
// CTA that gives up sets device error 2 and skips the remaining steps, so every
// CTA finishes.  The grid barrier's two words live in the workspace: the count is
// left at zero by a completed call, the generation only advances; both are
// cleared by moe_clear_device_status after an error.
#pragma once
#include "gemm_tc.cuh"

namespace moe {

struct DecodeParams {
  TcParams gu;                    // gate/up GEMM (routed + shared problems)
  TcParams dn;                    // down GEMM
  const __nv_bfloat16* x;         // [T, d]
  const float* gamma;             // [d]
  const __nv_bfloat16* w_router;  // [d, E]
  const float* bias;              // [E] or nullptr
  __nv_bfloat16* xn;              // [T, d]
  float* part;                    // [ns, T, E] router partial sums
  int32_t* idx;                   // [T, k]
  float* gate;                    // [T, k]
  int32_t* counts;                // [E]
  int32_t* offsets;               // [E + 1]
  int32_t* perm;                  // [T * k]
  int32_t* slot;                  // [T * k]
  int32_t* dropped;               // [1]
  float* logits_out;              // [T, E] or nullptr
  const uint8_t* w_down;          // [E, f, d] bf16 routed experts' down weights
  const uint8_t* sh_down;         // [S, f, d] or nullptr
  const __nv_bfloat16* y;         // [T * k, d] gated routed rows (written by the down GEMM)
  const float* ys;                // [S, T, d]
  void* out;                      // [T, d] bf16 or fp32
  int out_f32;
  int32_t* err;
  unsigned* grid_bar;             // [2]: arrivals, generation
  long long wait_cycles;
  double eps;
  int T, d, E, k, S, mode, renorm, cap;
  int ns, rows;                   // router: ns K-slices of `rows` rows
  int route_all;                  // every CTA routes every token (no barrier before permuting)
  int n_split_cnt;                // split-K tile counters (gu.split_cnt == dn.split_cnt)
};

constexpr int kDecodeThreads = kTcBaseThreads;
constexpr int kDecodeMaxT = 32;

// Bounded grid-wide barrier of a cooperative launch.  Thread 0 of every CTA
// arrives on bar[0] (adding 1, plus kBarErr if this CTA's step ran out of time);
// the last arrival resets the count and publishes the next generation in bar[1]
// (with its top bit set if any CTA reported a time-out), which the others wait
// for.  Thread 0 keeps the generation it expects in `gen`, read once when the
// kernel starts, so that an arrival costs one atomic and the release one store
// and one reduction, with no other round trip to L2.  Returns false (and sets
// device error 2) if the wait ran out, and when some CTA reported a time-out:
// the caller then takes no further step and arrives at no further barrier, so
// no CTA is ever released from a barrier that another has not reached.  All
// threads of the CTA return the same value.
// Data that one step writes with ordinary stores and a later step reads through
// the TMA (the normalised rows, h) crosses from the generic to the async proxy:
// every thread fences its own stores before the barrier and its later copies
// after it.
constexpr unsigned kBarErr = 1u << 16;
constexpr unsigned kGenErr = 1u << 31;
MOE_DEV bool grid_barrier(unsigned* bar, int nblocks, unsigned& gen, bool mine_ok,
                          long long limit, int32_t* err, int* s_ok) {
  fence_proxy_async_global();
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    // the fence orders the CTA's writes (made visible to this thread by the CTA
    // barrier) before the arrival; the last arrival fences again, so that its
    // release of the new generation carries every CTA's writes to the waiters
    __threadfence();
    const unsigned add = mine_ok ? 1u : 1u + kBarErr;
    const unsigned now = atomicAdd(bar, add) + add;
    const unsigned prev = gen;
    if ((now & (kBarErr - 1)) == (unsigned)nblocks) {
      __threadfence();
      st_relaxed_gpu(bar, 0u);
      const unsigned inc = (now >= kBarErr) ? 1u + kGenErr : 1u;
      red_release_add_gpu(bar + 1, inc);
      gen = prev + inc;
    } else {
      const long long t0 = clock64();
      unsigned g;
      while ((g = ld_acquire_gpu(bar + 1)) == prev) {
        __nanosleep(20);
        if (clock64() - t0 > limit) {
          set_error(err, DEV_TIMEOUT);
          ok = 0;
          break;
        }
      }
      gen = g;
    }
    if ((gen - prev) != 1u) ok = 0;   // a CTA reported a time-out
    *s_ok = ok;
  }
  __syncthreads();
  fence_proxy_async_global();
  return *s_ok != 0;
}

// The counting-sort permutation of n <= 1024 assignments by one warp: counts per
// expert (before capacity), offsets of kept = min(count, cap), and the stable rank
// of every assignment in flat order a = t*k + j.  Same rule as permute_cta.
// `cnt` and `offs` are shared scratches of E ints each.
MOE_DEV void permute_warp(const int32_t* idx, int n, int E, int cap, int32_t* counts,
                          int32_t* offsets, int32_t* perm_assign, int32_t* slot_of,
                          int32_t* n_dropped, int32_t* err, int* cnt, int* offs) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  for (int base = 0; base < n; base += 32) {
    const int a = base + lane;
    int e = -1;
    if (a < n) {
      e = idx[a];
      if (e < 0 || e >= E) { set_error(err, DEV_BAD_EXPERT); e = -1; }
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) cnt[e] += __popc(peers);
    __syncwarp();
  }
  // exclusive scan of kept over the experts, 32 at a time; the counts then restart
  // from zero as the running rank within each expert
  int carry = 0, drop = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    const int tot = e < E ? cnt[e] : 0;
    const int kept = min(tot, cap);
    drop += tot - kept;
    int v = kept;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (e < E) {
      counts[e] = tot;
      offsets[e] = carry + v - kept;
      offs[e] = carry + v - kept;
      cnt[e] = 0;
    }
    carry += __shfl_sync(0xffffffffu, v, 31);
  }
  drop = warp_sum(drop);
  if (lane == 0) {
    offsets[E] = carry;
    *n_dropped = drop;
  }
  __syncwarp();
  for (int base = 0; base < n; base += 32) {
    const int a = base + lane;
    int e = -1;
    if (a < n) {
      e = idx[a];
      if (e < 0 || e >= E) e = -1;
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    int rank = 0;
    if (e >= 0) rank = cnt[e] + __popc(peers & lt);
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) cnt[e] += __popc(peers);
    __syncwarp();
    if (a < n) {
      if (e >= 0 && rank < cap) {
        const int sl = offs[e] + rank;
        slot_of[a] = sl;
        perm_assign[sl] = a;
      } else {
        slot_of[a] = -1;
      }
    }
  }
}

template <int EPL, int BN, int MAXV>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    k_decode_layer(const __grid_constant__ DecodeParams p) {
  using CG = TcConfig<EPI_GATEUP, BN, false, WQ_BF16>;
  using CD = TcConfig<EPI_DOWN, BN, false, WQ_BF16>;
  constexpr uint32_t TMEM_COLS = CG::TMEM_COLS > CD::TMEM_COLS ? CG::TMEM_COLS : CD::TMEM_COLS;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ int s_ok;
  __shared__ double red[8];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = gridDim.x;
  if (warp == 1) {
    tmem_alloc(&tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  unsigned gen = 0;   // thread 0: the grid barrier's current generation
  if (threadIdx.x == 0) gen = ld_acquire_gpu(p.grid_bar + 1);
  bool ok = true;
  // 1. RMSNorm (and the split-K tile counters zeroed, in case a call was cut short)
  if (p.gu.split_cnt)
    for (int i = blockIdx.x * kDecodeThreads + threadIdx.x; i < p.n_split_cnt;
         i += nb * kDecodeThreads)
      p.gu.split_cnt[i] = 0;
  for (int t = blockIdx.x; t < p.T; t += nb)
    rmsnorm_row_bf16v<256, MAXV>(p.x + (size_t)t * p.d, p.gamma, p.xn + (size_t)t * p.d, p.d,
                                 p.eps, red);   // the chain's partition: identical bits
  ok = grid_barrier(p.grid_bar, nb, gen, true, p.wait_cycles, p.err, &s_ok);
  // 2. router partial logits: work item (token group of 8, K-slice)
  if (ok) {
    float* sm_r = reinterpret_cast<float*>(smem);
    const int groups = (p.T + 7) / 8;
    for (int w = blockIdx.x; w < groups * p.ns; w += nb)
      router_vec_tile<8, kDecodeThreads>(p.xn, p.w_router, p.part, p.T, p.d, p.E, p.rows,
                                         (w % groups) * 8, w / groups, sm_r);
    ok = grid_barrier(p.grid_bar, nb, gen, true, p.wait_cycles, p.err, &s_ok);
  }
  // 3. routing.  Small problems (T * ns * E partial sums, at most 32K): every CTA
  //    routes every token itself -- all threads add the partial logits of
  //    (token, expert) pairs in slice order, then warp w selects for tokens w,
  //    w + 10, ... -- writing the same routes to the workspace, so that no grid
  //    barrier is needed before the permutation.  Otherwise CTA t routes token t
  //    and a barrier follows.
  if (ok) {
    float* s_lg = reinterpret_cast<float*>(smem);
    const size_t stride = (size_t)p.T * p.E;
    if (p.route_all) {
      for (int i = threadIdx.x; i < p.T * p.E; i += kDecodeThreads) {
        const float* pe = p.part + i;   // [slice][t][e], i = t * E + e
        float acc = 0.f;
#pragma unroll 8
        for (int sl = 0; sl < p.ns; ++sl) acc += pe[sl * stride];
        s_lg[i] = acc;
      }
      __syncthreads();
      for (int t = warp; t < p.T; t += kDecodeThreads / 32) {
        float lg[EPL];
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          lg[i] = lane + 32 * i < p.E ? s_lg[t * p.E + lane + 32 * i] : 0.f;
        route_select<EPL>(lg, p.E, p.k, p.bias, p.mode, p.renorm, p.idx, p.gate, p.logits_out,
                          t, lane);
      }
      __syncthreads();   // this CTA's routes, written above, are what its permutation reads
    } else {
      for (int t = blockIdx.x; t < p.T; t += nb) {
        for (int e = threadIdx.x; e < p.E; e += kDecodeThreads) {
          const float* pe = p.part + (size_t)t * p.E + e;
          float acc = 0.f;
#pragma unroll 8
          for (int sl = 0; sl < p.ns; ++sl) acc += pe[sl * stride];
          s_lg[e] = acc;
        }
        __syncthreads();
        if (warp == 0) {
          float lg[EPL];
#pragma unroll
          for (int i = 0; i < EPL; ++i) lg[i] = lane + 32 * i < p.E ? s_lg[lane + 32 * i] : 0.f;
          route_select<EPL>(lg, p.E, p.k, p.bias, p.mode, p.renorm, p.idx, p.gate, p.logits_out,
                            t, lane);
        }
        __syncthreads();
      }
      ok = grid_barrier(p.grid_bar, nb, gen, true, p.wait_cycles, p.err, &s_ok);
    }
  }
  // the permutation of the T*k <= 1024 assignments: every CTA builds it (one warp),
  // writing the same values to the workspace, and reads back only what it wrote
  // itself -- so no CTA waits for another before its gate/up tiles
  if (ok) {
    if (warp == 0)
      permute_warp(p.idx, p.T * p.k, p.E, p.cap, p.counts, p.offsets, p.perm, p.slot, p.dropped,
                   blockIdx.x == 0 ? p.err : nullptr, reinterpret_cast<int*>(smem),
                   reinterpret_cast<int*>(smem) + p.E);
    __syncthreads();
  }
  // 4. + 5. the expert GEMMs.  The CTAs that get no gate/up tile first bring the
  // touched experts' down weights into L2, 32 KB per prefetch, spread over them,
  // so that the down step starts on warm lines while gate/up streams its own.
  if (ok && warp == 0) {
    const int nt = p.dn.prob[0].K / 128;   // gate/up feature tiles per token tile (f / 128)
    int gu_tiles = 0;
    for (int g = lane; g < p.E; g += 32) {
      const int rows = p.offsets[g + 1] - p.offsets[g];
      gu_tiles += (rows + BN - 1) / BN;
    }
    gu_tiles = warp_sum(gu_tiles) * nt + p.S * ((p.T + BN - 1) / BN) * nt;
    const int items = gu_tiles * split_parts(p.gu, gu_tiles, nb);   // the GEMM's work items
    const int idle = nb - items, me = (int)blockIdx.x - items;
    if (me >= 0) {
      constexpr uint32_t kChunk = 32 * 1024;
      const size_t per = (size_t)p.dn.prob[0].K * p.d * 2;   // one expert's W_down bytes
      const uint32_t chunks = (uint32_t)(per / kChunk);        // f, d multiples of 128: exact
      uint32_t c0 = 0;                                         // chunks of the experts before
      for (int g = 0; g < p.E + p.S; ++g) {
        const bool routed = g < p.E;
        if (routed && p.offsets[g + 1] == p.offsets[g]) continue;
        const uint8_t* base = routed ? p.w_down + (size_t)g * per : p.sh_down + (size_t)(g - p.E) * per;
        // chunk j of this expert goes to idle CTA (c0 + j) % idle
        for (uint32_t j = (uint32_t)lane; j < chunks; j += 32)
          if ((int)((c0 + j) % (uint32_t)idle) == me) prefetch_l2_bulk(base + (size_t)j * kChunk, kChunk);
        c0 += chunks;
      }
    }
  }
  if (ok) {
    const bool mine = tc_gemm_run<EPI_GATEUP, BN, false, WQ_BF16>(p.gu, smem, &tmem_slot,
                                                                 blockIdx.x, nb, false);
    ok = grid_barrier(p.grid_bar, nb, gen, mine, p.wait_cycles, p.err, &s_ok);
  }
  if (ok) {
    const bool mine = tc_gemm_run<EPI_DOWN, BN, false, WQ_BF16>(p.dn, smem, &tmem_slot,
                                                               blockIdx.x, nb, false);
    ok = grid_barrier(p.grid_bar, nb, gen, mine, p.wait_cycles, p.err, &s_ok);
  }
  // 6. combine (4 columns per thread; every tensor is 16-byte aligned here)
  if (ok) {
    const size_t n = (size_t)p.T * (p.d / 4);
    for (size_t i = (size_t)blockIdx.x * kDecodeThreads + threadIdx.x; i < n;
         i += (size_t)nb * kDecodeThreads) {
      if (p.out_f32)
        combine_elems<__nv_bfloat16, float, __nv_bfloat16, 4>(
            p.y, p.slot, p.ys, p.S, p.x, static_cast<float*>(p.out), p.T, p.d, p.k, i);
      else
        combine_elems<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16, 4>(
            p.y, p.slot, p.ys, p.S, p.x, static_cast<__nv_bfloat16*>(p.out), p.T, p.d, p.k, i);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_slot, TMEM_COLS);
  }
}

}  // namespace moe
