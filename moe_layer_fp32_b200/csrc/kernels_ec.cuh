// Expert-choice routing ("MoE: dynamism the compiler cannot remove", capacity
// section: instead of each token picking k experts, each expert picks its top
// T*k/E tokens; every expert then holds exactly C rows, and a token may get
// several experts or none).
//
//   k_ec_scores   one warp per token: the router partial sums added in order, the
//                 FP32 softmax over the experts -> scores, stored expert-major
//                 [E][T] for the selection (and token-major [T][E] on request);
//   k_ec_select   one CTA per expert: radix select of the C-th largest score
//                 (8 bits per pass, most significant first), then an ordered
//                 compaction in token order -- ties at the threshold go to the
//                 lower tokens -- that writes the expert's C slots e*C + c:
//                 token, gate (its score), the identity output row, and the
//                 token x expert slot map (-1 where not picked).  No global
//                 atomics; deterministic;
//   k_combine_ec  one CTA per token: the token's slots in ascending expert order
//                 (compacted from the slot map), then out = residual + shared
//                 experts + the picked experts' gated rows, summed in FP32 in that
//                 fixed order.
#pragma once
#include "kernels_small.cuh"

namespace moe {

template <int EPL>
__global__ void __launch_bounds__(256) k_ec_scores(const float* __restrict__ part, int ns, int T,
                                                   int E, const float* __restrict__ bias,
                                                   int mode, float* __restrict__ scores_t,
                                                   float* __restrict__ scores_out,
                                                   float* __restrict__ logits_out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  float lg[EPL];
  router_logits_of_lane<EPL>(part, ns, T, E, t, lane, lg);
  float pin[EPL];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    pin[i] = -INFINITY;
    if (e < E) {
      if (logits_out) logits_out[(size_t)t * E + e] = lg[i];
      pin[i] = (mode == 1 && bias) ? lg[i] + bias[e] : lg[i];
      mx = fmaxf(mx, pin[i]);
    }
  }
  mx = warp_max(mx);
  float ex[EPL];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    ex[i] = (lane + 32 * i < E) ? expf(pin[i] - mx) : 0.f;
    sum += ex[i];
  }
  sum = warp_sum(sum);
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const float pv = ex[i] / sum;
      scores_t[(size_t)e * T + t] = pv;
      if (scores_out) scores_out[(size_t)t * E + e] = pv;
    }
  }
}

// Order-preserving key of a score (scores are >= 0): NaN below every number.
MOE_DEV uint32_t ec_key(float f) { return isnan(f) ? 0u : __float_as_uint(f) + 1u; }

// Exclusive prefix of a 0/1 flag over the 1024 threads of the CTA, in thread order,
// and the CTA's total.  `wsum` is a shared scratch of 32 ints.
MOE_DEV int block_flag_scan_1024(bool flag, int* wsum, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t b = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(b & ((1u << lane) - 1u));
  __syncthreads();   // wsum of the previous use has been read
  if (lane == 0) wsum[warp] = __popc(b);
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll 8
  for (int w = 0; w < 32; ++w) {
    const int c = wsum[w];
    if (w < warp) before += c;
    total += c;
  }
  return before + in_warp;
}

__global__ void __launch_bounds__(1024) k_ec_select(const float* __restrict__ scores_t, int T,
                                                    int E, int C, int32_t* __restrict__ tok,
                                                    float* __restrict__ gate,
                                                    int32_t* __restrict__ yrow,
                                                    int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ slot_te) {
  pdl_wait();
  pdl_trigger();
  __shared__ int hist[256];
  __shared__ int wsum[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_rank;
  const int e = blockIdx.x, tid = threadIdx.x;
  const float* key = scores_t + (size_t)e * T;
  // radix select of the C-th largest key: after the four passes `prefix` is that
  // key and `r` the number of keys equal to it that are picked
  uint32_t prefix = 0, mask = 0;
  int r = C;
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    for (int t = tid; t < T; t += 1024) {
      const uint32_t u = ec_key(key[t]);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // lane l holds bins 255 - 8l .. 248 - 8l (high bins first)
      int c[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = hist[255 - 8 * tid - j]; s += c[j]; }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      int above = incl - s;   // keys in higher bins than this lane's
      if (above < r && r <= incl) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (above < r && r <= above + c[j]) {
            s_prefix = prefix | ((uint32_t)(255 - 8 * tid - j) << shift);
            s_rank = r - above;
          }
          above += c[j];
        }
      }
    }
    __syncthreads();
    prefix = s_prefix;
    r = s_rank;
    mask |= 255u << shift;
  }
  // picked: key above the threshold, or equal to it and among the first r such
  // tokens; slots in token order
  int carry_tie = 0, carry_sel = 0;
  for (int t0 = 0; t0 < T; t0 += 1024) {
    const int t = t0 + tid;
    const uint32_t u = t < T ? ec_key(key[t]) : 0u;
    const bool tie = t < T && u == prefix;
    int n_tie, n_sel;
    const int tie_rank = carry_tie + block_flag_scan_1024(tie, wsum, n_tie);
    const bool sel = t < T && (u > prefix || (tie && tie_rank < r));
    const int pos = carry_sel + block_flag_scan_1024(sel, wsum, n_sel);
    if (t < T) {
      if (sel) {
        const int sl = e * C + pos;
        tok[sl] = t;
        gate[sl] = key[t];
        yrow[sl] = sl;
        slot_te[(size_t)t * E + e] = sl;
      } else {
        slot_te[(size_t)t * E + e] = -1;
      }
    }
    carry_tie += n_tie;
    carry_sel += n_sel;
  }
  if (tid == 0) {
    offsets[e] = e * C;
    counts[e] = C;
    if (e == E - 1) offsets[E] = E * C;
  }
}

template <typename TA, typename TO, typename TY, int VEC>
__global__ void __launch_bounds__(256) k_combine_ec(const TY* __restrict__ y,
                                                    const int32_t* __restrict__ slot_te, int E,
                                                    const float* __restrict__ ys, int S,
                                                    const TA* __restrict__ res,
                                                    TO* __restrict__ out, int T, int d) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_list[kMaxExpertsScan];
  __shared__ int wsum[8];
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // this token's slots in ascending expert order
  int n = 0;
  for (int e0 = 0; e0 < E; e0 += 256) {
    const int e = e0 + tid;
    const int sl = e < E ? slot_te[(size_t)t * E + e] : -1;
    const uint32_t b = __ballot_sync(0xffffffffu, sl >= 0);
    if (lane == 0) wsum[warp] = __popc(b);
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      if (w < warp) before += wsum[w];
      total += wsum[w];
    }
    if (sl >= 0) s_list[n + before + __popc(b & ((1u << lane) - 1u))] = sl;
    n += total;
    __syncthreads();
  }
  for (int c = tid * VEC; c < d; c += 256 * VEC) {
    float acc[VEC];
#pragma unroll
    for (int u = 0; u < VEC; ++u) acc[u] = 0.f;
    if (res) loadv<VEC>(res + (size_t)t * d + c, acc);
    for (int s = 0; s < S; ++s) {
      float v[VEC];
      loadv<VEC>(ys + ((size_t)s * T + t) * d + c, v);
#pragma unroll
      for (int u = 0; u < VEC; ++u) acc[u] += v[u];
    }
    for (int i = 0; i < n; ++i) {
      float v[VEC];
      loadv<VEC>(y + (size_t)s_list[i] * d + c, v);
#pragma unroll
      for (int u = 0; u < VEC; ++u) acc[u] += v[u];
    }
    storev<VEC>(out + (size_t)t * d + c, acc);
  }
}

}  // namespace moe
