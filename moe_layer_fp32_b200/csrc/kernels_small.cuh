// CUDA-core kernels of the layer: RMSNorm (a1), the split-K router for small
// batches (a2), softmax/top-k routing (a3), histogram + scan + permutation
// (a4/a5), the row gather for prefill tiles, the combine (a8), and the FP32
// grouped SwiGLU FFN used when the expert weights are fp32.
#pragma once
#include <type_traits>
#include "common.cuh"

namespace moe {

constexpr int kMaxExpertsScan = 512;

// ---------------------------------------------------------------------------
// block reductions
// ---------------------------------------------------------------------------
template <typename V>
MOE_DEV V warp_sum(V v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
MOE_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Tile prefix over the groups of a grouped problem: prefix[g] = number of
// BM-row tiles of groups < g.  rows(g) = off[g+1] - off[g], or `uniform` rows
// when off == nullptr.  Called by one warp; s_off is a shared scratch of G+1.
MOE_DEV void group_tile_prefix(const int32_t* off, int G, int uniform, int BM, int* prefix,
                               int* off_copy = nullptr) {
  const int lane = threadIdx.x & 31;
  int carry = 0;
  if (lane == 0) prefix[0] = 0;
  if (off_copy && lane == 0) off_copy[0] = off[0];
  for (int c = 0; c < G; c += 32) {
    int g = c + lane;
    int rows = 0;
    if (g < G) {
      const int o1 = off ? off[g + 1] : 0;
      rows = off ? (o1 - off[g]) : uniform;
      if (off_copy) off_copy[g + 1] = o1;
    }
    int v = (rows + BM - 1) / BM;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (g < G) prefix[g + 1] = carry + v;
    carry += __shfl_sync(0xffffffffu, v, 31);
  }
}
// Tile prefixes of the two classes of groups of a grouped problem with offsets:
// light groups (1..BM rows, one tile) and heavy groups (more rows).  hpre[g] =
// tiles of heavy groups < g, lpre[g] = light groups < g.  One warp.
MOE_DEV void group_class_prefix(const int32_t* off, int G, int BM, int* hpre, int* lpre) {
  const int lane = threadIdx.x & 31;
  int ch = 0, cl = 0;
  if (lane == 0) { hpre[0] = 0; lpre[0] = 0; }
  for (int c = 0; c < G; c += 32) {
    const int g = c + lane;
    const int rows = g < G ? off[g + 1] - off[g] : 0;
    const int t = (rows + BM - 1) / BM;
    int h = t > 1 ? t : 0, l = t == 1 ? 1 : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yh = __shfl_up_sync(0xffffffffu, h, o);
      const int yl = __shfl_up_sync(0xffffffffu, l, o);
      if (lane >= o) { h += yh; l += yl; }
    }
    if (g < G) { hpre[g + 1] = ch + h; lpre[g + 1] = cl + l; }
    ch += __shfl_sync(0xffffffffu, h, 31);
    cl += __shfl_sync(0xffffffffu, l, 31);
  }
}
// group of tile-row `mt`: largest g with prefix[g] <= mt
MOE_DEV int find_group(const int* prefix, int G, int mt) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------------------
// a1: RMSNorm, one CTA of 256 threads per token.  The sum of squares, the
// scale and the product are taken in double and rounded once to the
// activation type (round-to-nearest-even).
// ---------------------------------------------------------------------------
MOE_DEV void store_act(__nv_bfloat16* p, double v) { *p = bf16_from_double(v); }
MOE_DEV void store_act(float* p, double v) { *p = (float)v; }

// Both RMSNorm kernels also zero `nzero` ints at `zero` (CTA 0): the split-K
// counters of the expert GEMMs that follow later in the same layer.
template <typename TA>
__global__ void __launch_bounds__(256) k_rmsnorm(const TA* __restrict__ x,
                                                 const float* __restrict__ gamma,
                                                 TA* __restrict__ xn, int d, double eps,
                                                 int32_t* __restrict__ zero, int nzero) {
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < nzero; i += 256) zero[i] = 0;
  __shared__ double red[8];
  const size_t row = (size_t)blockIdx.x * d;
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += 256) {
    double v = (double)to_f32(x[row + i]);
    s += v * v;
  }
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  double tot = 0.0;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += red[w];
  const double r = 1.0 / sqrt(tot / d + eps);
  for (int i = threadIdx.x; i < d; i += 256) {
    double v = (double)to_f32(x[row + i]);
    store_act(&xn[row + i], (v * r) * (double)gamma[i]);
  }
}

// Vectorised RMSNorm: each thread keeps up to MAXV 16-byte vectors of the row in
// registers between the sum of squares and the scaling pass (d up to
// 256 * MAXV * 16 / sizeof(TA)).  Same arithmetic as k_rmsnorm.
MOE_DEV void unpack8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) { f[2 * i] = __low2float(h[i]); f[2 * i + 1] = __high2float(h[i]); }
}

// bf16 of (f r) g, the product taken in double and rounded once (bf16_from_double),
// computed in FP32 where that gives the same bf16: f is a bf16 value (exact in FP32),
// r32 = fl32(r), and the two FP32 products carry a relative error below 3 * 2^-24 --
// at most 3 units in the last place of y -- so y rounds to the same bf16 as the
// double product unless its 16 low bits lie within 8 units of the rounding midpoint
// 0x8000 (about 1 in 4000 values), or y is zero, subnormal, huge or not finite;
// those take the double product.
MOE_DEV __nv_bfloat16 bf16_of_scaled(float f, float g, double r, float r32) {
  const float y = (f * r32) * g;
  const uint32_t u = __float_as_uint(y);
  const uint32_t low = u & 0xFFFFu, ex = (u >> 23) & 0xFFu;
  if (ex > 1u && ex < 253u && (low < 0x8000u - 8u || low > 0x8000u + 8u))
    return __float2bfloat16_rn(y);
  return bf16_from_double(((double)f * r) * (double)g);
}

// One token row, vectorised: thread i < NT keeps up to MAXV 16-byte vectors of the
// row in registers between the sum of squares and the scaling pass (d up to
// NT * MAXV * 8).  `red` is a shared scratch of NT / 32 doubles.  Same arithmetic
// as k_rmsnorm.  Every thread of the CTA calls it (the CTA may have more than NT
// threads; the others only join its barriers), and the partition of the row over
// the NT threads -- hence the order of the double sum -- depends on NT alone.
template <int NT, int MAXV>
MOE_DEV void rmsnorm_row_bf16v(const __nv_bfloat16* __restrict__ xrow,
                               const float* __restrict__ gamma,
                               __nv_bfloat16* __restrict__ xnrow, int d, double eps,
                               double* red) {
  const int nv = threadIdx.x < NT ? d / 8 : 0;
  const uint4* xr = reinterpret_cast<const uint4*>(xrow);
  uint4* outr = reinterpret_cast<uint4*>(xnrow);
  uint4 buf[MAXV];
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int v = threadIdx.x + i * NT;
    if (v < nv) {
      buf[i] = xr[v];
      float f[8];
      unpack8(buf[i], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) s += (double)f[j] * (double)f[j];
    }
  }
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0 && threadIdx.x < NT) red[threadIdx.x >> 5] = s;
  __syncthreads();
  double tot = 0.0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) tot += red[w];
  const double r = 1.0 / sqrt(tot / d + eps);
  const float r32 = (float)r;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int v = threadIdx.x + i * NT;
    if (v < nv) {
      float f[8];
      unpack8(buf[i], f);
      const float4 g0 = reinterpret_cast<const float4*>(gamma)[2 * v];
      const float4 g1 = reinterpret_cast<const float4*>(gamma)[2 * v + 1];
      const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      uint4 o;
      __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(&o);
#pragma unroll
      for (int j = 0; j < 8; ++j) ob[j] = bf16_of_scaled(f[j], g[j], r, r32);
      outr[v] = o;
    }
  }
  __syncthreads();   // red may be reused
}

template <int MAXV>
__global__ void __launch_bounds__(256) k_rmsnorm_bf16v(const __nv_bfloat16* __restrict__ x,
                                                       const float* __restrict__ gamma,
                                                       __nv_bfloat16* __restrict__ xn, int d,
                                                       double eps, int32_t* __restrict__ zero,
                                                       int nzero) {
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < nzero; i += 256) zero[i] = 0;
  __shared__ double red[8];
  rmsnorm_row_bf16v<256, MAXV>(x + (size_t)blockIdx.x * d, gamma, xn + (size_t)blockIdx.x * d, d,
                               eps, red);
}

// ---------------------------------------------------------------------------
// a2 (small batches): router logits split over K.  CTA (blockIdx.x, blockIdx.y)
// computes part[y][t][e] = sum_{i in slice y} xn[t][i] * W_r[i][e] for a tile of
// TT tokens; the route kernel adds the slices in order.
// ---------------------------------------------------------------------------
template <typename TA, int TT>
__global__ void __launch_bounds__(256) k_router_split(const TA* __restrict__ xn,
                                                      const TA* __restrict__ wr,
                                                      float* __restrict__ part, int T, int d,
                                                      int E, int slice) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float xs[];   // [TT][slice]
  const int t0 = blockIdx.x * TT;
  const int k0 = blockIdx.y * slice;
  const int kn = min(slice, d - k0);
  for (int i = threadIdx.x; i < TT * slice; i += blockDim.x) {
    int tt = i / slice, kk = i % slice;
    float v = 0.f;
    if (t0 + tt < T && kk < kn) v = to_f32(xn[(size_t)(t0 + tt) * d + k0 + kk]);
    xs[i] = v;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float acc[TT];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) acc[tt] = 0.f;
    for (int kb = 0; kb < kn; kb += 16) {
      float w[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) w[u] = kb + u < kn ? to_f32(wr[(size_t)(k0 + kb + u) * E + e]) : 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (kb + u >= kn) break;
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) acc[tt] = fmaf(xs[tt * slice + kb + u], w[u], acc[tt]);
      }
    }
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
      if (t0 + tt < T) part[((size_t)blockIdx.y * T + t0 + tt) * E + e] = acc[tt];
  }
}

// a2 for small batches with a bf16 router: CTA (blockIdx.x, blockIdx.y) takes TT
// tokens and `rows` consecutive rows of W_r -- one contiguous block of rows * E
// bf16 -- streamed as 16-byte vectors, every load of a thread issued before its
// arithmetic.  Thread t always meets the same 8-column group (256 is a multiple
// of E/8), keeps TT x 8 partial sums in registers, and the threads of a column
// group are summed in a fixed order through shared memory.
// One router tile for TT tokens from t0 and K-slice `slice` of `rows` rows, by
// the first 256 of the calling threads (every calling thread must call it; NT is
// their number).  sm_r: TT * rows + 256 * 8 floats of shared memory.
template <int TT, int NT>
MOE_DEV void router_vec_tile(const __nv_bfloat16* __restrict__ xn,
                             const __nv_bfloat16* __restrict__ wr, float* __restrict__ part,
                             int T, int d, int E, int rows, int t0, int slice, float* sm_r) {
  float* xs = sm_r;                      // [TT][rows]
  float* red = sm_r + TT * rows;         // [256][8]
  const int tid = threadIdx.x;
  const int k0 = slice * rows;
  const int kn = min(rows, d - k0);
  for (int i = tid; i < TT * rows; i += NT) {
    const int tt = i / rows, kk = i % rows;
    xs[i] = (t0 + tt < T && kk < kn) ? __bfloat162float(xn[(size_t)(t0 + tt) * d + k0 + kk]) : 0.f;
  }
  __syncthreads();
  const int cgs = E / 8;
  const int nvec = kn * cgs;
  const uint4* wv = reinterpret_cast<const uint4*>(wr + (size_t)k0 * E);
  float acc[TT][8];
#pragma unroll
  for (int tt = 0; tt < TT; ++tt)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[tt][j] = 0.f;
  if (tid < 256) {
    for (int v0 = tid; v0 < nvec; v0 += 4 * 256) {
      uint4 w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * 256;
        w[u] = v < nvec ? wv[v] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * 256;
        if (v < nvec) {
          float f[8];
          unpack8(w[u], f);
          const int i = v / cgs;
#pragma unroll
          for (int tt = 0; tt < TT; ++tt) {
            const float x = xs[tt * rows + i];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[tt][j] = fmaf(x, f[j], acc[tt][j]);
          }
        }
      }
    }
  }
  const int per = 256 / cgs;   // threads per column group
  for (int tt = 0; tt < TT; ++tt) {
    if (t0 + tt >= T) break;
    if (tid < 256) {
#pragma unroll
      for (int j = 0; j < 8; ++j) red[tid * 8 + j] = acc[tt][j];
    }
    __syncthreads();
    for (int e = tid; e < E; e += NT) {
      const int g = e / 8, j = e % 8;
      float s = 0.f;
      for (int m = 0; m < per; ++m) s += red[(g + m * cgs) * 8 + j];
      part[((size_t)slice * T + t0 + tt) * E + e] = s;
    }
    __syncthreads();
  }
}

// a2 for small batches with a bf16 router: CTA (blockIdx.x, blockIdx.y) takes TT
// tokens and `rows` consecutive rows of W_r -- one contiguous block of rows * E
// bf16 -- streamed as 16-byte vectors, every load of a thread issued before its
// arithmetic.  Thread t always meets the same 8-column group (256 is a multiple
// of E/8), keeps TT x 8 partial sums in registers, and the threads of a column
// group are summed in a fixed order through shared memory.
template <int TT>
__global__ void __launch_bounds__(256) k_router_vec(const __nv_bfloat16* __restrict__ xn,
                                                    const __nv_bfloat16* __restrict__ wr,
                                                    float* __restrict__ part, int T, int d,
                                                    int E, int rows) {
  extern __shared__ float sm_r[];
  pdl_wait();
  pdl_trigger();
  router_vec_tile<TT, 256>(xn, wr, part, T, d, E, rows, blockIdx.x * TT, blockIdx.y, sm_r);
}

// ---------------------------------------------------------------------------
// a3: softmax + top-k + bias + renormalisation, one warp per token.  Lane l
// holds experts l, l+32, ...  Keys are FP32 (logit, plus bias in LOGIT/SELECT
// mode); selection order is (key descending, expert ascending), NaN keys count
// as -inf.  Gates are the FP32 softmax over all E.
// ---------------------------------------------------------------------------
MOE_DEV bool key_better(float ka, int ea, float kb, int eb) {
  return ka > kb || (ka == kb && ea < eb);
}

// Logits of token t for the calling lane's experts (lane, lane + 32, ...): the
// router partials of the ns K-slices added in slice order; their loads are issued
// SU slices at a time for all of the lane's experts together, so that they overlap
// instead of each waiting for the previous add.
template <int EPL>
MOE_DEV void router_logits_of_lane(const float* part, int ns, int T, int E, int t, int lane,
                                   float (&lg)[EPL]) {
  constexpr int SU = EPL <= 4 ? 4 : EPL <= 8 ? 2 : 1;
  const size_t sstride = (size_t)T * E;
  const float* pt = part + (size_t)t * E + lane;
#pragma unroll
  for (int i = 0; i < EPL; ++i) lg[i] = 0.f;
  for (int s0 = 0; s0 < ns; s0 += SU) {
    float v[EPL][SU];
#pragma unroll
    for (int i = 0; i < EPL; ++i)
#pragma unroll
      for (int u = 0; u < SU; ++u)
        v[i][u] = (lane + 32 * i < E && s0 + u < ns) ? pt[(size_t)(s0 + u) * sstride + 32 * i] : 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
#pragma unroll
      for (int u = 0; u < SU; ++u)
        if (s0 + u < ns) lg[i] += v[i][u];
  }
}

// Routes token t with the calling warp, from its logits lg (lane holds experts
// lane, lane + 32, ...).
template <int EPL>
MOE_DEV void route_select(const float (&lg)[EPL], int E, int k, const float* bias, int mode,
                          int renorm, int32_t* idx, float* gate, float* logits_out, int t,
                          int lane) {
  float key[EPL], pin[EPL];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = -INFINITY;
    pin[i] = -INFINITY;
    if (e < E) {
      const float l = lg[i];
      if (logits_out) logits_out[(size_t)t * E + e] = l;
      float b = (mode != 0 && bias) ? bias[e] : 0.f;
      float sk = (mode != 0) ? l + b : l;
      pin[i] = (mode == 1) ? sk : l;
      key[i] = isnan(sk) ? -INFINITY : sk;
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
  uint32_t taken = 0;
  int my_e = 0;
  float my_p = 0.f;
  for (int j = 0; j < k; ++j) {
    float bk = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && key_better(key[i], e, bk, be)) {
        bk = key[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (key_better(ok, oe, bk, be)) { bk = ok; be = oe; }
    }
    const int owner = be & 31, slot = be >> 5;
    float pv = 0.f;
    if (lane == owner) {
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (i == slot) { taken |= 1u << i; pv = ex[i] / sum; }
    }
    pv = __shfl_sync(0xffffffffu, pv, owner);
    if (lane == j) { my_e = be; my_p = pv; }
  }
  if (renorm) {
    float s = warp_sum(lane < k ? my_p : 0.f);
    my_p = my_p / s;
  }
  if (lane < k) {
    idx[(size_t)t * k + lane] = my_e;
    gate[(size_t)t * k + lane] = my_p;
  }
}

// Routes token t with the calling warp: the router partials added in slice order,
// then the selection.
template <int EPL>
MOE_DEV void route_token(const float* part, int ns, int T, int E, int k, const float* bias,
                         int mode, int renorm, int32_t* idx, float* gate, float* logits_out,
                         int t, int lane) {
  float lg[EPL];
  router_logits_of_lane<EPL>(part, ns, T, E, t, lane, lg);
  route_select<EPL>(lg, E, k, bias, mode, renorm, idx, gate, logits_out, t, lane);
}

template <int EPL>
__global__ void __launch_bounds__(256) k_route(const float* __restrict__ part, int ns, int T,
                                               int E, int k, const float* __restrict__ bias,
                                               int mode, int renorm, int32_t* __restrict__ idx,
                                               float* __restrict__ gate,
                                               float* __restrict__ logits_out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  route_token<EPL>(part, ns, T, E, k, bias, mode, renorm, idx, gate, logits_out, t,
                   threadIdx.x & 31);
}

// ---------------------------------------------------------------------------
// a4 + a5: histogram, scan, capacity and stable permutation in one CTA of
// 1024 threads.  Warp w owns a contiguous chunk of the flat assignments; no
// global atomics.  Pass 1 counts per (warp, expert) with __match_any_sync;
// a per-expert scan over warps gives each warp's base rank; a block scan over
// experts of kept = min(count, cap) gives the offsets; pass 2 assigns
// rank = base + running count + lanes before it with the same expert.
// ---------------------------------------------------------------------------
// idx may have been written earlier in the same kernel (by other warps of this
// CTA, before a __syncthreads), so it is read through the coherent path.
MOE_DEV void permute_cta(const int32_t* idx, int n, int E, int cap, int32_t* counts,
                         int32_t* offsets, int32_t* perm_assign, int32_t* slot_of,
                         int32_t* n_dropped, int32_t* err) {
  extern __shared__ int sm[];
  int* cnt = sm;               // [32][E]
  int* s_off = sm + 32 * E;    // [E]
  __shared__ int wsum[32];
  __shared__ int s_drop;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < 32 * E; i += 1024) cnt[i] = 0;
  if (tid == 0) s_drop = 0;
  __syncthreads();
  const int chunk = (((n + 31) / 32) + 31) & ~31;
  const int beg = warp * chunk, end = min(n, beg + chunk);
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = beg; base < end; base += 32) {
    const int a = base + lane;
    int e = -1;
    if (a < end) {
      e = idx[a];
      if (e < 0 || e >= E) { set_error(err, DEV_BAD_EXPERT); e = -1; }
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) cnt[warp * E + e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  int tot = 0;
  if (tid < E) {
    for (int w = 0; w < 32; ++w) {
      int c = cnt[w * E + tid];
      cnt[w * E + tid] = tot;
      tot += c;
    }
  }
  const int kept = (tid < E) ? min(tot, cap) : 0;
  if (tid < E) {
    counts[tid] = tot;
    if (tot > kept) atomicAdd(&s_drop, tot - kept);
  }
  int v = kept;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) wsum[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    wsum[lane] = w;
  }
  __syncthreads();
  if (tid < E) {
    const int excl = v - kept + (warp > 0 ? wsum[warp - 1] : 0);
    offsets[tid] = excl;
    s_off[tid] = excl;
    if (tid == E - 1) offsets[E] = excl + kept;
  }
  if (tid == 0) *n_dropped = s_drop;
  __syncthreads();
  for (int base = beg; base < end; base += 32) {
    const int a = base + lane;
    int e = -1;
    if (a < end) {
      e = idx[a];
      if (e < 0 || e >= E) e = -1;
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    int rank = 0;
    if (e >= 0) rank = cnt[warp * E + e] + __popc(peers & lt);
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) cnt[warp * E + e] += __popc(peers);
    __syncwarp();
    if (a < end) {
      if (e >= 0 && rank < cap) {
        const int s = s_off[e] + rank;
        slot_of[a] = s;
        perm_assign[s] = a;
      } else {
        slot_of[a] = -1;
      }
    }
  }
}

__global__ void __launch_bounds__(1024) k_permute(const int32_t* __restrict__ idx, int n, int E,
                                                  int cap, int32_t* __restrict__ counts,
                                                  int32_t* __restrict__ offsets,
                                                  int32_t* __restrict__ perm_assign,
                                                  int32_t* __restrict__ slot_of,
                                                  int32_t* __restrict__ n_dropped,
                                                  int32_t* err) {
  pdl_wait();
  pdl_trigger();
  permute_cta(idx, n, E, cap, counts, offsets, perm_assign, slot_of, n_dropped, err);
}

// a3 + a4 + a5 in one CTA for small batches: the 32 warps route the tokens, then
// the same CTA builds the permutation from the routes it just wrote.
template <int EPL>
__global__ void __launch_bounds__(1024) k_route_permute(
    const float* __restrict__ part, int ns, int T, int E, int k, const float* __restrict__ bias,
    int mode, int renorm, int32_t* idx, float* __restrict__ gate, float* __restrict__ logits_out,
    int cap, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm_assign, int32_t* __restrict__ slot_of,
    int32_t* __restrict__ n_dropped, int32_t* err) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = warp; t < T; t += 32)
    route_token<EPL>(part, ns, T, E, k, bias, mode, renorm, idx, gate, logits_out, t, lane);
  __syncthreads();
  permute_cta(idx, T * k, E, cap, counts, offsets, perm_assign, slot_of, n_dropped, err);
}

// ---------------------------------------------------------------------------
// a4 + a5 for large batches: the same counting sort over many CTAs, in three
// launches and still without global atomics.
//   count: CTA b counts its chunk of kPermChunk assignments per expert and
//          writes blk[e * nb + b];
//   scan:  one CTA turns blk into exclusive per-expert bases over the CTAs,
//          and kept / offsets / dropped as in the one-CTA kernel;
//   rank:  CTA b recounts its chunk per warp and assigns
//          rank = CTA base + earlier warps + running count + earlier lanes.
// Each lane holds kPermPerLane assignments in registers (loads issued together).
// ---------------------------------------------------------------------------
constexpr int kPermPerLane = 8;
constexpr int kPermWarps = 8;
constexpr int kPermChunk = kPermWarps * 32 * kPermPerLane;   // 2048 assignments per CTA

MOE_DEV void perm_load_chunk(const int32_t* idx, int n, int E, int base, int lane,
                             int (&e)[kPermPerLane], int32_t* err) {
#pragma unroll
  for (int r = 0; r < kPermPerLane; ++r) {
    const int a = base + r * 32 + lane;
    e[r] = a < n ? idx[a] : -1;
  }
#pragma unroll
  for (int r = 0; r < kPermPerLane; ++r) {
    const int a = base + r * 32 + lane;
    if (a < n && (e[r] < 0 || e[r] >= E)) {
      if (err) set_error(err, DEV_BAD_EXPERT);
      e[r] = -1;
    }
  }
}

MOE_DEV void perm_count_warp(const int (&e)[kPermPerLane], int* cnt_w, int lane) {
#pragma unroll
  for (int r = 0; r < kPermPerLane; ++r) {
    const uint32_t peers = __match_any_sync(0xffffffffu, e[r]);
    if (e[r] >= 0 && lane == __ffs(peers) - 1) cnt_w[e[r]] += __popc(peers);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(256) k_perm_count(const int32_t* __restrict__ idx, int n, int E,
                                                    int nb, int32_t* __restrict__ blk,
                                                    int32_t* err) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int cnt[];   // [8][E]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kPermWarps * E; i += 256) cnt[i] = 0;
  __syncthreads();
  int e[kPermPerLane];
  perm_load_chunk(idx, n, E, blockIdx.x * kPermChunk + warp * 32 * kPermPerLane, lane, e, err);
  perm_count_warp(e, cnt + warp * E, lane);
  __syncthreads();
  for (int x = tid; x < E; x += 256) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < kPermWarps; ++w) s += cnt[w * E + x];
    blk[(size_t)x * nb + blockIdx.x] = s;
  }
}

MOE_DEV int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// exclusive scan of kept = min(tot, cap) over experts (thread e < E holds tot),
// for a CTA of 1024 threads; writes counts, offsets, dropped and s_off
MOE_DEV void expert_offsets_1024(int tot, int E, int cap, int32_t* counts, int32_t* offsets,
                                 int32_t* n_dropped, int* s_off, int* wsum, int* s_drop) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kept = (tid < E) ? min(tot, cap) : 0;
  if (tid < E) {
    counts[tid] = tot;
    if (tot > kept) atomicAdd(s_drop, tot - kept);
  }
  const int v = warp_incl_scan(kept, lane);
  if (lane == 31) wsum[warp] = v;
  __syncthreads();
  if (warp == 0) wsum[lane] = warp_incl_scan(wsum[lane], lane);
  __syncthreads();
  if (tid < E) {
    const int excl = v - kept + (warp > 0 ? wsum[warp - 1] : 0);
    offsets[tid] = excl;
    if (s_off) s_off[tid] = excl;
    if (tid == E - 1) offsets[E] = excl + kept;
  }
  __syncthreads();
  if (tid == 0) *n_dropped = *s_drop;
}

__global__ void __launch_bounds__(1024) k_perm_scan(int32_t* __restrict__ blk, int nb, int E,
                                                    int cap, int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ n_dropped) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_tot[kMaxExpertsScan];
  __shared__ int wsum[32];
  __shared__ int s_drop;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_drop = 0;
  const int nch = (nb + 31) / 32;
  const int per_w = (E + 31) / 32;
  const int pairs = per_w * nch;
  int carry = 0;
  for (int p0 = 0; p0 < pairs; p0 += 8) {
    int v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int p = p0 + u;
      const int e = warp + 32 * (p / nch), b = (p % nch) * 32 + lane;
      v[u] = (p < pairs && e < E && b < nb) ? blk[(size_t)e * nb + b] : 0;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int p = p0 + u;
      if (p >= pairs) break;
      const int e = warp + 32 * (p / nch), c = p % nch, b = c * 32 + lane;
      if (c == 0) carry = 0;
      const int incl = warp_incl_scan(v[u], lane);
      if (e < E && b < nb) blk[(size_t)e * nb + b] = carry + incl - v[u];
      carry += __shfl_sync(0xffffffffu, incl, 31);
      if (c == nch - 1 && lane == 0 && e < E) s_tot[e] = carry;
    }
  }
  __syncthreads();
  expert_offsets_1024(tid < E ? s_tot[tid] : 0, E, cap, counts, offsets, n_dropped, nullptr,
                      wsum, &s_drop);
}

__global__ void __launch_bounds__(256) k_perm_rank(const int32_t* __restrict__ idx, int n, int E,
                                                   int nb, int cap,
                                                   const int32_t* __restrict__ blk,
                                                   const int32_t* __restrict__ offsets,
                                                   int32_t* __restrict__ perm_assign,
                                                   int32_t* __restrict__ slot_of) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int sm[];
  int* cnt = sm;                       // [8][E]
  int* s_off = sm + kPermWarps * E;    // [E]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kPermWarps * E; i += 256) cnt[i] = 0;
  for (int i = tid; i < E; i += 256) s_off[i] = offsets[i];
  __syncthreads();
  const int base = blockIdx.x * kPermChunk + warp * 32 * kPermPerLane;
  int e[kPermPerLane];
  perm_load_chunk(idx, n, E, base, lane, e, nullptr);
  perm_count_warp(e, cnt + warp * E, lane);
  __syncthreads();
  for (int x = tid; x < E; x += 256) {
    int run = blk[(size_t)x * nb + blockIdx.x];
#pragma unroll
    for (int w = 0; w < kPermWarps; ++w) {
      const int c = cnt[w * E + x];
      cnt[w * E + x] = run;
      run += c;
    }
  }
  __syncthreads();
  int* cw = cnt + warp * E;
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int r = 0; r < kPermPerLane; ++r) {
    const int a = base + r * 32 + lane;
    const uint32_t peers = __match_any_sync(0xffffffffu, e[r]);
    int rank = 0;
    if (e[r] >= 0) rank = cw[e[r]] + __popc(peers & lt);
    __syncwarp();
    if (e[r] >= 0 && lane == __ffs(peers) - 1) cw[e[r]] += __popc(peers);
    __syncwarp();
    if (a < n) {
      if (e[r] >= 0 && rank < cap) {
        const int sl = s_off[e[r]] + rank;
        slot_of[a] = sl;
        perm_assign[sl] = a;
      } else {
        slot_of[a] = -1;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// gather for wide (prefill) token tiles: xp[s] = xn[perm_assign[s] / k] for
// s < offsets[E]; one warp per row, 16-byte vectors (d * sizeof(TA) is a multiple
// of 16).  Narrow tiles gather inside the GEMM instead.
// ---------------------------------------------------------------------------
template <typename TA>
__global__ void __launch_bounds__(256) k_gather_rows(const TA* __restrict__ xn,
                                                     const int32_t* __restrict__ perm_assign,
                                                     const int32_t* __restrict__ n_rows_ptr,
                                                     int k, int d, TA* __restrict__ xp) {
  pdl_wait();
  pdl_trigger();
  const int n_rows = *n_rows_ptr;
  const int vec_per_row = d * (int)sizeof(TA) / 16;
  const int warps = gridDim.x * 8;
  const int lane = threadIdx.x & 31;
  constexpr int U = 8;   // vectors per lane loaded before they are stored
  for (int s = blockIdx.x * 8 + (threadIdx.x >> 5); s < n_rows; s += warps) {
    const int t = perm_assign[s] / k;
    const uint4* src = reinterpret_cast<const uint4*>(xn + (size_t)t * d);
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)s * d);
    for (int i0 = lane; i0 < vec_per_row; i0 += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + 32 * u < vec_per_row) v[u] = src[i0 + 32 * u];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + 32 * u < vec_per_row) dst[i0 + 32 * u] = v[u];
    }
  }
}

// The same gather token by token: xp[slot_of[t k + j]] = xn[t] for every kept
// assignment (slot >= 0).  One warp per token reads its row once and writes it to
// each of its (at most 32) slots, so that xn is read from memory once instead of
// once per assignment; the rows written are those of k_gather_rows.
template <typename TA>
__global__ void __launch_bounds__(256) k_gather_rows_by_token(const TA* __restrict__ xn,
                                                              const int32_t* __restrict__ slot_of,
                                                              int T, int k, int d,
                                                              TA* __restrict__ xp) {
  pdl_wait();
  pdl_trigger();
  const int vec_per_row = d * (int)sizeof(TA) / 16;
  const int warps = gridDim.x * 8;
  const int lane = threadIdx.x & 31;
  constexpr int U = 8;   // vectors per lane loaded before they are stored
  for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < T; t += warps) {
    const int my_slot = lane < k ? slot_of[(size_t)t * k + lane] : -1;
    const uint4* src = reinterpret_cast<const uint4*>(xn + (size_t)t * d);
    for (int i0 = lane; i0 < vec_per_row; i0 += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + 32 * u < vec_per_row) v[u] = src[i0 + 32 * u];
      for (int j = 0; j < k; ++j) {
        const int sl = __shfl_sync(0xffffffffu, my_slot, j);
        if (sl < 0) continue;
        uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)sl * d);
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (i0 + 32 * u < vec_per_row) dst[i0 + 32 * u] = v[u];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// a8: combine, VEC consecutive elements per thread.  out = residual + shared
// experts (s ascending) + kept assignments (j ascending), summed in FP32.  The
// routed rows are FP32, or bf16 inside the layer forward (tensor-core experts),
// widened before the sum.  VEC = 4 needs every tensor 16-byte aligned (d % 8 == 0
// always holds); VEC = 1 takes any alignment.
// ---------------------------------------------------------------------------
template <int VEC>
MOE_DEV void loadv(const float* p, float (&v)[VEC]) {
  if constexpr (VEC == 4 || VEC == 8) {
#pragma unroll
    for (int h = 0; h < VEC / 4; ++h) {
      const float4 a = *reinterpret_cast<const float4*>(p + 4 * h);
      v[4 * h] = a.x; v[4 * h + 1] = a.y; v[4 * h + 2] = a.z; v[4 * h + 3] = a.w;
    }
  } else {
#pragma unroll
    for (int u = 0; u < VEC; ++u) v[u] = p[u];
  }
}
template <int VEC>
MOE_DEV void loadv(const __nv_bfloat16* p, float (&v)[VEC]) {
  if constexpr (VEC == 8) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&w[h]);
      v[2 * h] = __low2float(a); v[2 * h + 1] = __high2float(a);
    }
  } else if constexpr (VEC == 4) {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&q.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&q.y);
    v[0] = __low2float(a); v[1] = __high2float(a); v[2] = __low2float(b); v[3] = __high2float(b);
  } else {
#pragma unroll
    for (int u = 0; u < VEC; ++u) v[u] = __bfloat162float(p[u]);
  }
}
template <int VEC>
MOE_DEV void storev(float* p, const float (&v)[VEC]) {
  if constexpr (VEC == 4 || VEC == 8) {
#pragma unroll
    for (int h = 0; h < VEC / 4; ++h)
      *reinterpret_cast<float4*>(p + 4 * h) =
          make_float4(v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]);
  } else {
#pragma unroll
    for (int u = 0; u < VEC; ++u) p[u] = v[u];
  }
}
template <int VEC>
MOE_DEV void storev(__nv_bfloat16* p, const float (&v)[VEC]) {
  if constexpr (VEC == 8) {
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      __nv_bfloat162 a = __floats2bfloat162_rn(v[2 * h], v[2 * h + 1]);
      w[h] = *reinterpret_cast<uint32_t*>(&a);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (VEC == 4) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) =
        make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
  } else {
#pragma unroll
    for (int u = 0; u < VEC; ++u) p[u] = __float2bfloat16_rn(v[u]);
  }
}

// Element group i (token i / (d / VEC), VEC columns) of the combine.  The rows of
// JB assignments are loaded together, unconditionally (a dropped slot's row is
// read but not added; past k the token's first row is re-read), so that their
// memory latencies overlap; the adds then follow in j order.
template <typename TA, typename TO, typename TY, int VEC>
MOE_DEV void combine_elems(const TY* __restrict__ y, const int32_t* __restrict__ slot_of,
                           const float* __restrict__ ys, int S, const TA* __restrict__ res,
                           TO* __restrict__ out, int T, int d, int k, size_t i) {
  constexpr int JB = 8;
  const int q = d / VEC;
  const int t = (int)(i / q);
  const int c = (int)(i % q) * VEC;
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
  const size_t a0 = (size_t)t * k;
  for (int j0 = 0; j0 < k; j0 += JB) {
    int sl[JB];
#pragma unroll
    for (int jj = 0; jj < JB; ++jj) sl[jj] = j0 + jj < k ? slot_of[a0 + j0 + jj] : -1;
    float v[JB][VEC];
#pragma unroll
    for (int jj = 0; jj < JB; ++jj)
      loadv<VEC>(y + (a0 + (j0 + jj < k ? j0 + jj : 0)) * d + c, v[jj]);
#pragma unroll
    for (int jj = 0; jj < JB; ++jj)
      if (sl[jj] >= 0) {
#pragma unroll
        for (int u = 0; u < VEC; ++u) acc[u] += v[jj][u];
      }
  }
  storev<VEC>(out + (size_t)t * d + c, acc);
}

template <typename TA, typename TO, typename TY, int VEC>
__global__ void __launch_bounds__(256) k_combine(const TY* __restrict__ y,
                                                 const int32_t* __restrict__ slot_of,
                                                 const float* __restrict__ ys, int S,
                                                 const TA* __restrict__ res, TO* __restrict__ out,
                                                 int T, int d, int k) {
  pdl_wait();
  pdl_trigger();
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)T * (d / VEC)) return;
  combine_elems<TA, TO, TY, VEC>(y, slot_of, ys, S, res, out, T, d, k, i);
}

// ---------------------------------------------------------------------------
// FP32 grouped SwiGLU FFN on the CUDA cores (fp32 expert weights).
// A CTA of 128 threads takes a tile of up to RB rows of one group and 128
// output features; each thread owns one feature.  Groups come from the routed
// segments (offsets) followed by the shared experts (T rows each).
// ---------------------------------------------------------------------------
struct SimtArgs {
  const float* xn;           // [T, d] (rows gathered through perm_assign)
  const int32_t* offsets;    // [E+1]
  const int32_t* perm_assign;
  const float* gate;         // [T*k]
  const float* wg; const float* wu; const float* wd;        // routed [E,...]
  const float* swg; const float* swu; const float* swd;     // shared [S,...]
  float* h;                  // [T*k + S*T, f]
  float* y;                  // [T*k, d]
  float* ys;                 // [S, T, d]
  int T, d, f, k, E, S;
};

constexpr int kSimtRB = 8;     // rows (token slots) per tile
constexpr int kSimtKC = 256;   // k-rows of x staged in shared memory at a time
constexpr int kSimtWarps = 8;  // warps per CTA, each taking every 8th k-row
constexpr int kSimtBatch = 8;  // k-rows of weights loaded before they are used
static_assert(kSimtRB == kSimtWarps, "warp w finishes row w of the tile");

MOE_DEV float silu_f32(float u) { return u / (1.f + expf(-u)); }

// Tile of kSimtRB rows x (32 * VEC) columns.  Each warp accumulates the rows'
// products over its share of K (k-rows w, w + 8, ...), a lane holding VEC
// adjacent columns loaded as one vector; the 8 warps' partial sums are then added
// in warp order in shared memory, so the result does not depend on timing.
// Dynamic shared memory: kSimtWarps * kSimtRB * 32 * VEC * (DOWN ? 1 : 2) floats
// (this also holds the staged x rows, kSimtRB * kSimtKC floats).
template <bool DOWN, int VEC>
__global__ void __launch_bounds__(256) k_simt_ffn(SimtArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int TW = 32 * VEC;
  using VT = typename std::conditional<VEC == 4, float4, float>::type;
  extern __shared__ float sm_f[];
  float* xs = sm_f;     // [kSimtRB][kSimtKC] during the K loop
  float* red = sm_f;    // [NM][kSimtWarps][kSimtRB][TW] afterwards
  __shared__ int prefix[520];   // at most 512 groups + 1
  __shared__ int rows_src[kSimtRB];
  __shared__ int rows_out[kSimtRB];
  __shared__ float rows_scale[kSimtRB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = DOWN ? a.d : a.f;
  const int K = DOWN ? a.f : a.d;
  const int n_tiles = (N + TW - 1) / TW;
  if (threadIdx.x < 32) group_tile_prefix(a.offsets, a.E, 0, kSimtRB, prefix);
  __syncthreads();
  const int routed_mt = prefix[a.E];
  const int shared_mt_per = (a.T + kSimtRB - 1) / kSimtRB;
  const int total = (routed_mt + a.S * shared_mt_per) * n_tiles;
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const int mt = tile / n_tiles, nt = tile % n_tiles;
    const bool shared = mt >= routed_mt;
    int g, r0, rows;
    if (!shared) {
      g = find_group(prefix, a.E, mt);
      r0 = a.offsets[g] + (mt - prefix[g]) * kSimtRB;
      rows = min(kSimtRB, a.offsets[g + 1] - r0);
    } else {
      const int m2 = mt - routed_mt;
      g = m2 / shared_mt_per;
      r0 = (m2 % shared_mt_per) * kSimtRB;
      rows = min(kSimtRB, a.T - r0);
    }
    __syncthreads();   // the previous tile is done with rows_* and the buffer
    if (threadIdx.x < kSimtRB) {
      const int r = threadIdx.x;
      int src = -1, dst = -1;
      float sc = 1.f;
      if (r < rows) {
        if (DOWN) {
          src = shared ? a.T * a.k + g * a.T + r0 + r : r0 + r;        // row of h
          if (shared) {
            dst = g * a.T + r0 + r;                                     // row of ys
          } else {
            dst = a.perm_assign[r0 + r];                                // row of y
            sc = a.gate[dst];
          }
        } else {
          src = shared ? r0 + r : a.perm_assign[r0 + r] / a.k;          // row of xn
          dst = shared ? a.T * a.k + g * a.T + r0 + r : r0 + r;         // row of h
        }
      }
      rows_src[r] = src;
      rows_out[r] = dst;
      rows_scale[r] = sc;
    }
    const float* W0;
    const float* W1 = nullptr;
    if (DOWN) {
      W0 = (shared ? a.swd : a.wd) + (size_t)g * a.f * a.d;
    } else {
      W0 = (shared ? a.swg : a.wg) + (size_t)g * a.d * a.f;
      W1 = (shared ? a.swu : a.wu) + (size_t)g * a.d * a.f;
    }
    const int n = nt * TW + lane * VEC;
    const bool n_ok = n < N;   // N % VEC == 0, so the whole vector is in range
    float acc0[kSimtRB][VEC], acc1[kSimtRB][VEC];
#pragma unroll
    for (int r = 0; r < kSimtRB; ++r)
#pragma unroll
      for (int v = 0; v < VEC; ++v) { acc0[r][v] = 0.f; acc1[r][v] = 0.f; }
    for (int k0 = 0; k0 < K; k0 += kSimtKC) {
      const int kn = min(kSimtKC, K - k0);
      __syncthreads();
#pragma unroll
      for (int i0 = 0; i0 < kSimtRB * kSimtKC; i0 += 256) {
        const int i = i0 + threadIdx.x;
        const int r = i / kSimtKC, kk = i % kSimtKC;
        float v = 0.f;
        if (rows_src[r] >= 0 && kk < kn) {
          const float* src = DOWN ? a.h + (size_t)rows_src[r] * a.f : a.xn + (size_t)rows_src[r] * a.d;
          v = src[k0 + kk];
        }
        xs[i] = v;
      }
      __syncthreads();
      if (n_ok) {
        for (int kb = warp; kb < kn; kb += kSimtWarps * kSimtBatch) {
          VT wa[kSimtBatch], wb[kSimtBatch];
#pragma unroll
          for (int u = 0; u < kSimtBatch; ++u) {
            const int kk = kb + u * kSimtWarps;
            const size_t off = (size_t)(k0 + kk) * N + n;
            if (kk < kn) {
              wa[u] = *reinterpret_cast<const VT*>(W0 + off);
              if (!DOWN) wb[u] = *reinterpret_cast<const VT*>(W1 + off);
            }
          }
#pragma unroll
          for (int u = 0; u < kSimtBatch; ++u) {
            const int kk = kb + u * kSimtWarps;
            if (kk >= kn) break;
            const float* fa = reinterpret_cast<const float*>(&wa[u]);
            const float* fb = reinterpret_cast<const float*>(&wb[u]);
#pragma unroll
            for (int r = 0; r < kSimtRB; ++r) {
              const float x = xs[r * kSimtKC + kk];
#pragma unroll
              for (int v = 0; v < VEC; ++v) {
                acc0[r][v] = fmaf(x, fa[v], acc0[r][v]);
                if (!DOWN) acc1[r][v] = fmaf(x, fb[v], acc1[r][v]);
              }
            }
          }
        }
      }
    }
    __syncthreads();   // the staged rows are no longer read: reuse the buffer
#pragma unroll
    for (int r = 0; r < kSimtRB; ++r)
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        red[((0 * kSimtWarps + warp) * kSimtRB + r) * TW + lane * VEC + v] = acc0[r][v];
        if (!DOWN) red[((1 * kSimtWarps + warp) * kSimtRB + r) * TW + lane * VEC + v] = acc1[r][v];
      }
    __syncthreads();
    // thread (warp w, lane l) finishes row w, columns l*VEC .. l*VEC+VEC-1
    const int r = warp;
    if (r < rows && n_ok) {
      float o[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int w = 0; w < kSimtWarps; ++w) {
          s0 += red[((0 * kSimtWarps + w) * kSimtRB + r) * TW + lane * VEC + v];
          if (!DOWN) s1 += red[((1 * kSimtWarps + w) * kSimtRB + r) * TW + lane * VEC + v];
        }
        o[v] = DOWN ? s0 * rows_scale[r] : silu_f32(s0) * s1;
      }
      float* dst = DOWN ? (shared ? a.ys : a.y) + (size_t)rows_out[r] * a.d + n
                        : a.h + (size_t)rows_out[r] * a.f + n;
      *reinterpret_cast<VT*>(dst) = *reinterpret_cast<const VT*>(o);
    }
  }
}

}  // namespace moe
