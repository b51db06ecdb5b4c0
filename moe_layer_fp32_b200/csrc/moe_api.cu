// Host side of the C ABI declared in include/moe.h: argument validation,
// workspace layout, TMA tensor-map encoding and the kernel launches.  All
// launches go to the caller's stream; nothing here synchronises except
// moe_get_device_status.
#include <cuda.h>
#include <cuda_runtime.h>
#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels_small.cuh"
#include "gemm_tc.cuh"
#include "gemm_pair.cuh"
#include "kernels_ec.cuh"
#include "decode_layer.cuh"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

inline bool tc_experts(const moe_config* c) { return c->expert_dtype != MOE_F32; }
// the router runs on the tensor cores from this batch size up (bf16 router)
constexpr int kTcRouterMinT = 128;
inline bool tc_router(const moe_config* c) {
  return c->router_dtype == MOE_BF16 && c->T >= kTcRouterMinT;
}
constexpr int kRouterSlice = 128;
constexpr int kRouterTT = 8;
// the vectorised small-batch router needs a bf16 router and E/8 dividing 256
inline bool vec_router(const moe_config* c) {
  return !tc_router(c) && c->router_dtype == MOE_BF16 && c->E % 8 == 0 && 256 % (c->E / 8) == 0;
}
int num_sms();
// Tensor-core router: 128-token tiles, K split into parts (partial logits, added
// in order by the routing kernel) until the SMs are filled; at most 8 parts of at
// least 4 k-blocks each.
inline int tc_router_splits(const moe_config* c) {
  const int tiles = (c->T + 127) / 128 * ((c->E + 127) / 128);
  int s = num_sms() / tiles;
  const int kmax = c->d / 64 / 4;
  if (s > kmax) s = kmax;
  if (s > 8) s = 8;
  return s < 1 ? 1 : s;
}
inline int router_splits(const moe_config* c) {
  if (tc_router(c)) return tc_router_splits(c);
  if (vec_router(c)) return (c->d + kRouterSlice - 1) / kRouterSlice;
  // K-slices of at least 16 rows: small batches get enough CTAs in flight that the
  // weight loads of the many short slices overlap
  int ns = (c->d + 15) / 16;
  int ttiles = (c->T + kRouterTT - 1) / kRouterTT;
  // enough CTAs to cover the SMs a couple of times, no more slices than needed
  int want = (296 + ttiles - 1) / ttiles;
  return ns < want ? ns : (want < 1 ? 1 : want);
}
inline int router_slice(const moe_config* c, int ns) {
  int s = (c->d + ns - 1) / ns;
  return (s + 7) / 8 * 8;
}

// Expert-choice routing: every expert picks C = ceil(C_f * T*k/E) tokens (C_f = 1
// when capacity_factor <= 0), at most T.
inline bool expert_choice(const moe_config* c) { return c->routing == MOE_ROUTE_EXPERT_CHOICE; }
int ec_capacity(const moe_config* c) {
  const double cf = c->capacity_factor > 0.f ? (double)c->capacity_factor : 1.0;
  const double v = std::ceil(cf * c->T * c->k / c->E);
  return v >= (double)c->T ? c->T : (int)v;
}
// routed rows the expert GEMMs hold at most: T*k assignments, or E*C picks
inline size_t n_slots(const moe_config* c) {
  return expert_choice(c) ? (size_t)c->E * ec_capacity(c) : (size_t)c->T * c->k;
}

inline bool quantised(const moe_config* c) {
  return c->expert_dtype == MOE_INT8 || c->expert_dtype == MOE_INT4 ||
         c->expert_dtype == MOE_FP8;
}

// Token-tile width of the expert GEMMs.  Up to 64 rows per expert on average
// (decode), the weights sit on the MMA's M side and a tile holds up to 16, 32 or
// 64 tokens -- as many as one expert can receive (T, or C under expert choice) --
// while each tile's MMA covers only its own rows (rounded up to 16): lightly
// loaded experts cost no more than before and the heavily loaded ones of a skewed
// routing stream their weights once per 64 rows instead of once per 16.  Wider
// (prefill) batches put 128 tokens on M and N = 256 features on the B side; the
// B operand of quantised experts is expanded by the dequantisation warps into
// shared memory (one expansion per 128 tokens, four MMAs per k-block).
int pick_bn(const moe_config* c) {
  const double mean = (double)n_slots(c) / c->E;
  if (mean > 64) return 128;
  const int most = expert_choice(c) ? ec_capacity(c) : c->T;   // rows one expert can get
  return most <= 16 ? 16 : most <= 32 ? 32 : 64;
}
// Decode tiles of bf16 experts gather their rows inside the gate/up GEMM
// (tile::gather4, four rows per copy, only the tile's own rows: a few copies per
// stage, hidden behind the weight stream); prefill tiles would be bound by the
// copy rate, so their rows are gathered once by a kernel into xp and loaded as
// whole tiles.
constexpr int kGather4MaxBN = 64;
constexpr bool kGather4Int = false;   // int8 / int4 / fp8 stages hold 2-4x fewer weight bytes
inline bool gather_in_gemm(const moe_config* c) {
  return pick_bn(c) <= kGather4MaxBN && (kGather4Int || c->expert_dtype == MOE_BF16);
}
// Quantised decode batches whose expert tiles (estimated from the experts they
// can touch) fill the SMs take the direct orientation of the prefill tiles too:
// per k-block four N = 256 MMAs instead of eight N <= 64 ones, the expanded
// weights in shared memory.  The 128 token rows of such a tile are mostly padding,
// but the tensor cores are idle at decode while the issue cost of each MMA and the
// weight expansion bound the swapped tiles.  Smaller batches keep the swapped
// tiles, split along K.
inline bool direct_quant_decode(const moe_config* c) {
  if (!quantised(c) || pick_bn(c) > 64) return false;
  const double touched = std::min<double>((double)c->E, (double)n_slots(c));
  return touched * ((c->f + 127) / 128) >= num_sms();
}
// Token-tile width the expert GEMMs launch with.
inline int tile_bn(const moe_config* c) { return direct_quant_decode(c) ? 128 : pick_bn(c); }
// Split-K of decode tiles when the expert tiles fill at most half the SMs; the
// GEMM decides per launch from the actual tile count.
constexpr bool kSplitBf16 = false;   // int experts only: bf16 tiles stream faster whole
inline bool split_k(const moe_config* c) {
  return tc_experts(c) && tile_bn(c) <= kGather4MaxBN &&
         (kSplitBf16 || c->expert_dtype != MOE_BF16);
}
inline int split_counters() { return num_sms() * 8; }
// Prefill tiles of bf16 experts take the interleaved tile order (light experts'
// tiles spread between the heavy ones'); it changes nothing when every expert
// fills more than one tile.
inline bool interleave_tiles(const moe_config* c) {
  return c->expert_dtype == MOE_BF16 && pick_bn(c) == 128;
}
// Pair tiles of 256 tokens halve each SM's operand traffic per MMA, but an
// expert's last tile is on average half empty, and a half-empty pair tile costs
// what two single tiles do.  Measured on B200 (same bits either way): pairs are
// 2-12% faster from 512 rows per expert up (OLMoE-shaped T=4096, 16384,
// V2-Lite-shaped T=8192) and 7% slower at 295 (DeepSeek-V3-shaped T=9440).
constexpr double kPairMinRowsPerExpert = 512.0;
// Quantised experts on pairs (each CTA expanding half of the 256 weight columns)
// measured slower than on single CTAs (Qwen3-shaped int4 T=16384 gate/up: 1.57 ms
// against 1.16 ms): the automatic choice keeps them on single CTAs.
inline bool pair_tiles(const moe_config* c) {
  if (c->prefill_tiles != 0) return c->prefill_tiles == 2;
  return c->expert_dtype == MOE_BF16 && (double)n_slots(c) / c->E >= kPairMinRowsPerExpert;
}
// Inside the layer forward the gated routed rows of tensor-core experts are kept
// in bf16 (half the bytes the down GEMM writes and the combine reads); the
// grouped-FFN and combine entry points exchange them in FP32.
inline bool y_bf16(const moe_config* c) { return tc_experts(c); }


struct Layout {
  size_t err, xn, part, idx, gate, counts, offsets, perm, slot, dropped, blk, xp, split,
      splitcnt, tilectr, h, y, ys, sct,
      total;
  int ns;
};

moe_status validate(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID;
  if (c->T < 1 || c->d < 8 || c->d % 8 || c->E < 1 || c->E > kMaxGroups || c->k < 1 ||
      c->k > c->E || c->k > 32 || c->f < 1 || c->n_shared < 0 || c->n_shared > 8)
    return MOE_ERR_INVALID;
  if ((long long)c->T * c->k > (1LL << 30)) return MOE_ERR_INVALID;
  if (c->act_dtype != MOE_BF16 && c->act_dtype != MOE_F32) return MOE_ERR_INVALID;
  if (c->out_dtype != MOE_BF16 && c->out_dtype != MOE_F32) return MOE_ERR_INVALID;
  if (c->act_dtype == MOE_F32 && c->out_dtype != MOE_F32) return MOE_ERR_UNSUPPORTED;
  if (c->router_dtype != c->act_dtype) return MOE_ERR_UNSUPPORTED;
  if (c->bias_mode < MOE_BIAS_NONE || c->bias_mode > MOE_BIAS_SELECT) return MOE_ERR_INVALID;
  if (!(c->rms_eps >= 0.f) || !std::isfinite(c->capacity_factor)) return MOE_ERR_INVALID;
  if (c->wait_kcycles < 0) return MOE_ERR_INVALID;
  if (c->routing != MOE_ROUTE_TOPK && c->routing != MOE_ROUTE_EXPERT_CHOICE)
    return MOE_ERR_INVALID;
  if (c->prefill_tiles < 0 || c->prefill_tiles > 2) return MOE_ERR_INVALID;
  if (c->routing == MOE_ROUTE_EXPERT_CHOICE) {
    // the expert picks rank tokens by their gate probability: a selection-only bias
    // has no meaning there; the FP32 (CUDA-core) experts take the top-k path only
    if (c->bias_mode == MOE_BIAS_SELECT) return MOE_ERR_UNSUPPORTED;
    if (c->expert_dtype == MOE_F32) return MOE_ERR_UNSUPPORTED;
    if ((double)c->E * c->T > (double)(1 << 30)) return MOE_ERR_INVALID;
  }
  switch (c->expert_dtype) {
    case MOE_F32:
      if (c->act_dtype != MOE_F32) return MOE_ERR_UNSUPPORTED;
      break;
    case MOE_BF16:
      if (c->act_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
      if (c->d % 128 || c->f % 128 || c->E % 8) return MOE_ERR_UNSUPPORTED;
      break;
    case MOE_INT8:
    case MOE_INT4:
    case MOE_FP8:
      if (c->act_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
      if (c->d % 128 || c->f % 128 || c->E % 8) return MOE_ERR_UNSUPPORTED;
      if (c->expert_dtype == MOE_INT4 && c->group_size != 128) return MOE_ERR_UNSUPPORTED;
      break;
    default:
      return MOE_ERR_INVALID;
  }
  return MOE_OK;
}

Layout layout(const moe_config* c) {
  Layout L{};
  const size_t T = c->T, d = c->d, E = c->E, k = c->k, f = c->f, S = c->n_shared;
  const size_t act = c->act_dtype == MOE_BF16 ? 2 : 4;
  const size_t hb = tc_experts(c) ? 2 : 4;
  L.ns = router_splits(c);
  size_t o = 0;
  L.err = o;      o = align_up(o + 16);
  L.xn = o;       o = align_up(o + T * d * act);
  L.part = o;     o = align_up(o + (size_t)L.ns * T * E * 4);
  // routed rows: T*k assignments (top-k) or E*C picks (expert choice); with expert
  // choice idx / gate / perm hold the picks' token / gate / output row, slot the
  // token x expert slot map and sct the scores expert-major
  const size_t R = n_slots(c);
  const size_t nslot = expert_choice(c) ? T * E : T * k;
  L.idx = o;      o = align_up(o + R * 4);
  L.gate = o;     o = align_up(o + R * 4);
  L.counts = o;   o = align_up(o + E * 4);
  L.offsets = o;  o = align_up(o + (E + 1) * 4);
  L.perm = o;     o = align_up(o + R * 4);
  L.slot = o;     o = align_up(o + nslot * 4);
  L.dropped = o;  o = align_up(o + 16);
  L.blk = o;      o = align_up(o + (size_t)E * ((T * k + kPermChunk - 1) / kPermChunk) * 4);
  L.xp = o;       o = align_up(o + (tc_experts(c) && !gather_in_gemm(c) ? R * d * act : 0));
  L.split = o;    o = align_up(o + (split_k(c) ? (size_t)num_sms() * 2 * pick_bn(c) * 128 * 4 : 0));
  L.splitcnt = o; o = align_up(o + (split_k(c) ? (size_t)split_counters() * 4 : 0));
  // right after the split-K counters (one range zeroes both): the dynamic tile
  // counters of the two expert GEMMs
  L.tilectr = o;  o = align_up(o + 2 * 4);
  L.h = o;        o = align_up(o + (R + S * T) * f * hb);
  L.y = o;        o = align_up(o + R * d * (y_bf16(c) ? 2 : 4));
  L.ys = o;       o = align_up(o + S * T * d * 4);
  L.sct = o;      o = align_up(o + (expert_choice(c) ? T * E * 4 : 0));
  L.total = o;
  return L;
}

template <typename P>
P* at(void* ws, size_t off) { return reinterpret_cast<P*>(static_cast<char*>(ws) + off); }

inline cudaStream_t S_(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Optional per-kernel timing marks: event i+1 is recorded after the i-th launch.
struct Marks {
  cudaEvent_t* ev = nullptr;
  int n = 0, i = 0;
  void mark(cudaStream_t st) {
    if (ev && i < n) cudaEventRecord(ev[i++], st);
  }
};

// Every kernel is launched with programmatic stream serialisation, so that its
// launch overlaps the previous kernel of the stream (the kernels wait for their
// predecessor with griddepcontrol.wait before touching memory).
template <typename Kern, typename... Args>
cudaError_t launch_k(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args... args) {
  cudaLaunchConfig_t c = {};
  c.gridDim = grid;
  c.blockDim = block;
  c.dynamicSmemBytes = smem;
  c.stream = st;
  cudaLaunchAttribute a[1];
  a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a[0].val.programmaticStreamSerializationAllowed = 1;
  c.attrs = a;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, kern, args...);
}
#define MOE_LAUNCH(...)                                             \
  do {                                                              \
    if (launch_k(__VA_ARGS__) != cudaSuccess) return MOE_ERR_CUDA;  \
  } while (0)

moe_status check_launch() {
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status check_ws(const moe_config* c, void* ws, size_t ws_bytes) {
  if (!ws) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return MOE_ERR_WORKSPACE;
  if (ws_bytes < layout(c).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// ----------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// weights [G][K][N] bf16, N contiguous; box 64 features x 64 k x 1
bool map_weights(CUtensorMap* m, const void* base, int G, int K, int N) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !base) return false;
  cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)K, (cuuint64_t)G};
  cuuint64_t strides[2] = {(cuuint64_t)N * 2, (cuuint64_t)K * N * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// raw quantised codes stored K-contiguous, [G][N][KB] bytes (KB = K for int8 /
// fp8, K/2 for int4), no swizzle; box = the codes of one 64-deep k-block
// (row_bytes) for 128 features
bool map_raw(CUtensorMap* m, const void* base, int G, int N, int KB, int row_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !base) return false;
  cuuint64_t dims[3] = {(cuuint64_t)KB, (cuuint64_t)N, (cuuint64_t)G};
  cuuint64_t strides[2] = {(cuuint64_t)KB, (cuuint64_t)N * KB};
  cuuint32_t box[3] = {(cuuint32_t)row_bytes, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// quantisation scales, bf16: int8 [G][N] as (N, G, 1); int4 [G][K/128][N] as
// (N, K/128, G); box 128 features
bool map_scales(CUtensorMap* m, const moe_config* c, const void* base, int G, int K, int N) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !base) return false;
  const bool i4 = c->expert_dtype == MOE_INT4;
  const cuuint64_t kg = i4 ? (cuuint64_t)(K / 128) : (cuuint64_t)G;
  const cuuint64_t g3 = i4 ? (cuuint64_t)G : 1;
  cuuint64_t dims[3] = {(cuuint64_t)N, kg, g3};
  cuuint64_t strides[2] = {(cuuint64_t)N * 2, (cuuint64_t)N * 2 * kg};
  cuuint32_t box[3] = {128, 1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// expert weight matrix of K x N in the storage the GEMM reads (wq): bf16 [G][K][N],
// quantised codes [G][N][K] (int4 [G][N][K/2])
bool map_expert(CUtensorMap* m, int wq, const void* base, int G, int K, int N) {
  if (wq == WQ_INT8 || wq == WQ_FP8) return map_raw(m, base, G, N, K, 64);
  if (wq == WQ_INT4) return map_raw(m, base, G, N, K / 2, 32);
  return map_weights(m, base, G, K, N);
}

inline int wq_of(const moe_config* c) {
  return c->expert_dtype == MOE_INT8   ? WQ_INT8
         : c->expert_dtype == MOE_INT4 ? WQ_INT4
         : c->expert_dtype == MOE_FP8  ? WQ_FP8
                                       : WQ_BF16;
}

// activations [R][K] bf16, K contiguous; box 64 k x BN rows
bool map_rows(CUtensorMap* m, const void* base, int R, int K, int BN) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !base) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)R};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)BN};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, int BN, bool DIRECT = false, int WQ = WQ_BF16>
moe_status launch_tc(const TcParams& p, cudaStream_t st) {
  using C = TcConfig<EPI, BN, DIRECT, WQ>;
  auto kern = k_tc_gemm<EPI, BN, DIRECT, WQ>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  MOE_LAUNCH((kern), num_sms(), C::THREADS, C::SMEM_BYTES, st, p);
  return check_launch();
}

// CTA pairs that can be resident at once.  A cluster's two CTAs must sit in one
// GPC, so a GPC with an odd number of free SMs leaves one idle: the persistent
// grid must not ask for more pairs than fit, or the last ones would run as a
// second wave after the others have finished their share of the tiles.
template <int EPI, int WQ>
int resident_pairs() {
  static int cached[8] = {};   // per device and kernel, on first use
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 8 && cached[dev] > 0) return cached[dev];
  using C = PairConfig<EPI, WQ>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms() / 2 * 2);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (void*)k_tc_gemm_pair<EPI, WQ>, &cfg) != cudaSuccess ||
      n < 1)
    n = 0;
  if (n > num_sms() / 2) n = num_sms() / 2;
  if (dev < 8 && n > 0) cached[dev] = n;
  return n;
}

template <int EPI, int WQ>
moe_status launch_pair(const TcParams& p, cudaStream_t st) {
  using C = PairConfig<EPI, WQ>;
  auto kern = k_tc_gemm_pair<EPI, WQ>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  const int pairs = resident_pairs<EPI, WQ>();
  if (pairs < 1) return MOE_ERR_CUDA;
  MOE_LAUNCH((kern), 2 * pairs, C::THREADS, C::SMEM_BYTES, st, p);
  return check_launch();
}

// Prefill tiles of bf16 experts run on CTA pairs (256 tokens per tile, one
// cta_group::2 MMA per k-step) or on single CTAs (128 tokens), as
// moe_config.prefill_tiles and pair_tiles() decide.
template <int EPI, int WQ>
moe_status launch_tc_bn_q(int bn, bool pair, const TcParams& p, cudaStream_t st) {
  switch (bn) {
    case 16: return launch_tc<EPI, 16, false, WQ>(p, st);
    case 32: return launch_tc<EPI, 32, false, WQ>(p, st);
    case 64: return launch_tc<EPI, 64, false, WQ>(p, st);
    default:   // prefill tiles
      // tokens on M (quantised weights expanded into shared memory)
      if (pair) return launch_pair<EPI, WQ>(p, st);
      return launch_tc<EPI, 128, true, WQ>(p, st);
  }
}

template <int EPI>
moe_status launch_tc_bn(int bn, int wq, bool pair, const TcParams& p, cudaStream_t st) {
  if (wq == WQ_INT8) return launch_tc_bn_q<EPI, WQ_INT8>(bn, pair, p, st);
  if (wq == WQ_INT4) return launch_tc_bn_q<EPI, WQ_INT4>(bn, pair, p, st);
  if (wq == WQ_FP8) return launch_tc_bn_q<EPI, WQ_FP8>(bn, pair, p, st);
  return launch_tc_bn_q<EPI, WQ_BF16>(bn, pair, p, st);
}


// limit of the pipeline waits inside the tensor-core kernels, in clock cycles
long long wait_cycles(const moe_config* c) {
  return c->wait_kcycles > 0 ? (long long)c->wait_kcycles * 1024 : kWaitCycles;
}

int capacity_rows(const moe_config* c) {
  if (!(c->capacity_factor > 0.f)) return INT_MAX;
  double v = std::ceil((double)c->capacity_factor * c->T * c->k / c->E);
  return v >= (double)INT_MAX ? INT_MAX : (int)v;
}

// ----------------------------------------------------------------- the steps
moe_status run_rmsnorm(const moe_config* c, const moe_weights* w, const void* x, void* xn,
                       cudaStream_t st, int32_t* zero = nullptr, int nzero = 0) {
  if (c->act_dtype == MOE_BF16 && c->d <= 256 * 8 * 4 &&
      reinterpret_cast<uintptr_t>(x) % 16 == 0 && reinterpret_cast<uintptr_t>(xn) % 16 == 0 &&
      reinterpret_cast<uintptr_t>(w->rms_gamma) % 16 == 0) {
    const int nv = c->d / 8;
    const double eps = (double)c->rms_eps;
    auto xb = static_cast<const __nv_bfloat16*>(x);
    auto g = static_cast<const float*>(w->rms_gamma);
    auto ob = static_cast<__nv_bfloat16*>(xn);
    if (nv <= 256)
      MOE_LAUNCH((k_rmsnorm_bf16v<1>), c->T, 256, 0, st, xb, g, ob, c->d, eps, zero, nzero);
    else if (nv <= 512)
      MOE_LAUNCH((k_rmsnorm_bf16v<2>), c->T, 256, 0, st, xb, g, ob, c->d, eps, zero, nzero);
    else
      MOE_LAUNCH((k_rmsnorm_bf16v<4>), c->T, 256, 0, st, xb, g, ob, c->d, eps, zero, nzero);
    return check_launch();
  }
  if (c->act_dtype == MOE_BF16)
    MOE_LAUNCH((k_rmsnorm<__nv_bfloat16>), c->T, 256, 0, st, 
        static_cast<const __nv_bfloat16*>(x), static_cast<const float*>(w->rms_gamma),
        static_cast<__nv_bfloat16*>(xn), c->d, (double)c->rms_eps, zero, nzero);
  else
    MOE_LAUNCH((k_rmsnorm<float>), c->T, 256, 0, st, static_cast<const float*>(x),
                                           static_cast<const float*>(w->rms_gamma),
                                           static_cast<float*>(xn), c->d, (double)c->rms_eps,
                                           zero, nzero);
  return check_launch();
}

moe_status run_router(const moe_config* c, const moe_weights* w, const void* xn, float* part,
                      int ns, int32_t* err, cudaStream_t st) {
  if (tc_router(c)) {
    TcParams p{};
    TcProblem& P = p.prob[0];
    if (!map_weights(&P.tmA, w->w_router, 1, c->d, c->E)) return MOE_ERR_CUDA;
    P.tmA2 = P.tmA;
    P.offsets = nullptr;
    P.G = 1;
    P.uniform_rows = c->T;
    P.b_row_base = 0;
    P.b_group_stride = 0;
    P.N = c->E;
    P.K = c->d;
    P.out = part;
    P.out_row_base = 0;
    P.ld_out = c->E;
    P.n_valid = c->E;
    p.n_prob = 1;
    p.err = err;
    p.wait_cycles = wait_cycles(c);
    p.k_splits = ns;
    p.split_out_stride = (size_t)c->T * c->E;
    if (!map_rows(&P.tmB, xn, c->T, c->d, 128)) return MOE_ERR_CUDA;
    return launch_tc<EPI_ROUTER, 128>(p, st);
  }
  // the vectorised router loads 16-byte weight vectors; other alignments take the
  // split kernel below with the same slices
  if (vec_router(c) && (reinterpret_cast<uintptr_t>(w->w_router) & 15) == 0) {
    dim3 grid((c->T + kRouterTT - 1) / kRouterTT, ns);
    const size_t smem = ((size_t)kRouterTT * kRouterSlice + 256 * 8) * 4;
    MOE_LAUNCH((k_router_vec<kRouterTT>), grid, 256, smem, st,
               static_cast<const __nv_bfloat16*>(xn),
               static_cast<const __nv_bfloat16*>(w->w_router), part, c->T, c->d, c->E,
               kRouterSlice);
    return check_launch();
  }
  const int slice = router_slice(c, ns);
  dim3 grid((c->T + kRouterTT - 1) / kRouterTT, ns);
  const size_t smem = (size_t)kRouterTT * slice * 4;
  int threads = c->E >= 256 ? 256 : ((c->E + 31) / 32) * 32;
  if (c->act_dtype == MOE_BF16)
    MOE_LAUNCH((k_router_split<__nv_bfloat16, kRouterTT>), grid, threads, smem, st, 
        static_cast<const __nv_bfloat16*>(xn), static_cast<const __nv_bfloat16*>(w->w_router),
        part, c->T, c->d, c->E, slice);
  else
    MOE_LAUNCH((k_router_split<float, kRouterTT>), grid, threads, smem, st, 
        static_cast<const float*>(xn), static_cast<const float*>(w->w_router), part, c->T,
        c->d, c->E, slice);
  return check_launch();
}

moe_status run_route(const moe_config* c, const float* part, int ns, const float* bias,
                     int32_t* idx, float* gate, float* logits_out, cudaStream_t st) {
  const int blocks = (c->T + 7) / 8;
  const int mode = c->bias_mode;
  if (mode != MOE_BIAS_NONE && !bias) return MOE_ERR_INVALID;
#define MOE_ROUTE(EPL)                                                                     \
  MOE_LAUNCH((k_route<EPL>), blocks, 256, 0, st, part, ns, c->T, c->E, c->k, bias, mode,             \
                                       c->renormalize ? 1 : 0, idx, gate, logits_out)
  if (c->E <= 32) MOE_ROUTE(1);
  else if (c->E <= 64) MOE_ROUTE(2);
  else if (c->E <= 128) MOE_ROUTE(4);
  else if (c->E <= 256) MOE_ROUTE(8);
  else MOE_ROUTE(16);
#undef MOE_ROUTE
  return check_launch();
}

// assignments above which the permutation runs on many CTAs
constexpr int kPermSingleMax = 4096;
inline int perm_blocks(const moe_config* c) {
  return (c->T * c->k + kPermChunk - 1) / kPermChunk;
}

// routing and the one-CTA permutation share a launch up to this many tokens (one
// token per warp of the 1024-thread CTA; beyond that the warps would route in turn)
constexpr int kFusedRouteMaxT = 32;
inline bool fused_route_permute(const moe_config* c) {
  return c->T <= kFusedRouteMaxT && c->T * c->k <= kPermSingleMax;
}

moe_status run_route_permute(const moe_config* c, const float* part, int ns, const float* bias,
                             int32_t* idx, float* gate, float* logits_out, int32_t* counts,
                             int32_t* offsets, int32_t* perm, int32_t* slot, int32_t* dropped,
                             int32_t* err, cudaStream_t st) {
  const int mode = c->bias_mode;
  if (mode != MOE_BIAS_NONE && !bias) return MOE_ERR_INVALID;
  const size_t smem = (size_t)33 * c->E * 4;
#define MOE_ROUTE_PERMUTE(EPL)                                                              \
  do {                                                                                      \
    if (cudaFuncSetAttribute(k_route_permute<EPL>,                                          \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=     \
        cudaSuccess)                                                                        \
      return MOE_ERR_CUDA;                                                                  \
    MOE_LAUNCH((k_route_permute<EPL>), 1, 1024, smem, st, part, ns, c->T, c->E, c->k, bias, \
               mode, c->renormalize ? 1 : 0, idx, gate, logits_out, capacity_rows(c),       \
               counts, offsets, perm, slot, dropped, err);                                  \
  } while (0)
  if (c->E <= 32) MOE_ROUTE_PERMUTE(1);
  else if (c->E <= 64) MOE_ROUTE_PERMUTE(2);
  else if (c->E <= 128) MOE_ROUTE_PERMUTE(4);
  else if (c->E <= 256) MOE_ROUTE_PERMUTE(8);
  else MOE_ROUTE_PERMUTE(16);
#undef MOE_ROUTE_PERMUTE
  return check_launch();
}

moe_status run_permute(const moe_config* c, const int32_t* idx, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* slot, int32_t* dropped,
                       int32_t* err, int32_t* blk, cudaStream_t st) {
  const int n = c->T * c->k;
  if (n > kPermSingleMax && blk) {
    const int nb = perm_blocks(c);
    const size_t sm1 = (size_t)kPermWarps * c->E * 4;
    const size_t sm3 = sm1 + (size_t)c->E * 4;
    if (cudaFuncSetAttribute(k_perm_rank, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm3) != cudaSuccess)
      return MOE_ERR_CUDA;
    MOE_LAUNCH((k_perm_count), nb, 256, sm1, st, idx, n, c->E, nb, blk, err);
    MOE_LAUNCH((k_perm_scan), 1, 1024, 0, st, blk, nb, c->E, capacity_rows(c), counts, offsets, dropped);
    MOE_LAUNCH((k_perm_rank), nb, 256, sm3, st, idx, n, c->E, nb, capacity_rows(c), blk, offsets, perm,
                                      slot);
    return check_launch();
  }
  const size_t smem = (size_t)33 * c->E * 4;
  if (cudaFuncSetAttribute(k_permute, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  MOE_LAUNCH((k_permute), 1, 1024, smem, st, idx, c->T * c->k, c->E, capacity_rows(c), counts, offsets,
                                   perm, slot, dropped, err);
  return check_launch();
}

template <bool DOWN, int VEC>
moe_status launch_simt(const SimtArgs& a, int grid, cudaStream_t st) {
  const size_t red = (size_t)(DOWN ? 1 : 2) * kSimtWarps * kSimtRB * 32 * VEC * 4;
  const size_t stage = (size_t)kSimtRB * kSimtKC * 4;
  const size_t smem = red > stage ? red : stage;
  if (cudaFuncSetAttribute(k_simt_ffn<DOWN, VEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  MOE_LAUNCH((k_simt_ffn<DOWN, VEC>), grid, 256, smem, st, a);
  return check_launch();
}

// Routed rows of the expert GEMMs: slot s (< offsets[E]) gathers token
// src[s] / src_k of xn, and the down GEMM stores its row, scaled by gate[dst[s]],
// as row dst[s] of y.  Top-k: src = dst = perm_assign, src_k = k.  Expert choice:
// src = the picked tokens (src_k = 1), dst = the identity.
struct RoutedRows {
  const int32_t* src;
  int src_k;
  const int32_t* dst;
  const int32_t* slot_of = nullptr;   // [T, k] slot of each assignment (-1: dropped), if known
};

// Parameters of the grouped gate/up GEMM: the routed problem (rows gathered by the
// GEMM from xn through rr.src, or read from the gathered rows xp) and the shared
// experts' problem (every token of xn).
moe_status gateup_params(const moe_config* c, const moe_weights* w, const moe_weights& wl, int wq,
                         const void* xn, const void* xp, const int32_t* offsets, RoutedRows rr,
                         __nv_bfloat16* h, float* split_part, int32_t* split_cnt, int32_t* err,
                         TcParams& p) {
  const int T = c->T, S = c->n_shared, bn = tile_bn(c), R = (int)n_slots(c);
  const bool g4 = gather_in_gemm(c);
  p = TcParams{};
  TcProblem& P = p.prob[0];
  if (!map_expert(&P.tmA, wq, wl.w_gate, c->E, c->d, c->f)) return MOE_ERR_CUDA;
  if (!map_expert(&P.tmA2, wq, wl.w_up, c->E, c->d, c->f)) return MOE_ERR_CUDA;
  if (g4) {
    // routed rows: slot s reads token perm[s] / k of xn, four rows per copy
    if (!map_rows(&P.tmB, xn, T, c->d, 1)) return MOE_ERR_CUDA;
    P.gather_rows = rr.src;
    P.gather_k = rr.src_k;
  } else if (!map_rows(&P.tmB, xp, R, c->d, bn)) {
    return MOE_ERR_CUDA;
  }
  // bf16 direct tiles: 64-row copies for the tiles of at most 64 rows
  const bool m64_maps = bn == 128 && !g4 && wq == WQ_BF16;
  if (m64_maps && !map_rows(&P.tmB64, xp, R, c->d, 64)) return MOE_ERR_CUDA;
  if (wq != WQ_BF16 && (!map_scales(&P.tmS, c, w->s_gate, c->E, c->d, c->f) ||
                        !map_scales(&P.tmS2, c, w->s_up, c->E, c->d, c->f)))
    return MOE_ERR_CUDA;
  P.offsets = offsets;
  P.G = c->E;
  P.N = c->f;
  P.K = c->d;
  P.out = h;
  P.out_row_base = 0;
  P.ld_out = c->f;
  P.n_valid = c->f;
  p.n_prob = 1;
  if (S > 0) {
    TcProblem& Q = p.prob[1];
    if (!map_expert(&Q.tmA, wq, wl.sh_gate, S, c->d, c->f)) return MOE_ERR_CUDA;
    if (!map_expert(&Q.tmA2, wq, wl.sh_up, S, c->d, c->f)) return MOE_ERR_CUDA;
    if (!map_rows(&Q.tmB, xn, T, c->d, bn)) return MOE_ERR_CUDA;
    if (m64_maps && !map_rows(&Q.tmB64, xn, T, c->d, 64)) return MOE_ERR_CUDA;
    if (wq != WQ_BF16 && (!map_scales(&Q.tmS, c, w->sh_s_gate, S, c->d, c->f) ||
                          !map_scales(&Q.tmS2, c, w->sh_s_up, S, c->d, c->f)))
      return MOE_ERR_CUDA;
    Q.offsets = nullptr;
    Q.G = S;
    Q.uniform_rows = T;
    Q.b_row_base = 0;
    Q.b_group_stride = 0;
    Q.N = c->f;
    Q.K = c->d;
    Q.out = h;
    Q.out_row_base = (size_t)R;
    Q.ld_out = c->f;
    Q.n_valid = c->f;
    p.n_prob = 2;
  }
  p.err = err;
  p.wait_cycles = wait_cycles(c);
  p.split_part = split_part;
  p.split_cnt = split_cnt;
  p.interleave = interleave_tiles(c);
  return MOE_OK;
}

// Parameters of the grouped down GEMM: routed rows of h to rows rr.dst of y scaled
// by their gate, and the shared experts' rows of h to ys.
moe_status down_params(const moe_config* c, const moe_weights* w, const moe_weights& wl, int wq,
                       const int32_t* offsets, RoutedRows rr, const float* gate,
                       const __nv_bfloat16* h, void* y, bool rows_bf16, float* ys,
                       float* split_part, int32_t* split_cnt, int32_t* err, TcParams& p) {
  const int T = c->T, S = c->n_shared, bn = tile_bn(c), R = (int)n_slots(c);
  const int32_t* perm = rr.dst;
  p = TcParams{};
  TcProblem& P = p.prob[0];
  if (!map_expert(&P.tmA, wq, wl.w_down, c->E, c->f, c->d)) return MOE_ERR_CUDA;
  P.tmA2 = P.tmA;
  if (wq != WQ_BF16) {
    if (!map_scales(&P.tmS, c, w->s_down, c->E, c->f, c->d)) return MOE_ERR_CUDA;
    P.tmS2 = P.tmS;
  }
  if (!map_rows(&P.tmB, h, R + S * T, c->f, bn)) return MOE_ERR_CUDA;
  if (bn == 128 && wq == WQ_BF16 && !map_rows(&P.tmB64, h, R + S * T, c->f, 64))
    return MOE_ERR_CUDA;
  P.offsets = offsets;
  P.G = c->E;
  P.N = c->d;
  P.K = c->f;
  P.out = y;
  P.out_bf16 = rows_bf16 ? 1 : 0;
  P.out_row_base = 0;
  P.ld_out = c->d;
  P.perm_assign = perm;
  P.gate = gate;
  P.n_valid = c->d;
  p.n_prob = 1;
  if (S > 0) {
    TcProblem& Q = p.prob[1];
    if (!map_expert(&Q.tmA, wq, wl.sh_down, S, c->f, c->d)) return MOE_ERR_CUDA;
    Q.tmA2 = Q.tmA;
    if (wq != WQ_BF16) {
      if (!map_scales(&Q.tmS, c, w->sh_s_down, S, c->f, c->d)) return MOE_ERR_CUDA;
      Q.tmS2 = Q.tmS;
    }
    Q.tmB = P.tmB;
    Q.tmB64 = P.tmB64;
    Q.offsets = nullptr;
    Q.G = S;
    Q.uniform_rows = T;
    Q.b_row_base = R;
    Q.b_group_stride = T;
    Q.N = c->d;
    Q.K = c->f;
    Q.out = ys;
    Q.out_row_base = 0;
    Q.ld_out = c->d;
    Q.perm_assign = nullptr;
    Q.gate = nullptr;
    Q.n_valid = c->d;
    p.n_prob = 2;
  }
  p.err = err;
  p.wait_cycles = wait_cycles(c);
  p.split_part = split_part;
  p.split_cnt = split_cnt;
  p.interleave = interleave_tiles(c);
  return MOE_OK;
}

moe_status run_ffn(const moe_config* c, const moe_weights* w, const void* xn,
                   const int32_t* offsets, RoutedRows rr, const float* gate, void* y,
                   float* ys, void* ws, cudaStream_t st, Marks* mk = nullptr,
                   bool counters_zeroed = false, bool rows_bf16 = false) {
  Marks none;
  if (!mk) mk = &none;
  const Layout L = layout(c);
  int32_t* err = at<int32_t>(ws, L.err);
  const int T = c->T, k = c->k, S = c->n_shared;
  const int32_t* perm = rr.dst;
  if (!w->w_gate || !w->w_up || !w->w_down) return MOE_ERR_INVALID;
  if (S > 0 && (!w->sh_gate || !w->sh_up || !w->sh_down || !ys)) return MOE_ERR_INVALID;
  if (quantised(c)) {
    if (!w->s_gate || !w->s_up || !w->s_down) return MOE_ERR_INVALID;
    if (S > 0 && (!w->sh_s_gate || !w->sh_s_up || !w->sh_s_down)) return MOE_ERR_INVALID;
  }
  if (!tc_experts(c)) {
    SimtArgs a{};
    a.xn = static_cast<const float*>(xn);
    a.offsets = offsets;
    a.perm_assign = perm;
    a.gate = gate;
    a.wg = static_cast<const float*>(w->w_gate);
    a.wu = static_cast<const float*>(w->w_up);
    a.wd = static_cast<const float*>(w->w_down);
    a.swg = static_cast<const float*>(w->sh_gate);
    a.swu = static_cast<const float*>(w->sh_up);
    a.swd = static_cast<const float*>(w->sh_down);
    a.h = at<float>(ws, L.h);
    a.y = static_cast<float*>(y);
    a.ys = ys;
    a.T = T; a.d = c->d; a.f = c->f; a.k = k; a.E = c->E; a.S = S;
    // float4 columns where the rows and every matrix base allow 16-byte vectors
    auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    const bool v4_gu = c->f % 4 == 0 && a16(a.wg) && a16(a.wu) && a16(a.h) &&
                       (S == 0 || (a16(a.swg) && a16(a.swu)));
    const bool v4_dn = c->d % 4 == 0 && a16(a.wd) && a16(a.y) && (S == 0 || (a16(a.swd) && a16(a.ys)));
    const int grid = 2 * num_sms();
    moe_status s = v4_gu ? launch_simt<false, 4>(a, grid, st) : launch_simt<false, 1>(a, grid, st);
    if (s != MOE_OK) return s;
    mk->mark(st);
    s = v4_dn ? launch_simt<true, 4>(a, grid, st) : launch_simt<true, 1>(a, grid, st);
    mk->mark(st);
    return s;
  }
  // tensor-core experts: [gather the routed rows into xp], then gate/up and down on
  // the tensor cores (quantised weights are expanded inside their main loop).  The TMA (and the vector loads of the
  // gather and dequantisation kernels) need 16-byte aligned operands.
  {
    auto a16 = [](const void* q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    const void* ops[] = {xn, w->w_gate, w->w_up, w->w_down, w->s_gate, w->s_up, w->s_down,
                         w->sh_gate, w->sh_up, w->sh_down, w->sh_s_gate, w->sh_s_up,
                         w->sh_s_down};
    for (const void* o : ops)
      if (!a16(o)) return MOE_ERR_INVALID;
  }
  __nv_bfloat16* h = at<__nv_bfloat16>(ws, L.h);
  const int bn = tile_bn(c);
  const int R = (int)n_slots(c);
  const int wq = wq_of(c);
  const moe_weights& wl = *w;
  moe_status s = MOE_OK;
  const bool g4 = gather_in_gemm(c);
  float* split_part = split_k(c) ? at<float>(ws, L.split) : nullptr;
  int32_t* split_cnt = split_k(c) ? at<int32_t>(ws, L.splitcnt) : nullptr;
  // prefill tiles take their tiles in index order from a counter (the tiles that
  // share an expert's weights stay close in time)
  int32_t* tile_ctr = bn == 128 ? at<int32_t>(ws, L.tilectr) : nullptr;
  // the split-K and dynamic tile counters (zeroed by the layer's RMSNorm otherwise)
  if (!counters_zeroed && (split_cnt || tile_ctr) &&
      cudaMemsetAsync(at<int32_t>(ws, L.splitcnt), 0, L.tilectr + 8 - L.splitcnt, st) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  __nv_bfloat16* xp = at<__nv_bfloat16>(ws, L.xp);
  if (!g4 && rr.slot_of && k <= 32) {
    // token by token (each row of xn read once); 64 warps per SM
    MOE_LAUNCH((k_gather_rows_by_token<__nv_bfloat16>), 8 * num_sms(), 256, 0, st,
               static_cast<const __nv_bfloat16*>(xn), rr.slot_of, T, k, c->d, xp);
    if ((s = check_launch()) != MOE_OK) return s;
  } else if (!g4) {
    // 64 warps per SM, so that many rows are in flight at once
    MOE_LAUNCH((k_gather_rows<__nv_bfloat16>), 8 * num_sms(), 256, 0, st,
               static_cast<const __nv_bfloat16*>(xn), rr.src, offsets + c->E, rr.src_k, c->d,
               xp);
    if ((s = check_launch()) != MOE_OK) return s;
  }
  mk->mark(st);   // end of the (optional) gather step
  {
    TcParams p;
    if ((s = gateup_params(c, w, wl, wq, xn, xp, offsets, rr, h, split_part, split_cnt, err, p)) !=
        MOE_OK)
      return s;
    p.tile_ctr = tile_ctr;
    s = launch_tc_bn<EPI_GATEUP>(bn, wq, pair_tiles(c), p, st);
    if (s != MOE_OK) return s;
    mk->mark(st);
  }
  {
    TcParams p;
    if ((s = down_params(c, w, wl, wq, offsets, rr, gate, h, y, rows_bf16, ys, split_part,
                         split_cnt, err, p)) != MOE_OK)
      return s;
    p.tile_ctr = tile_ctr ? tile_ctr + 1 : nullptr;
    s = launch_tc_bn<EPI_DOWN>(bn, wq, pair_tiles(c), p, st);
    mk->mark(st);
  }
  return s;
}

template <int VEC>
moe_status launch_combine(const moe_config* c, const void* y, bool rows_bf16,
                          const int32_t* slot, const float* ys, const void* res, void* out,
                          cudaStream_t st) {
  const size_t n = (size_t)c->T * (c->d / VEC);
  const int blocks = (int)((n + 255) / 256);
  using bf = __nv_bfloat16;
  auto yf = static_cast<const float*>(y);
  auto yb = static_cast<const bf*>(y);
  auto rb = static_cast<const bf*>(res);
  auto rf = static_cast<const float*>(res);
  if (c->act_dtype == MOE_BF16 && c->out_dtype == MOE_BF16) {
    if (rows_bf16)
      MOE_LAUNCH((k_combine<bf, bf, bf, VEC>), blocks, 256, 0, st, yb, slot, ys, c->n_shared, rb,
                 static_cast<bf*>(out), c->T, c->d, c->k);
    else
      MOE_LAUNCH((k_combine<bf, bf, float, VEC>), blocks, 256, 0, st, yf, slot, ys, c->n_shared,
                 rb, static_cast<bf*>(out), c->T, c->d, c->k);
  } else if (c->act_dtype == MOE_BF16) {
    if (rows_bf16)
      MOE_LAUNCH((k_combine<bf, float, bf, VEC>), blocks, 256, 0, st, yb, slot, ys, c->n_shared,
                 rb, static_cast<float*>(out), c->T, c->d, c->k);
    else
      MOE_LAUNCH((k_combine<bf, float, float, VEC>), blocks, 256, 0, st, yf, slot, ys,
                 c->n_shared, rb, static_cast<float*>(out), c->T, c->d, c->k);
  } else {
    if (rows_bf16) return MOE_ERR_UNSUPPORTED;
    MOE_LAUNCH((k_combine<float, float, float, VEC>), blocks, 256, 0, st, yf, slot, ys,
               c->n_shared, rf, static_cast<float*>(out), c->T, c->d, c->k);
  }
  return check_launch();
}

moe_status run_combine(const moe_config* c, const void* y, bool rows_bf16, const int32_t* slot,
                       const float* ys, const void* res, void* out, cudaStream_t st) {
  auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  // eight columns per thread (16-byte bf16 loads) where the rows allow it: measured
  // 0.78x the time of four on the V3-shaped T=9440 combine
  if (a16(y) && a16(ys) && a16(res) && a16(out))
    return c->d % 8 == 0 ? launch_combine<8>(c, y, rows_bf16, slot, ys, res, out, st)
                         : launch_combine<4>(c, y, rows_bf16, slot, ys, res, out, st);
  return launch_combine<1>(c, y, rows_bf16, slot, ys, res, out, st);
}

template <int VEC>
moe_status launch_combine_ec(const moe_config* c, const void* y, bool rows_bf16,
                             const int32_t* slot_te, const float* ys, const void* res, void* out,
                             cudaStream_t st) {
  using bf = __nv_bfloat16;
  auto rb = static_cast<const bf*>(res);
  const int T = c->T, E = c->E, S = c->n_shared, d = c->d;
  if (!rows_bf16) return MOE_ERR_UNSUPPORTED;   // tensor-core experts: bf16 rows
  auto yb = static_cast<const bf*>(y);
  if (c->out_dtype == MOE_BF16)
    MOE_LAUNCH((k_combine_ec<bf, bf, bf, VEC>), T, 256, 0, st, yb, slot_te, E, ys, S, rb,
               static_cast<bf*>(out), T, d);
  else
    MOE_LAUNCH((k_combine_ec<bf, float, bf, VEC>), T, 256, 0, st, yb, slot_te, E, ys, S, rb,
               static_cast<float*>(out), T, d);
  return check_launch();
}

moe_status run_combine_ec(const moe_config* c, const void* y, bool rows_bf16,
                          const int32_t* slot_te, const float* ys, const void* res, void* out,
                          cudaStream_t st) {
  auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  if (a16(y) && a16(ys) && a16(res) && a16(out))
    return c->d % 8 == 0 ? launch_combine_ec<8>(c, y, rows_bf16, slot_te, ys, res, out, st)
                         : launch_combine_ec<4>(c, y, rows_bf16, slot_te, ys, res, out, st);
  return launch_combine_ec<1>(c, y, rows_bf16, slot_te, ys, res, out, st);
}

// Expert-choice routing from router partials (ns K-slices): FP32 scores, then each
// expert's C picks.  tok / gate / yrow [E*C], offsets [E+1], counts [E], slot_te [T, E].
moe_status run_route_ec(const moe_config* c, const float* part, int ns, const float* bias,
                        float* scores_t, float* scores_out, float* logits_out, int32_t* tok,
                        float* gate, int32_t* yrow, int32_t* offsets, int32_t* counts,
                        int32_t* slot_te, cudaStream_t st, Marks* mk = nullptr) {
  const int mode = c->bias_mode;
  if (mode != MOE_BIAS_NONE && !bias) return MOE_ERR_INVALID;
  const int blocks = (c->T + 7) / 8;
#define MOE_EC_SCORES(EPL)                                                                 \
  MOE_LAUNCH((k_ec_scores<EPL>), blocks, 256, 0, st, part, ns, c->T, c->E, bias, mode,     \
             scores_t, scores_out, logits_out)
  if (c->E <= 32) MOE_EC_SCORES(1);
  else if (c->E <= 64) MOE_EC_SCORES(2);
  else if (c->E <= 128) MOE_EC_SCORES(4);
  else if (c->E <= 256) MOE_EC_SCORES(8);
  else MOE_EC_SCORES(16);
#undef MOE_EC_SCORES
  if (mk) mk->mark(st);   // end of the routing step (scores)
  MOE_LAUNCH((k_ec_select), c->E, 1024, 0, st, scores_t, c->T, c->E, ec_capacity(c), tok, gate,
             yrow, offsets, counts, slot_te);
  return check_launch();
}

// ------------------------------------------------------ single-launch decode layer
// Offset of the decode kernel's grid-barrier words in the workspace (inside the
// first 256 bytes, which moe_clear_device_status zeroes).
constexpr size_t kGridBarOff = 64;

// The whole layer in one cooperative launch: decode batches (T <= 32) of bf16
// experts with a bf16 router of at most 256 experts, 16-byte aligned tensors.
bool single_launch(const moe_config* c) {
  return !expert_choice(c) && c->T <= kDecodeMaxT && c->expert_dtype == MOE_BF16 &&
         vec_router(c) && c->E <= 256 && gather_in_gemm(c) && c->d <= 256 * 4 * 8;
}

template <int EPL, int BN>
moe_status launch_decode(const DecodeParams& dp, cudaStream_t st) {
  using CG = TcConfig<EPI_GATEUP, BN, false, WQ_BF16>;
  using CD = TcConfig<EPI_DOWN, BN, false, WQ_BF16>;
  constexpr uint32_t smem = CG::SMEM_BYTES > CD::SMEM_BYTES ? CG::SMEM_BYTES : CD::SMEM_BYTES;
  auto kern = k_decode_layer<EPL, BN, 4>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  // every CTA must be resident at once (the grid barriers): one per SM
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecodeThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return MOE_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute a[1];
  a[0].id = cudaLaunchAttributeCooperative;
  a[0].val.cooperative = 1;
  cfg.attrs = a;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, dp) != cudaSuccess) return MOE_ERR_CUDA;
  return check_launch();
}

moe_status run_decode_layer(const moe_config* c, const moe_weights* w, const void* x, void* out,
                            void* ws, float* logits_out, int32_t* idx, int32_t* counts,
                            cudaStream_t st) {
  const Layout L = layout(c);
  DecodeParams dp{};
  int32_t* err = at<int32_t>(ws, L.err);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  float* gate = at<float>(ws, L.gate);
  __nv_bfloat16* h = at<__nv_bfloat16>(ws, L.h);
  void* xn = at<void>(ws, L.xn);
  void* y = at<void>(ws, L.y);
  float* ys = c->n_shared ? at<float>(ws, L.ys) : nullptr;
  const RoutedRows rr{perm, c->k, perm};
  float* split_part = split_k(c) ? at<float>(ws, L.split) : nullptr;
  int32_t* split_cnt = split_k(c) ? at<int32_t>(ws, L.splitcnt) : nullptr;
  moe_status s;
  if ((s = gateup_params(c, w, *w, WQ_BF16, xn, nullptr, offsets, rr, h, split_part, split_cnt,
                         err, dp.gu)) != MOE_OK)
    return s;
  if ((s = down_params(c, w, *w, WQ_BF16, offsets, rr, gate, h, y, true, ys, split_part,
                       split_cnt, err, dp.dn)) != MOE_OK)
    return s;
  dp.n_split_cnt = split_cnt ? split_counters() : 0;
  dp.x = static_cast<const __nv_bfloat16*>(x);
  dp.gamma = static_cast<const float*>(w->rms_gamma);
  dp.w_router = static_cast<const __nv_bfloat16*>(w->w_router);
  dp.bias = static_cast<const float*>(w->router_bias);
  dp.xn = static_cast<__nv_bfloat16*>(xn);
  dp.part = at<float>(ws, L.part);
  dp.idx = idx;
  dp.gate = gate;
  dp.counts = counts;
  dp.offsets = offsets;
  dp.perm = perm;
  dp.slot = at<int32_t>(ws, L.slot);
  dp.dropped = at<int32_t>(ws, L.dropped);
  dp.logits_out = logits_out;
  dp.w_down = static_cast<const uint8_t*>(w->w_down);
  dp.sh_down = static_cast<const uint8_t*>(w->sh_down);
  dp.y = static_cast<const __nv_bfloat16*>(y);
  dp.ys = ys;
  dp.out = out;
  dp.out_f32 = c->out_dtype == MOE_F32 ? 1 : 0;
  dp.err = err;
  dp.grid_bar = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + kGridBarOff);
  dp.wait_cycles = wait_cycles(c);
  dp.eps = (double)c->rms_eps;
  dp.T = c->T;
  dp.d = c->d;
  dp.E = c->E;
  dp.k = c->k;
  dp.S = c->n_shared;
  dp.mode = c->bias_mode;
  dp.renorm = c->renormalize ? 1 : 0;
  dp.cap = capacity_rows(c);
  dp.ns = L.ns;
  dp.rows = kRouterSlice;
  dp.route_all = (long long)c->T * L.ns * c->E <= 32768 ? 1 : 0;
  const int bn = pick_bn(c);
#define MOE_DECODE(EPL)                                                        \
  return bn == 16 ? launch_decode<EPL, 16>(dp, st) : launch_decode<EPL, 32>(dp, st)
  if (c->E <= 32) MOE_DECODE(1);
  if (c->E <= 64) MOE_DECODE(2);
  if (c->E <= 128) MOE_DECODE(4);
  MOE_DECODE(8);
#undef MOE_DECODE
}

moe_status layer_forward_impl(const moe_config* cfg, const moe_weights* w, const void* x,
                              void* out, void* ws, size_t ws_bytes, float* logits_out,
                              int32_t* topk_idx_out, int32_t* counts_out, cudaStream_t st,
                              Marks* mk) {
  moe_status s = validate(cfg);
  if (s != MOE_OK) return s;
  if (!w || !x || !out || !w->rms_gamma || !w->w_router) return MOE_ERR_INVALID;
  if (cfg->bias_mode != MOE_BIAS_NONE && !w->router_bias) return MOE_ERR_INVALID;
  if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
  const Layout L = layout(cfg);
  int32_t* err = at<int32_t>(ws, L.err);
  void* xn = at<void>(ws, L.xn);
  float* part = at<float>(ws, L.part);
  int32_t* idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.idx);
  float* gate = at<float>(ws, L.gate);
  int32_t* counts = counts_out ? counts_out : at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* slot = at<int32_t>(ws, L.slot);
  void* y = at<void>(ws, L.y);
  float* ys = cfg->n_shared ? at<float>(ws, L.ys) : nullptr;
  if (!mk->ev && single_launch(cfg)) {
    auto a16 = [](const void* q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    const void* ops[] = {x, out, w->rms_gamma, w->w_router, w->w_gate, w->w_up, w->w_down,
                         w->sh_gate, w->sh_up, w->sh_down};
    bool aligned = true;
    for (const void* o : ops) aligned = aligned && a16(o);
    if (aligned) return run_decode_layer(cfg, w, x, out, ws, logits_out, idx, counts, st);
  }
  mk->mark(st);
  // the expert GEMMs' split-K and dynamic tile counters, zeroed by the RMSNorm
  if ((s = run_rmsnorm(cfg, w, x, xn, st, at<int32_t>(ws, L.splitcnt),
                       (int)((L.tilectr + 8 - L.splitcnt) / 4))) != MOE_OK)
    return s;
  mk->mark(st);
  if ((s = run_router(cfg, w, xn, part, L.ns, err, st)) != MOE_OK) return s;
  mk->mark(st);
  if (expert_choice(cfg)) {
    // scores (the routing step), the experts' picks (the permutation step), the
    // expert GEMMs over the E*C picks, and the per-token combine
    if (topk_idx_out) return MOE_ERR_INVALID;
    int32_t* tok = at<int32_t>(ws, L.idx);
    int32_t* yrow = at<int32_t>(ws, L.perm);
    int32_t* slot_te = at<int32_t>(ws, L.slot);
    if ((s = run_route_ec(cfg, part, L.ns, static_cast<const float*>(w->router_bias),
                          at<float>(ws, L.sct), nullptr, logits_out, tok, gate, yrow, offsets,
                          counts, slot_te, st, mk)) != MOE_OK)
      return s;
    mk->mark(st);
    if ((s = run_ffn(cfg, w, xn, offsets, RoutedRows{tok, 1, yrow}, gate, y, ys, ws, st, mk,
                     true, y_bf16(cfg))) != MOE_OK)
      return s;
    s = run_combine_ec(cfg, y, y_bf16(cfg), slot_te, ys, x, out, st);
    mk->mark(st);
    return s;
  }
  if (fused_route_permute(cfg)) {
    // one launch; the permutation step has no time of its own in the profile
    if ((s = run_route_permute(cfg, part, L.ns, static_cast<const float*>(w->router_bias), idx,
                               gate, logits_out, counts, offsets, perm, slot,
                               at<int32_t>(ws, L.dropped), err, st)) != MOE_OK)
      return s;
    mk->mark(st);
  } else {
    if ((s = run_route(cfg, part, L.ns, static_cast<const float*>(w->router_bias), idx, gate,
                       logits_out, st)) != MOE_OK)
      return s;
    mk->mark(st);
    if ((s = run_permute(cfg, idx, counts, offsets, perm, slot, at<int32_t>(ws, L.dropped), err,
                         at<int32_t>(ws, L.blk), st)) != MOE_OK)
      return s;
  }
  mk->mark(st);
  if ((s = run_ffn(cfg, w, xn, offsets, RoutedRows{perm, cfg->k, perm, slot}, gate, y, ys, ws,
                   st, mk, true, y_bf16(cfg))) != MOE_OK)
    return s;
  s = run_combine(cfg, y, y_bf16(cfg), slot, ys, x, out, st);
  mk->mark(st);
  return s;
}

// ------------------------------------------------ allocation-free permutation
// Scratch of moe_permute_static: the per-CTA expert counts of the multi-CTA
// permutation live in this file-scope device array instead of a caller
// workspace.  Every GPU that loads the library holds it until the process ends.
constexpr size_t kStaticPermInts = size_t(1) << 18;           // 1 MiB of int32
static __device__ __align__(256) int32_t g_perm_counts[kStaticPermInts];

// Device address of g_perm_counts on the current device, looked up once per
// device (host code may not use the symbol's name as a device pointer).
int32_t* static_perm_counts() {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static int32_t* ptr[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_perm_counts) != cudaSuccess) return nullptr;
    ptr[dev] = static_cast<int32_t*>(p);
  }
  return ptr[dev];
}

// =================================================================== C ABI
}  // namespace

extern "C" {

size_t moe_workspace_size(const moe_config* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return layout(cfg).total;
}

moe_status moe_clear_device_status(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 16) return MOE_ERR_WORKSPACE;
  // the error word, and the single-launch decode layer's grid-barrier words
  const size_t n = ws_bytes < 256 ? 16 : 256;
  return cudaMemsetAsync(ws, 0, n, S_(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_rmsnorm_router(const moe_config* cfg, const moe_weights* w, const void* x,
                              void* xn_out, float* logits, void* ws, size_t ws_bytes,
                              void* stream) {
  moe_status s = validate(cfg);
  if (s != MOE_OK) return s;
  if (!w || !x || !logits || !w->rms_gamma || !w->w_router) return MOE_ERR_INVALID;
  if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
  const Layout L = layout(cfg);
  cudaStream_t st = S_(stream);
  void* xn = xn_out ? xn_out : at<void>(ws, L.xn);
  if ((s = run_rmsnorm(cfg, w, x, xn, st)) != MOE_OK) return s;
  float* part = at<float>(ws, L.part);
  if ((s = run_router(cfg, w, xn, part, L.ns, at<int32_t>(ws, L.err), st)) != MOE_OK) return s;
  // add the K slices in order into logits (the route kernel's reduction, no selection)
  if (L.ns == 1 && tc_router(cfg))
    return cudaMemcpyAsync(logits, part, (size_t)cfg->T * cfg->E * 4, cudaMemcpyDeviceToDevice,
                           st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  moe_config c1 = *cfg;
  c1.bias_mode = MOE_BIAS_NONE;
  return run_route(&c1, part, L.ns, nullptr, at<int32_t>(ws, L.idx), at<float>(ws, L.gate),
                   logits, st);
}

moe_status moe_route(const moe_config* cfg, const float* logits, const float* bias,
                     int32_t* topk_idx, float* topk_gate, void* stream) {
  moe_status s = validate(cfg);
  if (s != MOE_OK) return s;
  if (!logits || !topk_idx || !topk_gate) return MOE_ERR_INVALID;
  if (expert_choice(cfg)) return MOE_ERR_INVALID;   // moe_route_expert_choice
  return run_route(cfg, logits, 1, bias, topk_idx, topk_gate, nullptr, S_(stream));
}

int32_t moe_expert_choice_capacity(const moe_config* cfg) {
  if (validate(cfg) != MOE_OK || !expert_choice(cfg)) return 0;
  return ec_capacity(cfg);
}

moe_status moe_route_expert_choice(const moe_config* cfg, const float* logits, const float* bias,
                                   float* scores_out, int32_t* tok, float* gate,
                                   int32_t* slot_te, void* ws, size_t ws_bytes, void* stream) {
  moe_status s = validate(cfg);
  if (s != MOE_OK) return s;
  if (!expert_choice(cfg)) return MOE_ERR_INVALID;
  if (!logits || !tok || !gate || !slot_te) return MOE_ERR_INVALID;
  if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
  const Layout L = layout(cfg);
  return run_route_ec(cfg, logits, 1, bias, at<float>(ws, L.sct), scores_out, nullptr, tok, gate,
                      at<int32_t>(ws, L.perm), at<int32_t>(ws, L.offsets),
                      at<int32_t>(ws, L.counts), slot_te, S_(stream));
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, int32_t* counts,
                       int32_t* offsets, int32_t* perm_assign, int32_t* slot_of,
                       int32_t* n_dropped, void* ws, size_t ws_bytes, void* stream) {
  moe_status s = validate(cfg);
  if (s != MOE_OK) return s;
  if (!topk_idx || !counts || !offsets || !perm_assign || !slot_of || !n_dropped)
    return MOE_ERR_INVALID;
  if (!ws || ws_bytes < 16 || reinterpret_cast<uintptr_t>(ws) % kAlign) return MOE_ERR_WORKSPACE;
  // the multi-CTA path keeps per-CTA counts in the workspace when it is large enough
  int32_t* blk = ws_bytes >= layout(cfg).total ? at<int32_t>(ws, layout(cfg).blk) : nullptr;
  return run_permute(cfg, topk_idx, counts, offsets, perm_assign, slot_of, n_dropped,
                     static_cast<int32_t*>(ws), blk, S_(stream));
}

moe_status moe_permute_static(const moe_config* cfg, const int32_t* topk_idx, int32_t* counts,
                              int32_t* offsets, int32_t* perm_assign, int32_t* slot_of,
                              int32_t* n_dropped, void* stream) {
  moe_status s = validate(cfg);
  if (s != MOE_OK) return s;
  if (!topk_idx || !counts || !offsets || !perm_assign || !slot_of || !n_dropped)
    return MOE_ERR_INVALID;
  const int n = cfg->T * cfg->k;
  const size_t need = (size_t)cfg->E * ((n + kPermChunk - 1) / kPermChunk);
  if (need > kStaticPermInts) return MOE_ERR_WORKSPACE;
  int32_t* blk = static_perm_counts();
  if (!blk) return MOE_ERR_CUDA;
  cudaStream_t st = S_(stream);
  const int E = cfg->E, cap = capacity_rows(cfg);
  if (n <= kPermSingleMax) {
    const size_t smem = (size_t)33 * E * 4;
    if (cudaFuncSetAttribute(k_permute, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    MOE_LAUNCH((k_permute), 1, 1024, smem, st, topk_idx, n, E, cap, counts, offsets, perm_assign, slot_of,
                                     n_dropped, nullptr);
    return check_launch();
  }
  // every entry of blk that the scan reads is written by the count kernel first
  const int nb = (n + kPermChunk - 1) / kPermChunk;
  const size_t sm1 = (size_t)kPermWarps * E * 4;
  const size_t sm3 = sm1 + (size_t)E * 4;
  if (cudaFuncSetAttribute(k_perm_rank, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  MOE_LAUNCH((k_perm_count), nb, 256, sm1, st, topk_idx, n, E, nb, blk, nullptr);
  MOE_LAUNCH((k_perm_scan), 1, 1024, 0, st, blk, nb, E, cap, counts, offsets, n_dropped);
  MOE_LAUNCH((k_perm_rank), nb, 256, sm3, st, topk_idx, n, E, nb, cap, blk, offsets, perm_assign, slot_of);
  return check_launch();
}

moe_status moe_grouped_ffn(const moe_config* cfg, const moe_weights* w, const void* xn,
                           const int32_t* offsets, const int32_t* perm_assign,
                           const float* topk_gate, float* y_assign, float* y_shared, void* ws,
                           size_t ws_bytes, void* stream) {
  moe_status s = validate(cfg);
  if (s != MOE_OK) return s;
  if (!w || !xn || !offsets || !perm_assign || !topk_gate || !y_assign) return MOE_ERR_INVALID;
  if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
  if (expert_choice(cfg)) return MOE_ERR_UNSUPPORTED;   // the layer forward only
  return run_ffn(cfg, w, xn, offsets, RoutedRows{perm_assign, cfg->k, perm_assign}, topk_gate,
                 y_assign, y_shared, ws, S_(stream));
}

moe_status moe_combine(const moe_config* cfg, const float* y_assign, const int32_t* slot_of,
                       const float* y_shared, const void* residual, void* out, void* stream) {
  moe_status s = validate(cfg);
  if (s != MOE_OK) return s;
  if (!y_assign || !slot_of || !out || (cfg->n_shared > 0 && !y_shared)) return MOE_ERR_INVALID;
  return run_combine(cfg, y_assign, false, slot_of, y_shared, residual, out, S_(stream));
}

moe_status moe_layer_forward(const moe_config* cfg, const moe_weights* w, const void* x,
                             void* out, void* ws, size_t ws_bytes, float* logits_out,
                             int32_t* topk_idx_out, int32_t* counts_out, void* stream) {
  Marks none;
  return layer_forward_impl(cfg, w, x, out, ws, ws_bytes, logits_out, topk_idx_out, counts_out,
                            S_(stream), &none);
}

moe_status moe_layer_forward_profiled(const moe_config* cfg, const moe_weights* w,
                                      const void* x, void* out, void* ws, size_t ws_bytes,
                                      void* const* events, int32_t n_events, void* stream) {
  if (!events || n_events < moe_layer_step_count(cfg) + 1) return MOE_ERR_INVALID;
  Marks mk;
  mk.ev = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events));
  mk.n = n_events;
  return layer_forward_impl(cfg, w, x, out, ws, ws_bytes, nullptr, nullptr, nullptr, S_(stream),
                            &mk);
}

moe_status moe_get_device_status(const void* ws, int32_t* code, void* stream) {
  if (!ws || !code) return MOE_ERR_INVALID;
  if (cudaStreamSynchronize(S_(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  *code = v;
  return v ? MOE_ERR_DEVICE : MOE_OK;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID: return "MOE_ERR_INVALID";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
  }
  return "MOE_ERR_UNKNOWN";
}

int32_t moe_layer_step_count(const moe_config* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  // expert choice: rmsnorm, router, scores, picks, [gather], gate/up, down, combine
  // rmsnorm, router, route, permute, [dequantise + gather], gate/up, down, combine
  return tc_experts(cfg) ? 8 : 7;
}

int32_t moe_layer_launch_count(const moe_config* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  if (single_launch(cfg)) return 1;   // with 16-byte aligned tensors
  // rmsnorm, router, route, gate/up, down and combine, plus the permutation (its
  // own launch, three for large batches, or none when it shares the routing
  // launch), and for tensor-core experts at wide tiles the row gather
  const int gather = tc_experts(cfg) && !gather_in_gemm(cfg) ? 1 : 0;
  if (expert_choice(cfg))   // rmsnorm, router, scores, picks, gate/up, down, combine
    return 7 + gather;
  const int perm = fused_route_permute(cfg) ? 0 : cfg->T * cfg->k > kPermSingleMax ? 3 : 1;
  return 6 + perm + gather;
}

}  // extern "C"
