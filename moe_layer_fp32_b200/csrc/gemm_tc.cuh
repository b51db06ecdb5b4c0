// Grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM, TMA-fed) for the
// expert FFN (a6, a7) and the router at large batches (a2).
//
// "MoE: dynamism the compiler cannot remove", grouped GEMM section: one launch
// over a grid sized for the total work, each block finding its group (expert)
// from a small descriptor array -- here the per-expert offsets written by the
// permutation, turned into a tile prefix inside every CTA, so the grid never
// depends on the routing and no host synchronisation is needed.
//
// Shared-memory tiles, per pipeline stage:
//   weight tile: 128 output features x 64 k, loaded from W[G][K][N] (features
//       contiguous, MN-major) as two 64-feature TMA boxes, 128-byte swizzle;
//   token tile: BN rows x 64 k, loaded from X[R][K] (K-major), 128-byte
//       swizzle.  Rows past the end of an expert's segment belong to the next
//       segment or fall outside the tensor (zero fill); their accumulator
//       entries are simply not stored.
// Two orientations of the same tiles:
//   swapped (decode tiles, BN = 16..64 tokens): weights on the MMA's M side and
//       tokens on N, C^T[n, m] = sum_k W[k, n] X[m, k]; TMEM lane = feature, so
//       a narrow token tile costs no wasted MMA rows;
//   direct (prefill tiles, 128 tokens): tokens on M and weights on N; TMEM lane
//       = token, so each epilogue thread owns one output row and writes it with
//       16-byte stores, and looks up its row and gate once per tile.
// Accumulators live in TMEM, double buffered so that the epilogue of one tile
// overlaps the main loop of the next.
//
// Warp roles (320 threads): warp 0 lane 0 issues TMA; warp 1 allocates TMEM and
// its lane 0 issues tcgen05.mma; warps 2..9 drain TMEM (warp w reads lanes
// 32*(w%4) .. +31; warps w and w+4 split the columns) and run the epilogue.
//
// Epilogues:
//   GATEUP  two accumulators (gate, up); h = silu(gate) * up -> bf16 H row.
//   DOWN    y * gate(assignment) -> fp32 row perm_assign[slot] of Y (un-permuted),
//           or the shared expert's row of Ys (gate 1).
//   ROUTER  fp32 logits[t][e] for e < n_valid.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "kernels_small.cuh"

namespace moe {

enum Epi : int { EPI_GATEUP = 0, EPI_DOWN = 1, EPI_ROUTER = 2 };
// weight storage: bf16, or weight-only int8 / int4 / fp8 (E4M3) dequantised to
// bf16(q * s) in the main loop; int8 and fp8 share one layout (a byte per weight,
// a bf16 scale per output column)
enum WQuant : int { WQ_BF16 = 0, WQ_INT8 = 1, WQ_INT4 = 2, WQ_FP8 = 3 };
template <int WQ>
struct ByteWeights { static constexpr bool value = WQ == WQ_INT8 || WQ == WQ_FP8; };

constexpr int kTcBaseThreads = 320;   // producer, MMA, 8 epilogue warps
constexpr int kEpiWarps = 8;
constexpr int kMaxGroups = 512;

struct TcProblem {
  CUtensorMap tmA;            // weights [G][K][N] bf16 (dims n, k, g), box (64, 64, 1)
  CUtensorMap tmA2;           // second weight matrix (up) for GATEUP
  CUtensorMap tmB;            // activations [R][K] bf16 (dims k, r), box (64, BN); with
                              // gather_rows: box (64, 1), rows fetched four at a time
  CUtensorMap tmB64;          // bf16 direct tiles: the same rows, box (64, 64), for tiles
                              // of at most 64 rows
  const int32_t* offsets;     // [G+1] segments (B rows and output rows), or nullptr
  int G;                      // groups
  int uniform_rows;           // rows per group when offsets == nullptr
  int b_row_base;             // when offsets == nullptr: B row of group g's row 0 is
  int b_group_stride;         //   b_row_base + g * b_group_stride
  int N;                      // output features
  int K;                      // reduction length (multiple of 64)
  void* out;                  // H (bf16) / Y / Ys / logits (fp32; Y bf16 with out_bf16)
  int out_bf16;               // DOWN: store the gated rows in bf16
  size_t out_row_base;        // GATEUP / shared DOWN / ROUTER: row = base + seg + m
  int ld_out;                 // elements per output row
  const int32_t* gather_rows; // routed GATEUP: B row of slot s = gather_rows[s] / gather_k
  int gather_k;               //   (the token of the slot's assignment), or nullptr
  const int32_t* perm_assign; // routed DOWN: output row = perm_assign[slot]
  const float* gate;          // routed DOWN: scale
  int n_valid;                // features actually stored (n < n_valid)
  // int8 / int4 weights: tmA / tmA2 then map the raw bytes (uint8, no swizzle)
  // and tmS / tmS2 their bf16 scales, [G][N] (int8) or [G][K/128][N] (int4), box
  // 128 features
  CUtensorMap tmS;
  CUtensorMap tmS2;
};

struct TcParams {
  TcProblem prob[2];
  int n_prob;
  int32_t* err;
  long long wait_cycles;      // limit of every pipeline wait (clock cycles)
  // Split-K for swapped tiles (nullptr: off).  When the output tiles fill at most
  // half of the grid, each is split along K into S <= kMaxSplit parts.  Each part
  // stores its FP32 accumulators to split_part, and the last part of an output tile
  // to finish adds all S parts in split order and runs the epilogue.
  // split_part: gridDim.x * NA * BN * 128 floats.  split_cnt: gridDim.x * 8 zeroed
  // ints, left zeroed again.
  float* split_part;
  int32_t* split_cnt;
  // ROUTER: K is split into k_splits parts (>= 1); part s writes its partial logits
  // at out + s * split_out_stride (the routing kernel adds the parts in order)
  int k_splits;
  size_t split_out_stride;
  // problem 0 (routed, with offsets): interleave the tiles of light experts (one
  // token tile) evenly between the token tiles of the heavy ones, so that tiles
  // bound by streaming a light expert's weights run beside tiles bound by the
  // tensor cores instead of all at once
  int interleave;
  // Dynamic tile order (nullptr: static, tiles cta, cta + ncta, ...): each CTA takes
  // its first tile statically and every further one from this counter (zero when
  // the launch starts), so that tiles run in index order whatever their costs and no
  // CTA is left with a run of expensive tiles at the end of the launch
  int32_t* tile_ctr;
};

constexpr int kMaxSplit = 4;

struct TileInfo {
  int prob, g, m0, rows, n0;
  int b_row;          // B row of the tile's first token
  size_t out_seg;     // output row of the tile's first token (non-routed-DOWN cases)
  int slot0;          // routed: slot of the tile's first token
  int bt, ks;         // split-K: output tile and this work item's part of K
  int kb0, kb1;       // k-blocks [kb0, kb1) of this work item
  int whole;          // the tile holds all of its group's rows (its weights are read once)
};

// Weight blocks (128 features x 64 k) per pipeline stage: gate and up for
// GATEUP; for a direct DOWN tile, two neighbouring 128-feature blocks of W_down
// (a 256-wide tile); otherwise one.
template <int EPI, bool DIRECT>
struct TcShape {
  static constexpr int NA = (EPI == EPI_GATEUP) ? 2 : (EPI == EPI_DOWN && DIRECT) ? 2 : 1;
  static constexpr uint32_t A_BYTES = 128 * 64 * 2;
  static constexpr int TILE_N = (EPI == EPI_DOWN && DIRECT) ? 256 : 128;   // features per tile
};

template <int EPI, int BN, bool DIRECT, int WQ = WQ_BF16>
struct TcConfig {
  static constexpr int NA = TcShape<EPI, DIRECT>::NA;
  static constexpr int TILE_N = TcShape<EPI, DIRECT>::TILE_N;
  static constexpr uint32_t A_BYTES = TcShape<EPI, DIRECT>::A_BYTES;
  static constexpr uint32_t B_BYTES = BN * 64 * 2;
  // raw quantised weight block of 128 features x 64 k, stored K-contiguous: one row
  // of 64 codes per feature (int8 / fp8: 64 B, int4: 32 B)
  static constexpr uint32_t RAW_ROW = ByteWeights<WQ>::value ? 64 : WQ == WQ_INT4 ? 32 : 0;
  static constexpr uint32_t RAW_BYTES = 128 * RAW_ROW;
  static constexpr uint32_t SCALE_BYTES = WQ == WQ_BF16 ? 0 : 256;   // 128 bf16 scales
  // bf16 weights: one ring of TMA stages [weights NA x 16 KB | tokens].
  // int8 / int4 / fp8 weights: a deep ring of TMA stages [tokens | raw weights |
  // scales in a 1 KB slot] (so that enough weight bytes are in flight to cover
  // HBM latency); the dequantisation warps expand each block into a slot of bf16
  // weights: in TMEM for swapped tiles (the MMA's A operand), in shared memory for
  // direct tiles (the B operand, K-major, 128-byte swizzle, NA x 128 rows of 128 B
  // per slot).  Every stage is 1024-byte aligned.
  static constexpr uint32_t STAGE_BYTES =
      WQ == WQ_BF16 ? NA * A_BYTES + B_BYTES : B_BYTES + NA * RAW_BYTES + 1024;
  static constexpr uint32_t TOKEN_OFF = WQ == WQ_BF16 ? NA * A_BYTES : 0;
  static constexpr uint32_t RAW_OFF = B_BYTES;
  static constexpr uint32_t SCALE_OFF = B_BYTES + NA * RAW_BYTES;
  // bytes the TMA delivers per stage
  static constexpr uint32_t TX_BYTES =
      WQ == WQ_BF16 ? STAGE_BYTES : B_BYTES + NA * (RAW_BYTES + SCALE_BYTES);
  // one dequantisation thread per feature of each weight block (4 warps per block,
  // each warp on the TMEM lane quadrant its warp index allows); direct tiles, whose
  // expanded weights go to shared memory, two threads per feature (8 warps per
  // block), each for half of the k-block
  static constexpr int DEQ_WARPS = WQ == WQ_BF16 ? 0 : (DIRECT ? 8 : 4) * NA;
  static constexpr int THREADS = kTcBaseThreads + 32 * DEQ_WARPS;
  // direct tiles of quantised weights: two shared-memory slots of expanded weights
  static constexpr bool SMEM_W = DIRECT && WQ != WQ_BF16;
  static constexpr uint32_t W_SLOT_BYTES = SMEM_W ? NA * 128 * 128 : 0;
  static constexpr uint32_t A_REGION = 2 * W_SLOT_BYTES;
  static constexpr int STAGES_RAW = (200 * 1024 - A_REGION) / STAGE_BYTES;
  static constexpr int STAGE_CAP = WQ == WQ_BF16 ? 8 : 16;
  static constexpr int STAGES = STAGES_RAW > STAGE_CAP ? STAGE_CAP : STAGES_RAW;
  static constexpr uint32_t ACC_COLS = NA * BN;
  // TMEM: two accumulators, then (quantised weights) A_SLOTS slots of NA bf16
  // weight blocks, 128 lanes x 32 columns each (64 k, two per 32-bit column)
  static constexpr uint32_t A_COL0 = 2 * ACC_COLS;
  static constexpr uint32_t A_SLOT_COLS = (WQ == WQ_BF16 || SMEM_W) ? 0 : NA * 32;
  // as many weight slots as the TMEM left by the accumulators holds, at most 4, so
  // that the dequantisation warps run up to 4 k-blocks ahead of the MMA
  static constexpr int A_SLOTS_FIT =
      WQ == WQ_BF16 ? 2 : (int)((512 - 2 * ACC_COLS) / (A_SLOT_COLS ? A_SLOT_COLS : 1));
  static constexpr int A_SLOTS = (WQ == WQ_BF16 || SMEM_W) ? 2 : A_SLOTS_FIT > 4 ? 4 : A_SLOTS_FIT;
  static constexpr uint32_t TMEM_NEED = 2 * ACC_COLS + A_SLOTS * A_SLOT_COLS;
  static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                        : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
  // swapped: A = weights, M = 128 features, N = BN tokens (K-major), one MMA per
  //          weight block; bf16 weights come from shared memory (MN-major), the
  //          dequantised ones from TMEM (K-major);
  // direct:  A = tokens (K-major), B = all NA weight blocks at once (bf16: MN-major,
  //          the blocks 16 KB apart = two 64-feature boxes each at the 8 KB
  //          leading offset; expanded quantised weights: K-major, one 128-byte row
  //          per feature), M = 128 tokens, N = 128 * NA
  static constexpr uint32_t IDESC = DIRECT            ? idesc_bf16(128, 128 * NA, false, !SMEM_W)
                                    : WQ == WQ_BF16 ? idesc_bf16(128, BN, true, false)
                                                    : idesc_bf16(128, BN, false, false);
  // bf16 direct tiles of at most 64 rows: one M = 64 MMA per step over the first 64
  // token rows (a 64-row copy), the accumulator in lanes 0..15 of each TMEM lane
  // quadrant (row 16 q + i in lane 32 q + i)
  static constexpr bool M64 = DIRECT && WQ == WQ_BF16;
  static constexpr uint32_t IDESC_M64 = idesc_bf16(64, 128 * NA, false, true);
  // barriers + bookkeeping after the tiles
  // tile queue from the producer to the other roles
  static constexpr int TQ = 4;
  static constexpr int TQ_CONSUMERS = 1 + kEpiWarps + DEQ_WARPS;
  static constexpr uint32_t BAR_BYTES =
      8 * (2 * STAGES + 5 + 2 * A_SLOTS + 2 * TQ) + 16 + 4 * STAGES + 4 * TQ;
  // tile prefixes of the two problems, the heavy / light class prefixes of
  // problem 0 (interleaved order), and problem 0's group offsets
  static constexpr uint32_t PREFIX_BYTES = 5 * (kMaxGroups + 1) * 4;
  // swapped epilogue: per-tile output row and scale of each token, one copy per warp;
  // direct DOWN epilogue: a 32-row x 16-column FP32 staging tile per warp through
  // which rows are stored transposed
  static constexpr uint32_t EPI_BYTES =
      (EPI == EPI_DOWN && DIRECT) ? kEpiWarps * 32 * 16 * 4 : kEpiWarps * 128 * 8;
  static constexpr uint32_t SMEM_BYTES =
      1024 + STAGES * STAGE_BYTES + A_REGION + BAR_BYTES + PREFIX_BYTES + 16 + EPI_BYTES;
  static_assert(SMEM_BYTES + 64 <= 227 * 1024, "shared memory per CTA (dynamic + static)");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "tcgen05 M=128 needs N % 16 == 0");
  static_assert(!DIRECT || BN == 128, "direct tiles hold 128 tokens");
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep the 128-byte swizzle alignment");
  static_assert(NA * SCALE_BYTES <= 1024, "scale slot");
  static_assert(TMEM_NEED <= 512, "TMEM holds 512 columns");
};

// Decode a linear tile id.  Tiles run over problems, then (group, m-tile) in the
// tile prefix order, then the feature tiles innermost so that neighbouring CTAs
// share a token tile.
MOE_DEV void decode_tile(const TcParams& p, const int* prefix, int BN, int TN, int tile,
                         TileInfo& ti) {
  int pi = 0;
  for (; pi < p.n_prob; ++pi) {
    const TcProblem& P = p.prob[pi];
    const int* pre = prefix + pi * (kMaxGroups + 1);
    const int nt = (P.N + TN - 1) / TN;
    const int cnt = pre[P.G] * nt;
    if (tile < cnt) break;
    tile -= cnt;
  }
  const TcProblem& P = p.prob[pi];
  const int* pre = prefix + pi * (kMaxGroups + 1);
  const int nt = (P.N + TN - 1) / TN;
  const int mt = tile / nt;
  ti.prob = pi;
  ti.n0 = (tile % nt) * TN;
  int g;
  if (pi == 0 && p.interleave) {
    // position mt of the interleaved sequence: light tile number floor(mt L / N)
    // when that count steps up at mt, else heavy tile number mt - that count
    const int* hpre = prefix + 2 * (kMaxGroups + 1);
    const int* lpre = prefix + 3 * (kMaxGroups + 1);
    const int L = lpre[P.G], N = pre[P.G];
    const int lb = (int)((long long)mt * L / N);
    const int la = (int)((long long)(mt + 1) * L / N);
    if (la > lb) {
      g = find_group(lpre, P.G, lb);
      ti.m0 = 0;
    } else {
      const int h = mt - lb;
      g = find_group(hpre, P.G, h);
      ti.m0 = (h - hpre[g]) * BN;
    }
  } else {
    g = find_group(pre, P.G, mt);
    ti.m0 = (mt - pre[g]) * BN;
  }
  ti.g = g;
  int seg_start, seg_rows;
  if (P.offsets) {
    // problem 0's offsets were copied to shared memory with its tile prefix
    const int* so = pi == 0 ? prefix + 4 * (kMaxGroups + 1) : P.offsets;
    seg_start = so[g];
    seg_rows = so[g + 1] - seg_start;
    ti.b_row = seg_start + ti.m0;
  } else {
    seg_start = g * P.uniform_rows;
    seg_rows = P.uniform_rows;
    ti.b_row = P.b_row_base + g * P.b_group_stride + ti.m0;
  }
  ti.rows = min(BN, seg_rows - ti.m0);
  ti.whole = ti.m0 == 0 && seg_rows <= BN;
  ti.slot0 = seg_start + ti.m0;
  ti.out_seg = P.out_row_base + (size_t)seg_start + ti.m0;
}

// Work item t of an S-way split: output tile t / S, k-blocks of part t % S.
MOE_DEV void decode_work(const TcParams& p, const int* prefix, int BN, int TN, int S, int t,
                         TileInfo& ti) {
  ti.bt = t / S;
  ti.ks = t % S;
  decode_tile(p, prefix, BN, TN, ti.bt, ti);
  const int kbl = p.prob[ti.prob].K / 64;
  ti.kb0 = ti.ks * kbl / S;
  ti.kb1 = (ti.ks + 1) * kbl / S;
}
// K-parts of each output tile of a split-K launch (1 when the params hold no
// partial-sum buffer): as many as fit the grid, at most kMaxSplit, and at least
// two k-blocks per part.
MOE_DEV int split_parts(const TcParams& p, int out_tiles, int ncta) {
  if (p.split_part == nullptr || out_tiles <= 0) return 1;
  int kbmin = p.prob[0].K / 64;
  if (p.n_prob > 1 && p.prob[1].K / 64 < kbmin) kbmin = p.prob[1].K / 64;
  int S = ncta / out_tiles;
  if (S > kMaxSplit) S = kMaxSplit;
  if (S > kbmin / 2) S = kbmin / 2;
  return S < 1 ? 1 : S;
}

MOE_DEV int total_tiles(const TcParams& p, const int* prefix, int TN) {
  int tot = 0;
  for (int pi = 0; pi < p.n_prob; ++pi) {
    const TcProblem& P = p.prob[pi];
    tot += prefix[pi * (kMaxGroups + 1) + P.G] * ((P.N + TN - 1) / TN);
  }
  return tot;
}

MOE_DEV float silu_f(float u) { return __fdividef(u, 1.f + __expf(-u)); }

// Tokens a swapped tile's MMA covers: its rows rounded up to the MMA's N step of
// 16, at most the tile width BN.  A tile of a lightly loaded expert then costs MMA
// time (and, with the in-GEMM gather, copies) for its own rows only, while the
// heavily loaded experts get wide tiles that stream their weights fewer times.
MOE_DEV int tile_n(int rows, int BN) {
  const int n = (rows + 15) & ~15;
  return n < 16 ? 16 : n > BN ? BN : n;
}
// the instruction descriptor with its N field (bits 17..22, N >> 3) replaced
MOE_DEV uint32_t idesc_with_n(uint32_t idesc, int n) {
  return (idesc & ~(0x3Fu << 17)) | ((uint32_t)(n >> 3) << 17);
}

// Eight int4 codes of one 4-byte word (two's complement nibbles; nibble j of the
// little-endian word holds code (0, 2, 4, 6, 1, 3, 5, 7)[j] of the eight, the storage
// order of the layer's int4 weights) to bf16 q*s, packed as four bf16x2 pairs of
// consecutive codes.  XOR 8 turns each nibble into the offset value q + 8 in
// [0, 15]; masking nibbles j and j + 4 -- codes 2j and 2j+1 -- into the low mantissa
// bits of the two halves of bf16 128.0 (0x4300) gives exactly 136 + q; subtracting
// 136.0 (0x4308) leaves q exactly; one bf16x2 multiply by the scale pair yields the
// exact product q*s rounded once (round to nearest even).
MOE_DEV void int4x8_to_bf16(uint32_t v, const uint32_t (&s2)[4], uint32_t (&o)[4]) {
  v ^= 0x88888888u;
  const uint32_t magic = 0x43004300u;
  const __nv_bfloat162 k136 = __halves2bfloat162(__ushort_as_bfloat16(0x4308),
                                                 __ushort_as_bfloat16(0x4308));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t a = ((v >> (4 * i)) & 0x000F000Fu) | magic;   // codes (2i, 2i + 1)
    const __nv_bfloat162 q = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a), k136);
    const __nv_bfloat162 r = __hmul2(q, *reinterpret_cast<const __nv_bfloat162*>(&s2[i]));
    o[i] = *reinterpret_cast<const uint32_t*>(&r);
  }
}

// NC consecutive codes of one feature (64: a whole k-block, 32: half of it;
// stored K-contiguous in shared memory: int4 NC/2 bytes, int8 / fp8 NC bytes) to
// NC/2 bf16x2 words, code 2c in the low half of word c, each value bf16(q * s):
// the exact product rounded once.  The 16-byte pieces are read in a lane-rotated
// order so that the lanes of each quarter-warp spread over the banks.
template <int WQ, int NC = 64>
MOE_DEV void dequant_row(const uint8_t* row, __nv_bfloat16 s, int lane, uint32_t (&o)[NC / 2]) {
  constexpr int P = (WQ == WQ_INT4 ? NC / 2 : NC) / 16;   // 16-byte pieces of the codes
  // load j reads piece (j + r) % P, r depending on the lane; rotated back below
  const int r = P == 1 ? 0 : (lane >> (P == 2 ? 2 : 1)) & (P - 1);
  uint4 v[P];
#pragma unroll
  for (int j = 0; j < P; ++j) v[j] = *reinterpret_cast<const uint4*>(row + 16 * ((j + r) & (P - 1)));
  if (P == 2 && r) {
    const uint4 t = v[0];
    v[0] = v[P - 1];
    v[P - 1] = t;
  }
  if (P == 4) {
    if (r & 1) {
      const uint4 t = v[3 % P];
      v[3 % P] = v[2 % P];
      v[2 % P] = v[1 % P];
      v[1 % P] = v[0];
      v[0] = t;
    }
    if (r & 2) {
      uint4 t = v[0];
      v[0] = v[2 % P];
      v[2 % P] = t;
      t = v[1 % P];
      v[1 % P] = v[3 % P];
      v[3 % P] = t;
    }
  }
  uint32_t wd[4 * P];
#pragma unroll
  for (int j = 0; j < P; ++j) {
    wd[4 * j] = v[j].x;
    wd[4 * j + 1] = v[j].y;
    wd[4 * j + 2] = v[j].z;
    wd[4 * j + 3] = v[j].w;
  }
  if (WQ == WQ_INT4) {
    const uint32_t s2 = (uint32_t)__bfloat16_as_ushort(s) * 0x10001u;
    const uint32_t sp[4] = {s2, s2, s2, s2};
#pragma unroll
    for (int i = 0; i < 4 * P; ++i) {
      uint32_t q4[4];
      int4x8_to_bf16(wd[i], sp, q4);
#pragma unroll
      for (int j = 0; j < 4; ++j) o[4 * i + j] = q4[j];
    }
  } else {
    const float sf = __bfloat162float(s);
#pragma unroll
    for (int i = 0; i < 4 * P; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float q0, q1;
        if (WQ == WQ_FP8) {
          const float2 q = e4m3x2_to_float2(wd[i] >> (16 * h));
          q0 = q.x;
          q1 = q.y;
        } else {
          // offset binary u = q + 128 placed in the mantissa of 2^23: the float
          // 2^23 + u, minus 2^23 + 128, is q exactly (full-rate byte permute and
          // add instead of the quarter-rate integer-to-float conversion)
          const uint32_t u = wd[i] ^ 0x80808080u;
          q0 = __uint_as_float(__byte_perm(u, 0x4B000000u, h ? 0x7542 : 0x7540)) - 8388736.f;
          q1 = __uint_as_float(__byte_perm(u, 0x4B000000u, h ? 0x7543 : 0x7541)) - 8388736.f;
        }
        __nv_bfloat162 rr = __floats2bfloat162_rn(q0 * sf, q1 * sf);
        o[2 * i + h] = *reinterpret_cast<uint32_t*>(&rr);
      }
    }
  }
}

// Direct orientation (tokens on the MMA's M side): output row and scale of token
// row m of the tile (r = -1 past the end of the segment).
template <int EPI>
MOE_DEV void direct_row(const TcProblem& P, const TileInfo& ti, int m, int& r, float& sc) {
  r = -1;
  sc = 1.f;
  if (m < ti.rows) {
    if (EPI == EPI_DOWN && P.perm_assign) {
      r = P.perm_assign[ti.slot0 + m];
      sc = P.gate[r];
    } else {
      r = (int)(ti.out_seg + m);
    }
  }
}

// Staging tile of the direct DOWN epilogue: 32 rows x 16 floats per warp, the four
// 16-byte pieces of row r stored in the order j ^ ((r >> 1) & 3), so that the
// lane-per-row writes and the row-striped reads of both output types hit 32
// distinct banks per 8 lanes.
MOE_DEV int stg_at(int r, int j) { return r * 16 + 4 * (j ^ ((r >> 1) & 3)); }

// Direct-orientation epilogue: this thread holds TMEM lane (q*32 + lane) of the
// accumulator at t_base, i.e. one token row, whose output row is r (-1: none).
// GATEUP: 128 features, gate in columns [0,128), up in [128,256); each half of the
// warps takes 64 features and writes bf16 h.  DOWN: TN features, half each, scaled
// by the gate and stored through the warp's staging tile `stg` (32 rows x 16 floats).
template <int EPI, int TN>
MOE_DEV void direct_store(const TcProblem& P, const TileInfo& ti, int r, float sc,
                          uint32_t t_base, int half, int lane, float* stg) {
  constexpr int CPH = (EPI == EPI_GATEUP) ? 4 : TN / 32;   // chunks per half
#pragma unroll 1
  for (int c = half * CPH; c < half * CPH + CPH; ++c) {
    const int n = ti.n0 + c * 16;
    if (n >= P.n_valid) break;
    float v0[16];
    tmem_ld16(t_base + c * 16, v0);
    float v1[16];
    if (EPI == EPI_GATEUP) tmem_ld16(t_base + 128 + c * 16, v1);
    tmem_wait_ld();
    if (r >= 0 && EPI == EPI_GATEUP) {
      uint32_t pk[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(silu_f(v0[2 * j]) * v1[2 * j],
                                                  silu_f(v0[2 * j + 1]) * v1[2 * j + 1]);
        pk[j] = *reinterpret_cast<uint32_t*>(&h2);
      }
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(P.out) +
                                            (size_t)r * P.ld_out + n);
      dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    } else if (EPI != EPI_GATEUP) {
      // Through a per-warp staging tile: each lane writes its row's 16 scaled values,
      // then several lanes store one row's contiguous bytes (FP32: 4 lanes x 16 B,
      // 8 rows per instruction; bf16: 2 lanes x 16 B, 16 rows per instruction), so
      // every store fills whole 32-byte sectors.
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<float4*>(stg + stg_at(lane, j)) =
            make_float4(v0[4 * j] * sc, v0[4 * j + 1] * sc, v0[4 * j + 2] * sc,
                        v0[4 * j + 3] * sc);
      __syncwarp();
      if (P.out_bf16) {
        const int hh = (lane & 1) * 8;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int rr = (lane >> 1) + 16 * i;
          const int rout = __shfl_sync(0xffffffffu, r, rr);
          const float4 a = *reinterpret_cast<const float4*>(stg + stg_at(rr, 2 * (lane & 1)));
          const float4 b = *reinterpret_cast<const float4*>(stg + stg_at(rr, 2 * (lane & 1) + 1));
          __nv_bfloat162 h0 = __floats2bfloat162_rn(a.x, a.y);
          __nv_bfloat162 h1 = __floats2bfloat162_rn(a.z, a.w);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(b.x, b.y);
          __nv_bfloat162 h3 = __floats2bfloat162_rn(b.z, b.w);
          if (rout >= 0)
            *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(P.out) +
                                      (size_t)rout * P.ld_out + n + hh) =
                make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                           *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
        }
      } else {
        const int qq = (lane & 3) * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rr = (lane >> 2) + 8 * i;
          const int rout = __shfl_sync(0xffffffffu, r, rr);
          const float4 v = *reinterpret_cast<const float4*>(stg + stg_at(rr, lane & 3));
          if (rout >= 0)
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(P.out) + (size_t)rout * P.ld_out +
                                       n + qq) = v;
        }
      }
      __syncwarp();
    }
  }
}

// The grouped GEMM of one CTA over the work items cta, cta + ncta, ...: barrier
// set-up in its shared memory (`smem`, 1024-byte aligned, C::SMEM_BYTES - 1024
// bytes), the warp roles, and after an abort the drain of this CTA's copies still
// in flight.  The caller has allocated C::TMEM_COLS columns of TMEM, whose address
// is at *tmem_slot once the CTA has synchronised.  with_pdl: wait for the previous
// kernel of the stream (programmatic dependent launch) before reading global
// memory.  All threads of the CTA call it; it returns after a __syncthreads, with
// every MMA it issued complete and every barrier idle, true unless one of this
// CTA's waits ran out (device error 2 is then set).
template <int EPI, int BN, bool DIRECT, int WQ>
MOE_DEV bool tc_gemm_run(const TcParams& p, uint8_t* smem, const uint32_t* tmem_slot, int cta,
                         int ncta, bool with_pdl) {
  using C = TcConfig<EPI, BN, DIRECT, WQ>;
  constexpr int NA = C::NA;
  constexpr int STAGES = C::STAGES;
  uint8_t* tiles = smem;
  uint8_t* wslots = tiles + STAGES * C::STAGE_BYTES;   // direct quantised: expanded weights
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(wslots + C::A_REGION);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;   // [2]
  uint64_t* tempty_bar = tfull_bar + 2;       // [2]
  uint64_t* drain_bar = tempty_bar + 2;       // [1]
  uint64_t* deq_bar = drain_bar + 1;                   // [A_SLOTS] weight slot filled
  uint64_t* aempty_bar = deq_bar + C::A_SLOTS;         // [A_SLOTS] weight slot consumed
  uint64_t* tq_full = aempty_bar + C::A_SLOTS;         // [TQ] tile index written
  uint64_t* tq_empty = tq_full + C::TQ;                // [TQ] tile index read by every role
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tq_empty + C::TQ) + 1;
  int* issued = const_cast<int*>(abort_flag) + 2;               // [STAGES] last issued parity+1
  volatile int* tq = issued + STAGES;                           // [TQ] tile indices
  int* prefix = reinterpret_cast<int*>(
      reinterpret_cast<uint8_t*>(full_bar) + C::BAR_BYTES);
  // epilogue scratch, 16-byte aligned (float4 staging in the direct DOWN epilogue)
  int* epi_row = reinterpret_cast<int*>(
      (reinterpret_cast<uintptr_t>(prefix + 5 * (kMaxGroups + 1)) + 15) & ~uintptr_t(15));
  float* epi_scale = reinterpret_cast<float*>(epi_row + kEpiWarps * 128);  // [8 warps][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      issued[s] = 0;
    }
    for (int a = 0; a < C::A_SLOTS; ++a) {
      mbar_init(&deq_bar[a], C::DEQ_WARPS);
      mbar_init(&aempty_bar[a], 1);
    }
    for (int q = 0; q < C::TQ; ++q) {
      mbar_init(&tq_full[q], 1);
      mbar_init(&tq_empty[q], C::TQ_CONSUMERS);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    for (int pi = 0; pi < p.n_prob; ++pi) {
      tma_prefetch_desc(&p.prob[pi].tmA);
      if (NA == 2) tma_prefetch_desc(&p.prob[pi].tmA2);
      tma_prefetch_desc(&p.prob[pi].tmB);
    }
  }
  // everything above touched only this CTA's shared memory, TMEM and the kernel
  // parameters; from here on the previous kernel's outputs are read
  if (with_pdl) {
    pdl_wait();
    pdl_trigger();
  }
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
  constexpr int TN = C::TILE_N;
  const int out_tiles = total_tiles(p, prefix, TN);
  // split-K is compiled into the narrow swapped expert tiles only
  constexpr bool kCanSplit = !DIRECT && EPI != EPI_ROUTER && BN <= 64;
  int S = 1;
  if (EPI == EPI_ROUTER && p.k_splits > 1) S = p.k_splits;
  if (kCanSplit) S = split_parts(p, out_tiles, ncta);
  const int total = out_tiles * S;

  // Tile queue.  The producer's lane 0 decides each tile of this CTA -- statically,
  // or from the dynamic counter after the first -- and publishes it; the MMA thread,
  // the epilogue warps and the dequantisation warps read the same sequence.  An
  // index >= total ends it.
  auto next_tile = [&](int k) -> int {
    if (k == 0) return cta;
    return p.tile_ctr ? ncta + atomicAdd(p.tile_ctr, 1) : cta + k * ncta;
  };
  int tq_slot = 0;        // this thread's position in the queue
  uint32_t tq_phase = 0;
  auto push_tile = [&](int t) -> bool {
    if (!mbar_wait(&tq_empty[tq_slot], tq_phase ^ 1, p.err, abort_flag, p.wait_cycles)) return false;
    tq[tq_slot] = t;
    mbar_arrive(&tq_full[tq_slot]);
    if (++tq_slot == C::TQ) { tq_slot = 0; tq_phase ^= 1; }
    return true;
  };
  // one consumer: a whole warp (every lane reads, lane 0 counts) or a lone thread
  auto pop_tile = [&](bool whole_warp, bool patient) -> int {
    if (!mbar_wait(&tq_full[tq_slot], tq_phase, p.err, abort_flag, p.wait_cycles, patient))
      return total;
    const int t = tq[tq_slot];
    if (whole_warp) __syncwarp();
    if (!whole_warp || lane == 0) mbar_arrive(&tq_empty[tq_slot]);
    if (++tq_slot == C::TQ) { tq_slot = 0; tq_phase ^= 1; }
    return t;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Lane 0 waits for free stages, arms them and loads the weights.  Token rows: a
    // tiled load by lane 0, or (gathered problems) one tile::gather4 of four rows
    // per lane, lanes 0 .. BN/4-1, after lane 0 has armed the stage.  Without any
    // gathered problem lane 0 runs alone.
    const bool any_gather = p.prob[0].gather_rows != nullptr ||
                            (p.n_prob > 1 && p.prob[1].gather_rows != nullptr);
    // arm stage `stage` of tile ti, k-block kb, and request everything but gathered rows
    auto issue_stage = [&](uint8_t* st, int stage, uint32_t phase, const TileInfo& ti,
                           const TcProblem& P, int kb, bool gather) {
      // gathered rows: only the tile's own (rounded up to 16), 128 B each
      const bool m64 = C::M64 && ti.rows <= 64;
      mbar_arrive_expect_tx(&full_bar[stage],
                            gather ? C::TX_BYTES - C::B_BYTES + 128u * tile_n(ti.rows, BN)
                                   : C::TX_BYTES - (m64 ? 64u * 128u : 0u));
      issued[stage] = (int)phase + 1;
      // GATEUP: the up matrix at the same features; wide DOWN: features +128
      const void* m2 = (EPI == EPI_GATEUP) ? (const void*)&P.tmA2 : (const void*)&P.tmA;
      const int n2 = (EPI == EPI_GATEUP) ? ti.n0 : ti.n0 + 128;
      if (WQ == WQ_BF16 && DIRECT && ti.whole) {
        // the weights of a group that fits one token tile are read by this tile
        // only: first out of L2, after the lines that later token tiles re-read
        const uint64_t pol = l2_evict_first();
        tma_load_3d_hint(st, &P.tmA, &full_bar[stage], ti.n0, kb * 64, ti.g, pol);
        tma_load_3d_hint(st + 8192, &P.tmA, &full_bar[stage], ti.n0 + 64, kb * 64, ti.g, pol);
        if (NA == 2) {
          tma_load_3d_hint(st + C::A_BYTES, m2, &full_bar[stage], n2, kb * 64, ti.g, pol);
          tma_load_3d_hint(st + C::A_BYTES + 8192, m2, &full_bar[stage], n2 + 64, kb * 64, ti.g,
                           pol);
        }
      } else if (WQ == WQ_BF16) {
        tma_load_3d(st, &P.tmA, &full_bar[stage], ti.n0, kb * 64, ti.g);
        tma_load_3d(st + 8192, &P.tmA, &full_bar[stage], ti.n0 + 64, kb * 64, ti.g);
        if (NA == 2) {
          tma_load_3d(st + C::A_BYTES, m2, &full_bar[stage], n2, kb * 64, ti.g);
          tma_load_3d(st + C::A_BYTES + 8192, m2, &full_bar[stage], n2 + 64, kb * 64, ti.g);
        }
      } else {
        // raw codes stored K-contiguous [G][N][K bytes]: x is the byte offset of the
        // k-block within a feature's row, y the first feature
        uint8_t* raw = st + C::RAW_OFF;
        uint8_t* scl = st + C::SCALE_OFF;
        const int kx = kb * (int)C::RAW_ROW;
        const void* s2 = (EPI == EPI_GATEUP) ? (const void*)&P.tmS2 : (const void*)&P.tmS;
        tma_load_3d(raw, &P.tmA, &full_bar[stage], kx, ti.n0, ti.g);
        // int8: scales [G][N] (second coordinate g, third 0); int4: [G][K/128][N]
        if (WQ != WQ_INT4) tma_load_3d(scl, &P.tmS, &full_bar[stage], ti.n0, ti.g, 0);
        else tma_load_3d(scl, &P.tmS, &full_bar[stage], ti.n0, kb / 2, ti.g);
        if (NA == 2) {
          tma_load_3d(raw + C::RAW_BYTES, m2, &full_bar[stage], kx, n2, ti.g);
          if (WQ != WQ_INT4) tma_load_3d(scl + 256, s2, &full_bar[stage], n2, ti.g, 0);
          else tma_load_3d(scl + 256, s2, &full_bar[stage], n2, kb / 2, ti.g);
        }
      }
      if (!gather)
        tma_load_2d(st + C::TOKEN_OFF, m64 ? (const void*)&P.tmB64 : (const void*)&P.tmB,
                    &full_bar[stage], kb * 64, ti.b_row);
    };
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    if (!any_gather) {
      if (lane == 0) {
        for (int k = 0; ok; ++k) {
          const int tile = next_tile(k);
          if (!push_tile(tile)) { ok = false; break; }
          if (tile >= total) break;
          TileInfo ti;
          decode_work(p, prefix, BN, TN, S, tile, ti);
          const TcProblem& P = p.prob[ti.prob];
          for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
            if (!mbar_wait(&empty_bar[stage], phase ^ 1, p.err, abort_flag, p.wait_cycles)) { ok = false; break; }
            issue_stage(tiles + stage * C::STAGE_BYTES, stage, phase, ti, P, kb, false);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
      }
    } else {
      for (int k = 0; ok; ++k) {
        int tile = 0;
        if (lane == 0) {
          tile = next_tile(k);
          if (!push_tile(tile)) tile = -1;
        }
        tile = __shfl_sync(0xffffffffu, tile, 0);
        if (tile < 0) { ok = false; break; }
        if (tile >= total) break;
        TileInfo ti;
        decode_work(p, prefix, BN, TN, S, tile, ti);
        const TcProblem& P = p.prob[ti.prob];
        const bool gather = P.gather_rows != nullptr;
        // this lane's four rows; rows past the segment repeat the tile's first row
        // (their accumulators are never stored)
        int rr[4] = {0, 0, 0, 0};
        const int n_gather = gather ? tile_n(ti.rows, BN) / 4 : 0;   // copies of 4 rows
        if (lane < n_gather) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int m = 4 * lane + j;
            rr[j] = P.gather_rows[ti.slot0 + (m < ti.rows ? m : 0)] / P.gather_k;
          }
        }
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          int okw = 1;
          if (lane == 0) okw = mbar_wait(&empty_bar[stage], phase ^ 1, p.err, abort_flag, p.wait_cycles) ? 1 : 0;
          if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
          uint8_t* st = tiles + stage * C::STAGE_BYTES;
          if (lane == 0) issue_stage(st, stage, phase, ti, P, kb, gather);
          __syncwarp();   // the stage is armed before any gathered row can land
          if (lane < n_gather)
            tma_gather4(st + C::TOKEN_OFF + lane * 512, &P.tmB, &full_bar[stage], kb * 64,
                        rr[0], rr[1], rr[2], rr[3]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int aslot = 0;
      uint32_t aphase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      while (ok) {
        const int tile = pop_tile(false, false);
        if (tile >= total) break;
        TileInfo ti;
        decode_work(p, prefix, BN, TN, S, tile, ti);
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, p.err, abort_flag, p.wait_cycles)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::ACC_COLS;
        const uint32_t idesc = (C::M64 && ti.rows <= 64) ? C::IDESC_M64
                               : DIRECT ? C::IDESC
                                        : idesc_with_n(C::IDESC, tile_n(ti.rows, BN));
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, p.err, abort_flag, p.wait_cycles)) { ok = false; break; }
          if (WQ != WQ_BF16 &&
              !mbar_wait(&deq_bar[aslot], aphase, p.err, abort_flag, p.wait_cycles)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st_addr = smem_u32(tiles + stage * C::STAGE_BYTES);
          const uint32_t b_addr = st_addr + C::TOKEN_OFF;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // weights: MN-major SW128, 16 k-rows of 128 B per MMA step; the two
            //    64-feature halves sit 8 KB apart (leading offset), 8-row groups 1 KB
            //    apart.  tokens: K-major SW128, 16 k = 32 B per step, 8-row groups 1 KB.
            //    Dequantised weights: TMEM, 8 columns (16 k) per step.
            const uint64_t xd = sw128_desc(b_addr + kk * 32, 16, 1024);
            const uint32_t accum = (kb != ti.kb0 || kk != 0);
            if (C::SMEM_W) {
              const uint64_t wd =
                  sw128_desc(smem_u32(wslots + aslot * C::W_SLOT_BYTES) + kk * 32, 16, 1024);
              tc_mma_f16(d_tmem, xd, wd, C::IDESC, accum);   // N = 128 * NA at once
            } else if (WQ != WQ_BF16) {
              const uint32_t a_tm = tmem_base + C::A_COL0 + aslot * C::A_SLOT_COLS + kk * 8;
              tc_mma_f16_tmem_a(d_tmem, a_tm, xd, idesc, accum);
              if (NA == 2) tc_mma_f16_tmem_a(d_tmem + BN, a_tm + 32, xd, idesc, accum);
            } else if (DIRECT) {
              const uint64_t wd = sw128_desc(st_addr + kk * 2048, 8192, 1024);
              tc_mma_f16(d_tmem, xd, wd, idesc, accum);   // N = 128 * NA at once
            } else {
              const uint64_t wd = sw128_desc(st_addr + kk * 2048, 8192, 1024);
              tc_mma_f16(d_tmem, wd, xd, idesc, accum);
              if (NA == 2) {
                const uint64_t wd2 = sw128_desc(st_addr + C::A_BYTES + kk * 2048, 8192, 1024);
                tc_mma_f16(d_tmem + BN, wd2, xd, idesc, accum);
              }
            }
          }
          tc_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
          if (WQ != WQ_BF16) {
            tc_commit(&aempty_bar[aslot]);
            if (++aslot == C::A_SLOTS) { aslot = 0; aphase ^= 1; }
          }
        }
        if (!ok) break;
        tc_commit(&tfull_bar[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // wait until every MMA issued above has completed before TMEM is released
      tc_commit(drain_bar);
      long long t0 = clock64();
      while (!mbar_try_wait(drain_bar, 0) && clock64() - t0 < kWaitCycles) {}
    }
    __syncwarp();
  } else if (warp >= 2 + kEpiWarps) {
    // ------------------------------------------------------------ dequantisation
    if (WQ != WQ_BF16) {
      // swapped tiles: warp w expands weight block (w - 10) / 4 for the 32 features
      // of its TMEM lane quadrant w % 4, one thread per feature, its 64 codes of the
      // k-block; direct tiles: warp w, block (w - 10) / 8, codes [32 sub, 32 sub + 32)
      // with sub = ((w - 10) / 4) % 2, of the features of quadrant w % 4
      const int dw = warp - 2 - kEpiWarps;
      const int blk = C::SMEM_W ? dw >> 3 : dw >> 2;
      const int sub = C::SMEM_W ? (dw >> 2) & 1 : 0;
      const int qd = warp & 3;
      const int feat = qd * 32 + lane;
      int stage = 0;
      uint32_t phase = 0;
      int aslot = 0;
      uint32_t aphase = 0;
      bool ok = true;
      while (ok) {
        const int tile = pop_tile(true, true);
        if (tile >= total) break;
        TileInfo ti;
        decode_work(p, prefix, BN, TN, S, tile, ti);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, p.err, abort_flag, p.wait_cycles)) { ok = false; break; }
          if (!mbar_wait(&aempty_bar[aslot], aphase ^ 1, p.err, abort_flag, p.wait_cycles)) { ok = false; break; }
          tc_fence_after();
          const uint8_t* st = tiles + stage * C::STAGE_BYTES;
          const uint8_t* row = st + C::RAW_OFF + blk * C::RAW_BYTES + feat * C::RAW_ROW;
          const __nv_bfloat16 sc =
              reinterpret_cast<const __nv_bfloat16*>(st + C::SCALE_OFF)[128 * blk + feat];
          if (C::SMEM_W) {
            uint32_t w[16];
            dequant_row<WQ, 32>(row + sub * (C::RAW_ROW / 2), sc, lane, w);
            // row (blk*128 + feat) of the slot, 16-byte chunk c at c ^ (row & 7)
            const int wr = blk * 128 + feat;
            uint8_t* dst = wslots + aslot * C::W_SLOT_BYTES + wr * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4*>(dst + 16 * ((4 * sub + c) ^ (wr & 7))) =
                  make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
            fence_proxy_async_shared();   // the tensor core reads them through the async proxy
          } else {
            uint32_t w[32];
            dequant_row<WQ>(row, sc, lane, w);
            tmem_st32(tmem_base + ((uint32_t)(qd * 32) << 16) + C::A_COL0 +
                          aslot * C::A_SLOT_COLS + blk * 32,
                      w);
            tmem_wait_st();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&deq_bar[aslot]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
          if (++aslot == C::A_SLOTS) { aslot = 0; aphase ^= 1; }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int half = (warp - 2) >> 2;       // which half of the columns it drains
    int* s_row = epi_row + (warp - 2) * 128;
    float* s_scale = epi_scale + (warp - 2) * 128;
    int acc = 0;
    uint32_t acc_phase = 0;
    while (true) {
      const int tile = pop_tile(true, true);
      if (tile >= total) break;
      TileInfo ti;
      decode_work(p, prefix, BN, TN, S, tile, ti);
      const TcProblem& P = p.prob[ti.prob];
      const uint32_t t_base = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      if (DIRECT) {
        // this thread's token row; its output row and gate are fetched before the
        // accumulator wait so that the loads overlap the MMAs
        int r;
        float sc;
        const bool m64 = C::M64 && ti.rows <= 64;
        direct_row<EPI>(P, ti, m64 ? (lane < 16 ? q * 16 + lane : BN) : q * 32 + lane, r, sc);
        if (!mbar_wait(&tfull_bar[acc], acc_phase, p.err, abort_flag, p.wait_cycles, true)) break;
        tc_fence_after();
        direct_store<EPI, TN>(P, ti, r, sc, t_base, half, lane,
                              reinterpret_cast<float*>(epi_row) + (warp - 2) * (32 * 16));
      } else {
        // swapped: this thread owns feature n; the tile's token rows and scales are
        // staged in this warp's shared-memory slice (warp-private: __syncwarp only)
        __syncwarp();
        for (int m = lane; m < BN; m += 32) {
          int r = -1;
          float sc = 1.f;
          if (m < ti.rows) {
            if (EPI == EPI_DOWN && P.perm_assign) {
              r = P.perm_assign[ti.slot0 + m];
              sc = P.gate[r];
            } else {
              r = (int)(ti.out_seg + m);
            }
          }
          s_row[m] = r;
          s_scale[m] = sc;
        }
        __syncwarp();
        if (!mbar_wait(&tfull_bar[acc], acc_phase, p.err, abort_flag, p.wait_cycles, true)) break;
        tc_fence_after();
        const int n = ti.n0 + q * 32 + lane;
        const bool n_ok = n < P.n_valid;
        // split-K: this work item's partial sums, feature-contiguous per column
        // (column c*16+j of the gate block, BN + c*16+j of the up block)
        constexpr size_t PART = (size_t)NA * BN * 128;
        const int fo = q * 32 + lane;
        bool finish = true;   // this work item stores the tile's outputs
        if (kCanSplit && S > 1) {
          float* part = p.split_part + (size_t)tile * PART;
#pragma unroll 1
          for (int c = half; c < BN / 16; c += 2) {
            if (c * 16 >= ti.rows) break;
            float v0[16];
            tmem_ld16(t_base + c * 16, v0);
            float v1[16];
            if (NA == 2) tmem_ld16(t_base + BN + c * 16, v1);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              part[(size_t)(c * 16 + j) * 128 + fo] = v0[j];
              if (NA == 2) part[(size_t)(BN + c * 16 + j) * 128 + fo] = v1[j];
            }
          }
          // Count this part of the warp's slice once its stores are visible; the
          // last of the S parts adds them all in split order (the same sums
          // whichever part finishes last) and stores the outputs.  Nothing waits.
          __threadfence();
          __syncwarp();
          int last = 0;
          if (lane == 0) {
            int32_t* cnt = p.split_cnt + ti.bt * kEpiWarps + (warp - 2);
            last = atomicAdd(cnt, 1) == S - 1;
            if (last) atomicExch(cnt, 0);   // zero again for the next launch
          }
          finish = __shfl_sync(0xffffffffu, last, 0) != 0;
          if (finish) __threadfence();
        }
        const float* p0 = S > 1 ? p.split_part + (size_t)ti.bt * S * PART : nullptr;
#pragma unroll 1
        for (int c = half; c < BN / 16 && finish; c += 2) {
          if (c * 16 >= ti.rows) break;
          float v0[16], v1[16];
          if (!kCanSplit || S == 1) {
            tmem_ld16(t_base + c * 16, v0);
            if (NA == 2) tmem_ld16(t_base + BN + c * 16, v1);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float a0 = 0.f, a1 = 0.f;
              for (int ss = 0; ss < S; ++ss) {
                const float* ps = p0 + (size_t)ss * PART;
                a0 += __ldcg(ps + (size_t)(c * 16 + j) * 128 + fo);
                if (NA == 2) a1 += __ldcg(ps + (size_t)(BN + c * 16 + j) * 128 + fo);
              }
              v0[j] = a0;
              v1[j] = a1;
            }
          }
          if (EPI == EPI_GATEUP) {
            __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(P.out);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int r = s_row[c * 16 + j];
              if (r >= 0 && n_ok)
                H[(size_t)r * P.ld_out + n] = __float2bfloat16_rn(silu_f(v0[j]) * v1[j]);
            }
          } else if (EPI == EPI_DOWN && P.out_bf16) {
            __nv_bfloat16* Y = reinterpret_cast<__nv_bfloat16*>(P.out);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int r = s_row[c * 16 + j];
              if (r >= 0 && n_ok)
                Y[(size_t)r * P.ld_out + n] = __float2bfloat16_rn(v0[j] * s_scale[c * 16 + j]);
            }
          } else {
            float* Y = reinterpret_cast<float*>(P.out) +
                       (EPI == EPI_ROUTER ? ti.ks * p.split_out_stride : 0);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int r = s_row[c * 16 + j];
              if (r >= 0 && n_ok) Y[(size_t)r * P.ld_out + n] = v0[j] * s_scale[c * 16 + j];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // copies still in flight after an abort: wait (bounded) for each stage's last load
    for (int s = 0; s < STAGES; ++s) {
      if (issued[s]) {
        long long t0 = clock64();
        while (!mbar_try_wait(&full_bar[s], (uint32_t)(issued[s] - 1)) &&
               clock64() - t0 < kWaitCycles) {}
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  return *abort_flag == 0;
}

template <int EPI, int BN, bool DIRECT, int WQ>
__global__ void __launch_bounds__(TcConfig<EPI, BN, DIRECT, WQ>::THREADS, 1)
    k_tc_gemm(const __grid_constant__ TcParams p) {
  using C = TcConfig<EPI, BN, DIRECT, WQ>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if ((threadIdx.x >> 5) == 1) {
    tmem_alloc(&tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_gemm_run<EPI, BN, DIRECT, WQ>(p, smem, &tmem_slot, blockIdx.x, gridDim.x, true);
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_slot, C::TMEM_COLS);
  }
}

}  // namespace moe
