// fd_kernels.cuh — sm_100a kernels of split-KV decode attention.
//
// Split kernel: one CTA per (split, KV head, sequence).  It streams the
// split's K/V tiles from HBM through a multi-stage shared-memory pipeline
// fed by TMA tensor loads (128-byte swizzle; the first tiles are prefetched
// into L2 before the wait on the previous grid), and runs the scores and the
// P.V product for all G query heads of the KV head on the tensor cores
// (mma.sync in bf16, or f16 for an fp8 E4M3 cache converted in registers;
// fp32 accumulation), with an online softmax in between.
// Each split ends with a partial output and a log-sum-exp ("What is
// Flash-Decoding, and when does it speed up LLMs?", slavadubrov.com, section
// "Why decode needs a different schedule").  The running maximum and
// normaliser of the online softmax follow the FlashAttention-style streaming
// described in the last abstract of scifaro.com's "Related papers:
// INT-FlashAttention" list.
//
// Combine kernel: one warp per (sequence, query head) merges that row's
// partials with the log-sum-exp weights m = max_s lse_s,
// O = sum_s e^(lse_s - m) O_s / sum_s e^(lse_s - m), lse = m + ln sum_s
// e^(lse_s - m).  It is chained to the split kernel by programmatic
// dependent launch.  A sequence whose history fits one split gets its result
// straight from the split kernel.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "fd_ptx.cuh"

namespace fd {

constexpr int kTile = 64;           // tokens per pipeline stage
constexpr int kTileWarps = 4;       // consumer warps per tile, 16 tokens each
constexpr int kConsumerWarps = 4;   // consumer warps of a CTA sized for two CTAs per SM
constexpr int kCtasPerSm = 2;       // occupancy the split kernel is sized for
constexpr int kCombineWarps = 4;    // rows (one per warp) per combine CTA
// A CTA alone on its SM runs two sets of four consumer warps, which take the
// even and the odd tiles: one warp per SM sub-partition is bound by the
// latency of its tile loop, two hide it.
constexpr int kWideConsumerWarps = 8;
template <int CW>
constexpr int split_threads() { return (CW + 1) * 32; }
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s

// How the softmax weights P enter the bf16 P.V contraction.
//  kDup : G <= 4.  Query heads fill columns 0..3 of the n=8 MMA and are
//         duplicated into columns 4..7.  Columns 0..3 carry bf16(p), columns
//         4..7 carry the rounding residual p - bf16(p); their sum restores p
//         to ~16 bits at no extra MMA.
//  kHiLo: G = 8 per column block.  A second P.V MMA adds the residual.
//  kHi  : one P.V MMA with P as is: the fp8 path, whose P is f16 (11
//         significant bits).
enum PMode { kDup = 0, kHiLo = 1, kHi = 2 };

// Device error word: set when a bounded wait runs out.
__device__ unsigned int g_error_word;

struct SplitArgs {
  const __nv_bfloat16* q;       // [B, Hq, D]
  const int32_t* seqlens;       // [B] or null
  const int32_t* block_table;   // [B, max_blocks_per_seq] or null
  __nv_bfloat16* out;           // [B, Hq, D] bf16 result (null when out_f32 is set)
  float* out_f32;               // [B, Hq, D] fp32 result instead (partial over a shard)
  float* lse;                   // [B, Hq] or null     (one split)
  float* part_o;                // [B, Hq, S, D]       (several splits)
  float* part_lse;              // [B, Hq, S]          (several splits)
  int Hq, Hkv, G;
  int max_len;
  int block_size, log2_block_size;
  int log2_box_rows;            // rows per TMA box: 64, or the page size when smaller
  int max_blocks_per_seq;
  int tiles;                    // 64-token tiles of max_len, T = ceil(max_len / 64)
  int n_splits;                 // effective split count S = gridDim.x, 1 <= S <= max(T, 1)
  int tile_q, tile_r;           // T = tile_q * S + tile_r, 0 <= tile_r < S
  float scale_log2;             // scale * k_scale * log2(e)
  float v_scale;                // dequantisation scale of an fp8 V cache (1 for bf16)
  int prefetch_tiles;           // contiguous caches: tiles per CTA prefetched into L2 before
                                // the wait on the previous grid (0 = none)
  // Sparse decode (low-bit scan + top-delta) only:
  const int8_t* k8;             // [B, Hkv, max_len, D] int8 key codes
  const float* k8_scale;        // [B, Hkv, n_blocks] per 64-token block
  uint8_t* kept_out;            // [B, Hkv, n_blocks] 1 = block kept, or null
  int n_blocks;                 // ceil(max_len / 64)
  float scale;                  // softmax scale (natural-log domain)
  float delta;                  // top-delta threshold, natural-log units
};

// Longest split, in 64-token blocks, that the sparse scan handles, and the
// blocks one scan stage carries (one TMA box of 256 code rows).
constexpr int kMaxSparseTiles = 256;
constexpr int kScanTilesPerStage = 4;

// Token of row s (0..15) of the fp8 score MMA within a warp's 16-token slice:
// rows 2t, 2t+1 -> tokens 4t, 4t+1 and rows 8+2t, 8+2t+1 -> tokens 4t+2, 4t+3.
__host__ __device__ constexpr uint32_t perm16(uint32_t s) {
  return ((s & 7) >> 1) * 4 + (s >> 3) * 2 + (s & 1);
}

// Row of a warp's 16-row slice of the tile that holds the fp8 path's local
// token t: rows 8..15 swap in pairs (8 <-> 10, 9 <-> 11, 12 <-> 14,
// 13 <-> 15).  The eight rows of every 8-lane ldmatrix phase then sit in
// eight different 128-byte swizzle phases (row mod 8): for K the local tokens
// perm16(0..7) = 0, 1, 4, 5, 8, 9, 12, 13 (and perm16(8..15)), for V the
// local tokens 0..7 and 8..15.  Without the swap, rows r and r + 8 of one K
// phase shared a phase: one extra shared-memory wavefront per phase.  The
// attention sum does not depend on the order of its tokens, so only the
// addresses and the masks (which use the row) see the swap.
__host__ __device__ constexpr uint32_t rho16(uint32_t t) { return t ^ ((t >> 3) << 1); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float round_to_bf16(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

// Split s of S covers the tiles [floor(s T / S), floor((s + 1) T / S)) of
// every sequence: the splits differ by at most one tile, so any S up to T
// gives CTAs of balanced size.  With T = q S + r, floor(s T / S) =
// s q + floor(s r / S), and s r < S^2 <= 2^20 stays in 32 bits.
__device__ __forceinline__ int split_first_tile(const SplitArgs& a, int s) {
  return s * a.tile_q + static_cast<int>(static_cast<unsigned>(s * a.tile_r) /
                                         static_cast<unsigned>(a.n_splits));
}

// Splits that hold tokens of a sequence of n tokens: those whose first tile
// is below m = ceil(n / 64), i.e. ceil(m S / T) of them.
__device__ __forceinline__ int split_parts(const SplitArgs& a, int n) {
  const long long m = (n + kTile - 1) / kTile;
  if (m == 0) return 0;
  const long long p = (m * a.n_splits + a.tiles - 1) / a.tiles;
  return static_cast<int>(p < a.n_splits ? p : a.n_splits);
}

__device__ __forceinline__ int seq_length(const int32_t* seqlens, int b, int max_len) {
  int n = seqlens ? seqlens[b] : max_len;
  return n < 0 ? 0 : (n > max_len ? max_len : n);
}

__device__ __forceinline__ void raise_device_error(unsigned int code) {
  atomicOr(&g_error_word, code);
}

// Merge the n_parts partials of one (sequence, query head) row; one warp,
// lanes cover D.  Partial s of the row sits at po + s * o_stride (D floats)
// and pl[s * l_stride].  Partials written by other CTAs are read through L2
// (ld.global.cg).  The first 32 partials are requested together with the
// lse values, so a row with up to 32 of them (every fp8 call at S = 32
// included) costs one round trip.  They are summed in index order, so the
// result is deterministic and does not depend on the batch size.  A row whose
// partials are all empty (lse = -inf) gives 0 and -inf.  The result goes to
// orow (bf16) or, when orow_f32 is set, to orow_f32 (fp32).
template <int D>
__device__ __forceinline__ void combine_row(const float* po, const float* pl, int n_parts,
                                            size_t o_stride, size_t l_stride,
                                            __nv_bfloat16* orow, float* orow_f32,
                                            float* lse_out, int lane) {
  constexpr int VPL = D / 32;  // 4 or 2 values per lane
  constexpr int BATCH = 32;
  constexpr float kLog2e = 1.4426950408889634074f;
  const float* col = po + lane * VPL;
  float lb[BATCH], ob[BATCH][VPL];
  auto load_batch = [&](int s0) {
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      if (s0 + j < n_parts) {
        lb[j] = __ldcg(pl + (s0 + j) * l_stride);
        if constexpr (VPL == 4) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(col + (s0 + j) * o_stride));
          ob[j][0] = v.x; ob[j][1] = v.y; ob[j][2] = v.z; ob[j][3] = v.w;
        } else {
          const float2 v = __ldcg(reinterpret_cast<const float2*>(col + (s0 + j) * o_stride));
          ob[j][0] = v.x; ob[j][1] = v.y;
        }
      }
    }
  };
  load_batch(0);
  float mx = -INFINITY;
  if (n_parts <= BATCH) {  // every lane holds all the lse values already
#pragma unroll
    for (int j = 0; j < BATCH; ++j)
      if (j < n_parts) mx = fmaxf(mx, lb[j]);
  } else {
    for (int s = lane; s < n_parts; s += 32) mx = fmaxf(mx, __ldcg(pl + s * l_stride));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  float acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  float W = 0.f;
  if (mx != -INFINITY) {
    for (int s0 = 0; s0 < n_parts; s0 += BATCH) {
      if (s0 > 0) load_batch(s0);
#pragma unroll
      for (int j = 0; j < BATCH; ++j) {
        if (s0 + j < n_parts) {
          const float w = ex2((lb[j] - mx) * kLog2e);  // an empty partial weighs 0
          W += w;
#pragma unroll
          for (int i = 0; i < VPL; ++i) acc[i] += w * ob[j][i];
        }
      }
    }
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
  if (orow_f32) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) orow_f32[lane * VPL + i] = acc[i] * inv;
  } else if constexpr (VPL == 4) {
    uint2 pk;
    pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(orow + lane * VPL) = pk;
  } else {
    *reinterpret_cast<uint32_t*>(orow + lane * VPL) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (lse_out && lane == 0) *lse_out = mx == -INFINITY ? -INFINITY : mx + logf(W);
}

template <int D, int NB, int STAGES, bool FP8 = false, bool SPARSE = false,
          int CW = kConsumerWarps>
struct SplitSmem {
  // Rows are stored in 128-byte swizzle rows: a bf16 row of D = 128 takes two
  // (its column halves), an fp8 row of 128 takes one.
  static constexpr int kHalves = FP8 ? 1 : D / 64;
  static constexpr int kHalfBytes = kTile * 128;       // one 64-column half tile
  static constexpr int kTileBytes = kHalves * kHalfBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;   // K tile + V tile
  static constexpr int kBarOffset = STAGES * kStageBytes;
  // + error flag; sparse: + the kept-tile list (uint16) and its length, the
  // per-head thresholds and the block maxima [kMaxSparseTiles][NB * 8]
  static constexpr int kListOffset = kBarOffset + 2 * STAGES * 8 + 16;
  static constexpr int kCountOffset = kListOffset + 2 * kMaxSparseTiles;
  static constexpr int kThrOffset = kCountOffset + 16;
  static constexpr int kBmaxOffset = kThrOffset + 4 * NB * 8;
  static constexpr int kBytes =
      SPARSE ? kBmaxOffset + 4 * kMaxSparseTiles * NB * 8 : kListOffset;
  static constexpr int kDynamicBytes = kBytes + 1024;  // room to align to 1 KB
  // Epilogue scratch, laid over the drained pipeline buffers (floats):
  static constexpr int kNcol = NB * 8;
  // Rows of D floats padded by 4: the accumulator writes of lanes in
  // different column pairs then start in different banks.  (With two column
  // blocks the kernel is at its register cap and the padding's index
  // arithmetic spilled, so those rows stay unpadded.)
  static constexpr int kAccStride = NB == 1 ? D + 4 : D;
  static constexpr int kRedAcc = 0;                                   // [warp][col][kAccStride]
  static constexpr int kRedM = kRedAcc + CW * kNcol * kAccStride;     // [warp][col]
  static constexpr int kRedL = kRedM + CW * kNcol;                    // [warp][col]
  static constexpr int kScratchFloats = kRedL + CW * kNcol;
  static_assert(kScratchFloats * 4 <= kBarOffset, "epilogue scratch must fit the pipeline buffers");
};

// Sparse decode, selection ("Faster Than Flash: Exploiting Attention
// Sparsity for Efficient Long-Context Decoding", abstract: a scan of low-bit
// keys selects blocks by a top-delta rule that each unit of work applies on
// its own, with no global synchronisation).  The consumer warps' part of the
// scan: the int8 key codes of the split stream through the same mbarrier ring
// as the K/V tiles, kScanTilesPerStage blocks per stage; with CW consumer
// warps, warp w takes block w mod 4 of every (CW / 4)-th stage, starting at
// stage w / 4.  Per block and head the largest approximate logit
// ((scale * sq) * sk) * (q8 . k8) goes to bmax: the dot products are exact
// (int8 tensor cores, int32 accumulation), each product is rounded to fp32
// in that order, and q8 = rint(q / sq) with sq = max |q| / 127.
template <int D, int NB, int STAGES, int STAGE_BYTES, int CW>
__device__ __forceinline__ bool sparse_scan_consumer(const SplitArgs& a, uint32_t smem_base,
                                                     uint32_t bar_full, uint32_t bar_empty,
                                                     float* bmax, int warp, int lane, int b,
                                                     int h0, int start, int end, int n_tiles,
                                                     int n_scan) {
  static_assert(D == 128, "the scan reads 128-byte code rows");
  constexpr int KSTEPS = D / 32;
  static_assert(STAGE_BYTES >= kScanTilesPerStage * kTile * D, "a scan stage fits a ring stage");
  static_assert(kScanTilesPerStage == kTileWarps, "one block per warp of a set");
  constexpr int kSets = CW / kTileWarps;
  // B fragments of q8 (k = head dim, n = head): lane (g, t) holds entries
  // 32c + 4t .. +3 and 32c + 16 + 4t .. +3 of head nb*8 + g.
  uint32_t qb[NB][KSTEPS][2];
  float qsc[NB][2];     // scale * sq of this lane's two score columns
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int head = nb * 8 + (lane >> 2);
    const bool live = head < a.G;
    const __nv_bfloat16* qrow = a.q + (static_cast<size_t>(b) * a.Hq + h0 + (live ? head : 0)) * D;
    float v[KSTEPS][2][4];
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < KSTEPS; ++c)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint2 raw = live ? *reinterpret_cast<const uint2*>(qrow + 32 * c + 16 * h + 4 * (lane & 3))
                               : make_uint2(0u, 0u);
        const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        v[c][h][0] = f01.x;
        v[c][h][1] = f01.y;
        v[c][h][2] = f23.x;
        v[c][h][3] = f23.y;
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fabsf(v[c][h][i]));
      }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const float sq = amax > 0.f ? __fdiv_rn(amax, 127.f) : 1.f;
#pragma unroll
    for (int c = 0; c < KSTEPS; ++c)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int code = max(-127, min(127, __float2int_rn(__fdiv_rn(v[c][h][i], sq))));
          word |= (static_cast<uint32_t>(code) & 0xffu) << (8 * i);
        }
        qb[nb][c][h] = word;
      }
    const float qs = __fmul_rn(a.scale, sq);
    qsc[nb][0] = __shfl_sync(0xffffffffu, qs, 8 * (lane & 3));
    qsc[nb][1] = __shfl_sync(0xffffffffu, qs, 8 * (lane & 3) + 4);
  }

  const size_t srow = (static_cast<size_t>(b) * a.Hkv + (h0 / a.G)) * a.n_blocks + start / kTile;
  const int g = lane >> 2, t = lane & 3;
  for (int j = warp / kTileWarps; j < n_scan; j += kSets) {
    const int s = j % STAGES, k = j / STAGES;
    const bool ok = mbar_wait(bar_full + 8 * s, k & 1, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ok)) return false;
    const int blk = kScanTilesPerStage * j + warp % kTileWarps;
    if (blk < n_tiles) {
      const float sk = a.k8_scale[srow + blk];
      const uint32_t sb = smem_base + s * STAGE_BYTES;
      float mcol[NB][2];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) mcol[nb][0] = mcol[nb][1] = -INFINITY;
#pragma unroll
      for (int mg = 0; mg < kTile / 16; ++mg) {
        int acc[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[nb][i] = 0;
        const uint32_t row = (warp % kTileWarps) * kTile + mg * 16 + ((lane >> 3) & 1) * 8 +
                             (lane & 7);
#pragma unroll
        for (int kp = 0; kp < KSTEPS; ++kp) {
          const uint32_t chunk16 = 2 * kp + (lane >> 4);
          uint32_t r[4];
          ldmatrix_x4(sb + row * 128 + ((chunk16 ^ (row & 7)) << 4), r[0], r[1], r[2], r[3]);
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) mma_s8_16832(acc[nb], r, qb[nb][kp][0], qb[nb][kp][1]);
        }
        const int tok = start + blk * kTile + mg * 16 + g;   // C rows g and g + 8
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const bool valid = (i < 2 ? tok : tok + 8) < end;
            const float x = __fmul_rn(__fmul_rn(qsc[nb][i & 1], sk), __int2float_rn(acc[nb][i]));
            mcol[nb][i & 1] = fmaxf(mcol[nb][i & 1], valid ? x : -INFINITY);
          }
      }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int off = 4; off < 32; off <<= 1)
            mcol[nb][c] = fmaxf(mcol[nb][c], __shfl_xor_sync(0xffffffffu, mcol[nb][c], off));
          if (g == 0) bmax[blk * NB * 8 + nb * 8 + 2 * t + c] = mcol[nb][c];
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty + 8 * s);
  }
  return true;
}

// Consumer warps of the split kernel: scores, online softmax and P.V over the
// split's tiles, then the merge of the CW warps' softmax states into this
// split's result, which goes to `out` (the sequence has one split) or to the
// global partials (several splits).  Warp w takes tokens 16 (w mod 4) ..
// +15 of every (CW / 4)-th tile, starting at tile w / 4.
template <int D, int NB, int MODE, int STAGES, bool FP8, bool SPARSE, int CW = kConsumerWarps>
__device__ __forceinline__ void split_consumers(const SplitArgs& a, uint8_t* smem,
                                                uint32_t smem_base, uint32_t bar_full,
                                                uint32_t bar_empty, volatile int* cta_error,
                                                int warp, int lane, int b, int h0, int split,
                                                int start, int end, int n_tiles, int n_parts,
                                                const uint16_t* list, int it_base) {
  using L = SplitSmem<D, NB, STAGES, FP8, SPARSE, CW>;
  static_assert(CW % kTileWarps == 0, "whole sets of tile warps");
  constexpr int kSets = CW / kTileWarps;   // tiles in flight among the consumers
  // A set must see every phase of the stages it reads (a parity wait cannot
  // tell phase k from phase k - 2).  STAGES is a multiple of kSets, so the
  // tiles that share a stage (indices congruent modulo STAGES) belong to one
  // set.  Before the tiles, the sparse scan's stages (sets by stage index)
  // all complete ahead of a CTA-wide barrier, so a stage's first tile use
  // never waits behind another set's scan use.  Tiles go to sets by tile
  // index, which keeps the warp that sums each tile the same with or
  // without a scan in front.
  static_assert(STAGES % kSets == 0, "every stage belongs to one set of warps");
  const int wr = warp % kTileWarps;        // this warp's 16-token slice of a tile
  const int set = warp / kTileWarps;       // first tile of this warp
  constexpr int KSTEPS = D / 16;   // k-steps of the score MMA (over D)
  constexpr int DBLK = D / 16;     // m-blocks of the P.V MMA (over D)
  constexpr int NCOL = NB * 8;     // MMA columns (query heads, maybe doubled)
  static_assert(!FP8 || (D == 128 && MODE == kHi), "fp8 caches: D = 128, bf16-only P modes off");

  // B fragments of Q^T (k = head dim, n = query head), loaded once.
  uint32_t qf[NB][KSTEPS][2];
  if constexpr (FP8) {
    // f16 fragments, k order permuted to match the fp8 K fragments: k-step
    // c covers head-dim entries 16c..16c+15; slots 2t, 2t+1 hold 16c+4t,
    // 16c+4t+1 and slots 2t+8, 2t+9 hold 16c+4t+2, 16c+4t+3 (t = lane & 3).
    const int ncol = lane >> 2;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int head = nb * 8 + ncol;
      const bool live = head < a.G;
      const __nv_bfloat16* qrow = a.q + (static_cast<size_t>(b) * a.Hq + h0 + (live ? head : 0)) * D;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const uint2 raw = *reinterpret_cast<const uint2*>(qrow + ks * 16 + 4 * (lane & 3));
        const __nv_bfloat162 q01 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 q23 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        qf[nb][ks][0] = live ? pack_f16x2(__low2float(q01), __high2float(q01)) : 0u;
        qf[nb][ks][1] = live ? pack_f16x2(__low2float(q23), __high2float(q23)) : 0u;
      }
    }
  } else {
    const int ncol = lane >> 2;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int head = MODE == kDup ? (ncol & 3) : nb * 8 + ncol;
      const bool live = head < a.G;
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          a.q + (static_cast<size_t>(b) * a.Hq + h0 + (live ? head : 0)) * D);
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        qf[nb][ks][0] = live ? qrow[ks * 8 + (lane & 3)] : 0u;
        qf[nb][ks][1] = live ? qrow[ks * 8 + 4 + (lane & 3)] : 0u;
      }
    }
  }

  float m_run[NB][2], l_run[NB][2];
  float acc[NB][DBLK][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    m_run[nb][0] = m_run[nb][1] = -INFINITY;
    l_run[nb][0] = l_run[nb][1] = 0.f;
#pragma unroll
    for (int db = 0; db < DBLK; ++db)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nb][db][i] = 0.f;
  }

  // Row of the 16-token slice this lane addresses for ldmatrix, and its
  // 128-byte swizzle phase (row mod 8).  A tile is a stack of TMA boxes of
  // 2^log2_box_rows rows, each laid out [column half][row][128 bytes].
  //
  // FP8: row r of the score MMA is local token perm16(r), so that after the
  // P transpose the k-slots 2t, 2t+1 and 2t+8, 2t+9 of the P.V MMA are local
  // tokens 4t, 4t+1 and 4t+2, 4t+3: the order in which the byte-transposing
  // ldmatrix delivers V (see ldmatrix_x2_trans_b8).  Local token t sits in
  // row rho16(t) of the warp's slice.
  const uint32_t r16 = ((lane >> 3) & 1) * 8 + (lane & 7);
  const uint32_t rowK = wr * 16 + (FP8 ? rho16(perm16(r16)) : r16);
  const uint32_t rowV = wr * 16 + (FP8 ? rho16(lane & 15) : (lane >> 4) * 8 + (lane & 7));
  const uint32_t xv = rowV & 7;              // swizzle phases of the two rows
  const uint32_t xk = rowK & 7;
  const uint32_t lgr = a.log2_box_rows;
  const uint32_t half_bytes = 128u << lgr;                    // one column half of a box
  const uint32_t box_bytes = half_bytes * L::kHalves;
  const uint32_t offK = (rowK >> lgr) * box_bytes + (rowK & ((1u << lgr) - 1)) * 128;
  const uint32_t offV = (rowV >> lgr) * box_bytes + (rowV & ((1u << lgr) - 1)) * 128;
  // Token rows of the C fragment held by this lane.
  const int r_lo = wr * 16 + (FP8 ? rho16(perm16(lane >> 2)) : (lane >> 2));
  const int r_hi = wr * 16 + (FP8 ? rho16(perm16((lane >> 2) + 8)) : (lane >> 2) + 8);
  const float sl2 = a.scale_log2;
  bool failed = false;

  for (int it = set; it < n_tiles; it += kSets) {
    const int ig = it_base + it;                 // ring use, after any scan stages
    const int s = ig % STAGES, k = ig / STAGES;
    const bool ok = mbar_wait(bar_full + 8 * s, k & 1, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ok)) {
      failed = true;
      break;
    }
    const uint32_t kbase = smem_base + s * L::kStageBytes;
    const uint32_t vbase = kbase + L::kTileBytes;
    const int blk = SPARSE ? static_cast<int>(list[it]) : it;   // kept blocks only, in order
    const int tile_valid = min(kTile, end - (start + blk * kTile));
    const bool partial = tile_valid < kTile;

    // S^T = K Q^T for this warp's 16 tokens (two chains for ILP).
    float sc[NB][2][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[nb][c][i] = 0.f;
    if constexpr (FP8) {
      // One ldmatrix brings 16 bytes (16 head-dim entries) of 8 token rows
      // per matrix: tokens 0-7 and 8-15 of chunks 2kp and 2kp+1.  A lane's
      // register holds 4 consecutive entries of one token, converted to two
      // f16 pairs in the permuted k order of the q fragments.
#pragma unroll
      for (int kp = 0; kp < KSTEPS / 2; ++kp) {
        const uint32_t chunk16 = 2 * kp + (lane >> 4);
        const uint32_t addr = kbase + offK + ((chunk16 ^ xk) << 4);
        uint32_t r[4];
        ldmatrix_x4(addr, r[0], r[1], r[2], r[3]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int ks = 2 * kp + h;
          uint32_t af[4];
          af[0] = e4m3x2_to_f16x2(r[2 * h]);
          af[1] = e4m3x2_to_f16x2(r[2 * h + 1]);
          af[2] = e4m3x2_to_f16x2(r[2 * h] >> 16);
          af[3] = e4m3x2_to_f16x2(r[2 * h + 1] >> 16);
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) mma_f16_16816(sc[nb][ks & 1], af, qf[nb][ks][0], qf[nb][ks][1]);
        }
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const uint32_t chunk16 = ((ks & 3) << 1) + (lane >> 4);
        const uint32_t addr = kbase + offK + (ks >> 2) * half_bytes + ((chunk16 ^ xk) << 4);
        uint32_t af[4];
        ldmatrix_x4(addr, af[0], af[1], af[2], af[3]);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) mma_bf16_16816(sc[nb][ks & 1], af, qf[nb][ks][0], qf[nb][ks][1]);
      }
    }

    // Online softmax in the log2 domain; this lane holds tokens r_lo, r_hi
    // and columns 2*(lane&3), 2*(lane&3)+1.
    uint32_t pb[NB][2];
    uint32_t plo[NB][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      float t[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) t[i] = (sc[nb][0][i] + sc[nb][1][i]) * sl2;
      if (partial) {
        if (r_lo >= tile_valid) t[0] = t[1] = -INFINITY;
        if (r_hi >= tile_valid) t[2] = t[3] = -INFINITY;
      }
      float mx0 = fmaxf(t[0], t[2]), mx1 = fmaxf(t[1], t[3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m_run[nb][0], mx0), mn1 = fmaxf(m_run[nb][1], mx1);
      const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
      const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = ex2(m_run[nb][0] - mu0), al1 = ex2(m_run[nb][1] - mu1);
      const float p0 = ex2(t[0] - mu0), p1 = ex2(t[1] - mu1);
      const float p2 = ex2(t[2] - mu0), p3 = ex2(t[3] - mu1);
      l_run[nb][0] = l_run[nb][0] * al0 + (p0 + p2);
      l_run[nb][1] = l_run[nb][1] * al1 + (p1 + p3);
      m_run[nb][0] = mn0;
      m_run[nb][1] = mn1;
      if (__any_sync(0xffffffffu, (al0 != 1.f) | (al1 != 1.f))) {
#pragma unroll
        for (int db = 0; db < DBLK; ++db) {
          acc[nb][db][0] *= al0;
          acc[nb][db][1] *= al1;
          acc[nb][db][2] *= al0;
          acc[nb][db][3] *= al1;
        }
      }
      if constexpr (MODE == kDup) {
        // Columns 4..7 (lanes with lane&3 >= 2) carry the bf16 residual.
        const bool lo_lane = (lane & 2) != 0;
        const float e0 = lo_lane ? p0 - round_to_bf16(p0) : p0;
        const float e1 = lo_lane ? p1 - round_to_bf16(p1) : p1;
        const float e2 = lo_lane ? p2 - round_to_bf16(p2) : p2;
        const float e3 = lo_lane ? p3 - round_to_bf16(p3) : p3;
        pb[nb][0] = movmatrix_trans(pack_bf16x2(e0, e1));
        pb[nb][1] = movmatrix_trans(pack_bf16x2(e2, e3));
      } else if constexpr (FP8) {
        pb[nb][0] = movmatrix_trans(pack_f16x2(p0, p1));
        pb[nb][1] = movmatrix_trans(pack_f16x2(p2, p3));
      } else {
        pb[nb][0] = movmatrix_trans(pack_bf16x2(p0, p1));
        pb[nb][1] = movmatrix_trans(pack_bf16x2(p2, p3));
        if constexpr (MODE == kHiLo) {
          plo[nb][0] = movmatrix_trans(
              pack_bf16x2(p0 - round_to_bf16(p0), p1 - round_to_bf16(p1)));
          plo[nb][1] = movmatrix_trans(
              pack_bf16x2(p2 - round_to_bf16(p2), p3 - round_to_bf16(p3)));
        }
      }
    }

    // O^T += V^T P^T for this warp's 16 tokens.  Rows past the valid length
    // may hold anything (NaN included): on a partial tile their V values are
    // zeroed in registers so that 0 * NaN never reaches the accumulator.
    uint32_t vmask_lo = 0xffffffffu, vmask_hi = 0xffffffffu;
    if (partial) {
      if constexpr (FP8) {  // byte i of a register: local token 4t + i, in row rho16(4t + i)
        const int t4 = 4 * (lane & 3);
        const int base = wr * 16;
        vmask_lo = (base + static_cast<int>(rho16(t4)) < tile_valid ? 0xffu : 0u) |
                   (base + static_cast<int>(rho16(t4 + 1)) < tile_valid ? 0xff00u : 0u) |
                   (base + static_cast<int>(rho16(t4 + 2)) < tile_valid ? 0xff0000u : 0u) |
                   (base + static_cast<int>(rho16(t4 + 3)) < tile_valid ? 0xff000000u : 0u);
      } else {
        const int tk = wr * 16 + 2 * (lane & 3);
        vmask_lo = (tk < tile_valid ? 0x0000ffffu : 0u) | (tk + 1 < tile_valid ? 0xffff0000u : 0u);
        vmask_hi = (tk + 8 < tile_valid ? 0x0000ffffu : 0u) | (tk + 9 < tile_valid ? 0xffff0000u : 0u);
      }
    }
    if constexpr (FP8) {
      // The byte-transposing ldmatrix gives a lane, per 16-entry block,
      // tokens 4t .. 4t+3 of entries g and g + 8: exactly the A fragment
      // (rows g, g + 8; k-slots 2t, 2t+1 in the low halves, 2t+8, 2t+9 in the
      // high halves) after one conversion per half.
#pragma unroll
      for (int dp = 0; dp < DBLK / 2; ++dp) {
        const uint32_t chunk16 = 2 * dp + (lane >> 4);
        const uint32_t addr = vbase + offV + ((chunk16 ^ xv) << 4);
        uint32_t r[4];
        ldmatrix_x2_trans_b8(addr, r[0], r[1], r[2], r[3]);
        if (partial) {
#pragma unroll
          for (int i = 0; i < 4; ++i) r[i] &= vmask_lo;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int db = 2 * dp + h;
          uint32_t vf[4];
          vf[0] = e4m3x2_to_f16x2(r[2 * h]);
          vf[1] = e4m3x2_to_f16x2(r[2 * h + 1]);
          vf[2] = e4m3x2_to_f16x2(r[2 * h] >> 16);
          vf[3] = e4m3x2_to_f16x2(r[2 * h + 1] >> 16);
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) mma_f16_16816(acc[nb][db], vf, pb[nb][0], pb[nb][1]);
        }
      }
    } else {
#pragma unroll
    for (int db = 0; db < DBLK; ++db) {
      const uint32_t chunk16 = ((db & 3) << 1) + ((lane >> 3) & 1);
      const uint32_t addr = vbase + offV + (db >> 2) * half_bytes + ((chunk16 ^ xv) << 4);
      uint32_t vf[4];
      ldmatrix_x4_trans(addr, vf[0], vf[1], vf[2], vf[3]);
      if (partial) {
        vf[0] &= vmask_lo;
        vf[1] &= vmask_lo;
        vf[2] &= vmask_hi;
        vf[3] &= vmask_hi;
      }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        mma_bf16_16816(acc[nb][db], vf, pb[nb][0], pb[nb][1]);
        if constexpr (MODE == kHiLo) mma_bf16_16816(acc[nb][db], vf, plo[nb][0], plo[nb][1]);
      }
    }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty + 8 * s);
  }

  // The combine kernel (or the next call) may launch once every CTA is past
  // its tile loop: launched at the start it sat resident through the whole
  // split and measured 0.4-1.4 us slower per call.
  grid_dependents_launch();
  if (failed) {
    if (lane == 0) {
      raise_device_error(1u);
      *cta_error = 1;
    }
  }

  // Row sums: lanes sharing a column hold disjoint tokens.
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int off = 4; off < 32; off <<= 1)
        l_run[nb][j] += __shfl_xor_sync(0xffffffffu, l_run[nb][j], off);

  // Every consumer warp is past its last shared-memory read of the pipeline,
  // so the drained buffers hold the epilogue scratch: each warp's
  // accumulator [warp][col][D] and its running max and sum per column.
  named_barrier_sync(1, CW * 32);
  float* f = reinterpret_cast<float*>(smem);
  const bool live = !*cta_error;
  if (live) {
    const int j0 = 2 * (lane & 3);
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      float* base = f + L::kRedAcc + (warp * NCOL + nb * 8 + j0) * L::kAccStride;
      // Accumulator rows g and g + 8 of d-block db: head-dim entries
      // 16db + g and 16db + g + 8.
#pragma unroll
      for (int db = 0; db < DBLK; ++db) {
        const int d = db * 16 + (lane >> 2);
        base[d] = acc[nb][db][0];
        base[L::kAccStride + d] = acc[nb][db][1];
        base[d + 8] = acc[nb][db][2];
        base[L::kAccStride + d + 8] = acc[nb][db][3];
      }
      if (lane < 4) {
        f[L::kRedM + warp * NCOL + nb * 8 + j0] = m_run[nb][0];
        f[L::kRedM + warp * NCOL + nb * 8 + j0 + 1] = m_run[nb][1];
        f[L::kRedL + warp * NCOL + nb * 8 + j0] = l_run[nb][0];
        f[L::kRedL + warp * NCOL + nb * 8 + j0 + 1] = l_run[nb][1];
      }
    }
  }
  named_barrier_sync(1, CW * 32);
  if (!live) return;

  // One pass with no further barrier.  Each thread merges the CW warp
  // states for 4 * kParts head-dim entries of one head (4 at d0, and with
  // four consumer warps 4 more at d0 + D/2, so that a warp's 16-byte reads
  // and writes are contiguous) and computes that head's weights itself from a
  // few broadcast reads.  Eight consumer warps take 4 entries each, so that
  // all 256 threads share the merge of the G = 8 heads.  (A separate per-head
  // pass behind two more barriers took about 1.5 us per CTA.)
  constexpr int kParts = CW == kConsumerWarps ? 2 : 1;
  constexpr int kChunks = D / (4 * kParts);  // chunks of 4 * kParts entries per head
  const bool direct = n_parts == 1;
  for (int c = threadIdx.x; c < a.G * kChunks; c += CW * 32) {
    const int g = c / kChunks;
    const int d0 = (c - g * kChunks) * 4;
    float mw[CW];
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < CW; ++w) {
      mw[w] = f[L::kRedM + w * NCOL + g];
      M = fmaxf(M, mw[w]);
    }
    float wt[CW];
    float lse_s = -INFINITY;
    if (M == -INFINITY) {  // no token in this split
#pragma unroll
      for (int w = 0; w < CW; ++w) wt[w] = 0.f;
    } else {
      float Ls = 0.f;
#pragma unroll
      for (int w = 0; w < CW; ++w) {
        wt[w] = ex2(mw[w] - M);
        Ls += wt[w] * f[L::kRedL + w * NCOL + g];
      }
      const float inv = a.v_scale / Ls;  // an fp8 V cache is dequantised here
#pragma unroll
      for (int w = 0; w < CW; ++w) wt[w] *= inv;
      lse_s = (M + log2f(Ls)) * 0.69314718055994530942f;
    }
    float4 o[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
#pragma unroll
    for (int w = 0; w < CW; ++w) {
      const float* src = f + L::kRedAcc + (w * NCOL + g) * L::kAccStride + d0;
#pragma unroll
      for (int h = 0; h < kParts; ++h) {
        float4 v = *reinterpret_cast<const float4*>(src + h * (D / 2));
        if constexpr (MODE == kDup) {  // columns g + 4 hold the bf16 residuals
          const float4 r = *reinterpret_cast<const float4*>(src + 4 * L::kAccStride + h * (D / 2));
          v.x += r.x;
          v.y += r.y;
          v.z += r.z;
          v.w += r.w;
        }
        o[h].x += wt[w] * v.x;
        o[h].y += wt[w] * v.y;
        o[h].z += wt[w] * v.z;
        o[h].w += wt[w] * v.w;
      }
    }
    const size_t row = static_cast<size_t>(b) * a.Hq + h0 + g;
    if (direct) {
      if (a.out_f32) {
        float* dst = a.out_f32 + row * D + d0;
#pragma unroll
        for (int h = 0; h < kParts; ++h) *reinterpret_cast<float4*>(dst + h * (D / 2)) = o[h];
      } else {
        __nv_bfloat16* dst = a.out + row * D + d0;
#pragma unroll
        for (int h = 0; h < kParts; ++h)
          *reinterpret_cast<uint2*>(dst + h * (D / 2)) =
              make_uint2(pack_bf16x2(o[h].x, o[h].y), pack_bf16x2(o[h].z, o[h].w));
      }
      if (d0 == 0 && a.lse) a.lse[row] = lse_s;
    } else {
      float* dst = a.part_o + (row * a.n_splits + split) * D + d0;
#pragma unroll
      for (int h = 0; h < kParts; ++h) *reinterpret_cast<float4*>(dst + h * (D / 2)) = o[h];
      if (d0 == 0) a.part_lse[row * a.n_splits + split] = lse_s;
    }
  }
}

// Split kernel: one CTA per (split, KV head, sequence).  FP8: the cache
// holds e4m3 values (D = 128); the contraction runs on f16 tensor cores.
// CW consumer warps and one producer warp; kWideConsumerWarps for a CTA
// that has its SM to itself.
template <int D, int NB, int MODE, bool PAGED, int STAGES, bool FP8, bool SPARSE = false,
          int CW = kConsumerWarps>
__global__ void __launch_bounds__(split_threads<CW>(), CW == kConsumerWarps ? kCtasPerSm : 1)
    fd_split_kernel(const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmC,   // sparse: int8 key codes
                    const SplitArgs a) {
  using L = SplitSmem<D, NB, STAGES, FP8, SPARSE, CW>;
  static_assert(!SPARSE || (!PAGED && !FP8), "sparse decode: contiguous bf16 caches");
  static_assert(MODE != kDup || NB == 1, "duplicated columns need one column block");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_full = smem_base + L::kBarOffset;
  const uint32_t bar_empty = bar_full + STAGES * 8;
  volatile int* cta_error = reinterpret_cast<volatile int*>(smem + L::kBarOffset + 2 * STAGES * 8);

  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, kTileWarps);   // the four warps that read a tile
    }
    *cta_error = 0;
    fence_mbar_init();
  }
  if (warp == CW && lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  if constexpr (!PAGED) {
    // While the previous grid finishes, pull the first tiles of this split
    // into L2, one tile per lane.  Only kernel arguments are used (the
    // lengths may still be in flight), so the range stops at max_len.
    if (warp == CW && lane < a.prefetch_tiles) {
      const int tile0 = split_first_tile(a, split);
      const int t0 = (tile0 + lane) * kTile;
      if (tile0 + lane < split_first_tile(a, split + 1) && t0 < a.max_len) {
        tma_prefetch_l2_5d(&tmK, 0, kvh, t0, 0, b);
        tma_prefetch_l2_5d(&tmV, 0, kvh, t0, 0, b);
      }
    }
  }
  __syncthreads();

  // Inputs may be produced by the previous kernel on the stream.
  grid_dependency_wait();

  const int n = seq_length(a.seqlens, b, a.max_len);
  const int start = split_first_tile(a, split) * kTile;
  const int end = min(split_first_tile(a, split + 1) * kTile, n);
  const int h0 = kvh * a.G;
  const int n_tiles = start < end ? (end - start + kTile - 1) / kTile : 0;
  // Splits of this sequence that hold tokens.
  // Whether the sequence has tokens in other splits than split 0 (then this
  // split's result is a partial for the combine kernel): 1 = only split 0,
  // 2 = several.  Split 0 holds tiles [0, tile_q).
  const int n_parts = (a.n_splits == 1 || (n + kTile - 1) / kTile <= a.tile_q) ? 1 : 2;

  if (n_tiles == 0) {
    // Empty split.  Split 0 is empty only for an empty sequence, whose
    // result is out = 0, lse = -inf; other empty splits take no part.
    if (split == 0) {
      const size_t base = (static_cast<size_t>(b) * a.Hq + h0) * D;
      for (int i = threadIdx.x; i < a.G * D; i += split_threads<CW>()) {
        if (a.out_f32)
          a.out_f32[base + i] = 0.f;
        else
          a.out[base + i] = __float2bfloat16_rn(0.f);
      }
      if (a.lse && threadIdx.x < a.G) a.lse[static_cast<size_t>(b) * a.Hq + h0 + threadIdx.x] = -INFINITY;
    }
    return;
  }

  // Tiles the pipeline runs: all of the split's, or the kept ones in order,
  // after it_base ring uses by the sparse scan.
  int n_work = n_tiles;
  int it_base = 0;
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + L::kListOffset);
  if constexpr (SPARSE) {
    const int n_scan = (n_tiles + kScanTilesPerStage - 1) / kScanTilesPerStage;
    float* bmax = reinterpret_cast<float*>(smem + L::kBmaxOffset);
    float* thr = reinterpret_cast<float*>(smem + L::kThrOffset);
    int* count = reinterpret_cast<int*>(smem + L::kCountOffset);
    bool ok = true;
    if (warp == CW) {
      // Producer: one TMA box of kScanTilesPerStage blocks of codes per stage.
      const uint64_t policy = policy_evict_first();
      for (int j = 0; j < n_scan; ++j) {
        const int s = j % STAGES, k = j / STAGES;
        if (k > 0) ok = mbar_wait(bar_empty + 8 * s, (k - 1) & 1, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_full + 8 * s, kScanTilesPerStage * kTile * D);
          tma_load_5d(smem_base + s * L::kStageBytes, &tmC, bar_full + 8 * s, 0, kvh,
                      start + j * kScanTilesPerStage * kTile, 0, b, policy);
        }
        __syncwarp();
      }
      if (!ok && lane == 0) {  // no code copy may still be landing when the CTA retires
        for (int j = n_scan > STAGES ? n_scan - STAGES : 0; j < n_scan; ++j)
          if (!mbar_wait(bar_full + 8 * (j % STAGES), (j / STAGES) & 1, kWaitLimitNs))
            raise_device_error(2u);
      }
    } else {
      ok = sparse_scan_consumer<D, NB, STAGES, L::kStageBytes, CW>(a, smem_base, bar_full, bar_empty,
                                                             bmax, warp, lane, b, h0, start, end,
                                                             n_tiles, n_scan);
    }
    if (!ok && lane == 0) {
      raise_device_error(1u);
      *cta_error = 1;
    }
    __syncthreads();
    if (*cta_error) return;
    // Per head: M = the split's largest block maximum; the threshold M - delta.
    if (threadIdx.x < a.G) {
      float M = -INFINITY;
      for (int i = 0; i < n_tiles; ++i) M = fmaxf(M, bmax[i * NB * 8 + threadIdx.x]);
      thr[threadIdx.x] = __fsub_rn(M, a.delta);
    }
    __syncthreads();
    // Kept blocks in order: some head's block maximum reaches its threshold.
    if (warp == 0) {
      const size_t srow = (static_cast<size_t>(b) * a.Hkv + kvh) * a.n_blocks + start / kTile;
      int kept = 0;
      for (int i0 = 0; i0 < n_tiles; i0 += 32) {
        const int i = i0 + lane;
        bool keep = false;
        if (i < n_tiles) {
          for (int g = 0; g < a.G; ++g) keep |= bmax[i * NB * 8 + g] >= thr[g];
          if (a.kept_out) a.kept_out[srow + i] = keep ? 1 : 0;
        }
        const unsigned mask = __ballot_sync(0xffffffffu, keep);
        if (keep) list[kept + __popc(mask & ((1u << lane) - 1u))] = static_cast<uint16_t>(i);
        kept += __popc(mask);
      }
      if (lane == 0) *count = kept;
    }
    __syncthreads();
    n_work = *count;
    it_base = n_scan;
  }

  if (warp == CW) {
    // ------------------------------------------------------------- producer
    // Every lane waits (the decision is made warp-uniform); lane 0 issues.
    const uint64_t policy = policy_evict_first();
    int issued = it_base;   // ring uses so far (the sparse scan's stages)
    bool ok = true;
    if constexpr (!PAGED) {
      for (int it = 0; it < n_work; ++it) {
        const int ig = it_base + it;
        const int s = ig % STAGES, k = ig / STAGES;
        if (k > 0) ok = mbar_wait(bar_empty + 8 * s, (k - 1) & 1, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        if (lane == 0) {
          const int t0 = start + (SPARSE ? static_cast<int>(list[it]) : it) * kTile;
          const uint32_t dk = smem_base + s * L::kStageBytes;
          const uint32_t dv = dk + L::kTileBytes;
          mbar_arrive_expect_tx(bar_full + 8 * s, L::kStageBytes);
          tma_load_5d(dk, &tmK, bar_full + 8 * s, 0, kvh, t0, 0, b, policy);
          tma_load_5d(dv, &tmV, bar_full + 8 * s, 0, kvh, t0, 0, b, policy);
        }
        ++issued;
        __syncwarp();
      }
    } else {
      const int bs = a.block_size, lbs = a.log2_block_size;
      const int rows = bs < kTile ? bs : kTile;            // rows per TMA box
      const int pages_per_tile = bs < kTile ? kTile / bs : 1;
      const int n_pages = (n + bs - 1) >> lbs;
      const int32_t* bt = a.block_table + static_cast<size_t>(b) * a.max_blocks_per_seq;
      // A window of 32 page ids, one per lane, plus the next window in flight.
      int win = start >> lbs;
      int cur = (win + lane < n_pages) ? __ldg(bt + win + lane) : 0;
      int nxt = (win + 32 + lane < n_pages) ? __ldg(bt + win + 32 + lane) : 0;
      for (int it = 0; it < n_work; ++it) {
        const int s = it % STAGES, k = it / STAGES;
        if (k > 0) ok = mbar_wait(bar_empty + 8 * s, (k - 1) & 1, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        const int t0 = start + it * kTile;
        const int pg = t0 >> lbs;
        if (pg >= win + 32) {
          win += 32;
          cur = nxt;
          nxt = (win + 32 + lane < n_pages) ? __ldg(bt + win + 32 + lane) : 0;
        }
        const int row0 = bs > kTile ? (t0 & (bs - 1)) : 0;
        const int valid_pages = min(pages_per_tile, n_pages - pg);
        const uint32_t dk = smem_base + s * L::kStageBytes;
        const uint32_t dv = dk + L::kTileBytes;
        int pid[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) pid[j] = __shfl_sync(0xffffffffu, cur, (pg - win + j) & 31);
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_full + 8 * s,
                                valid_pages * rows * 128 * L::kHalves * 2);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j < valid_pages) {
              // page j of the tile: both column halves of `rows` rows
              const uint32_t off = j * rows * 128 * L::kHalves;
              tma_load_5d(dk + off, &tmK, bar_full + 8 * s, 0, kvh, row0, 0, pid[j], policy);
              tma_load_5d(dv + off, &tmV, bar_full + 8 * s, 0, kvh, row0, 0, pid[j], policy);
            }
          }
        }
        ++issued;
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {
      raise_device_error(1u);
      *cta_error = 1;
    }
    // No copy may still be landing in shared memory when the CTA retires.
    if (lane == 0) {
      for (int it = issued > STAGES ? issued - STAGES : 0; it < issued; ++it)
        if (!mbar_wait(bar_full + 8 * (it % STAGES), (it / STAGES) & 1, kWaitLimitNs))
          raise_device_error(2u);
    }
  } else {
    // ------------------------------------------------------------- consumers
    split_consumers<D, NB, MODE, STAGES, FP8, SPARSE, CW>(a, smem, smem_base, bar_full, bar_empty,
                                                      cta_error, warp, lane, b, h0, split,
                                                      start, end, n_work, n_parts, list,
                                                      it_base);
  }
}

template <int D>
__global__ void __launch_bounds__(kCombineWarps * 32) fd_combine_kernel(const SplitArgs a, int B) {
  const int row = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  // The lengths may be read before the wait: the split kernel, the grid this
  // one depends on, does not write them, and this grid launches only after
  // every split CTA passed its own wait, i.e. after all earlier writes to
  // them completed.  Read through L2 (coherent), not L1.
  int n_parts = 0;
  if (row < B * a.Hq) {
    int n = a.seqlens ? __ldcg(a.seqlens + row / a.Hq) : a.max_len;
    n = n < 0 ? 0 : (n > a.max_len ? a.max_len : n);
    n_parts = split_parts(a, n);
  }
  grid_dependency_wait();     // partials come from the split kernel
  // The next call's split kernel may now start its prologue, which pulls its
  // first tiles into L2 while this kernel merges.  (Triggering before the
  // wait lets it become resident while the split kernel still streams; its
  // prefetched tiles then sit in L2 for the whole split and were measured to
  // be evicted and read twice at 16K tokens.)
  grid_dependents_launch();
  if (row >= B * a.Hq) return;
  if (n_parts <= 1) return;
  combine_row<D>(a.part_o + static_cast<size_t>(row) * a.n_splits * D,
                 a.part_lse + static_cast<size_t>(row) * a.n_splits, n_parts, D, 1,
                 a.out_f32 ? nullptr : a.out + static_cast<size_t>(row) * D,
                 a.out_f32 ? a.out_f32 + static_cast<size_t>(row) * D : nullptr,
                 a.lse ? a.lse + row : nullptr, lane);
}

// Merge of R partial results: partial r of row i is the D floats at
// part_o + r * o_stride + i * D and the lse at part_lse[r * l_stride + i]
// ([R][rows][D] and [R][rows] when the strides are rows * D and rows; one
// packed buffer per part when both strides are the part's size).  One warp
// per row.
template <int D>
__global__ void __launch_bounds__(kCombineWarps * 32) fd_merge_kernel(const float* part_o, const float* part_lse,
                                                       int R, int rows, size_t o_stride,
                                                       size_t l_stride, __nv_bfloat16* out,
                                                       float* lse) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int row = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  combine_row<D>(part_o + static_cast<size_t>(row) * D, part_lse + row, R, o_stride, l_stride,
                 out + static_cast<size_t>(row) * D, nullptr, lse ? lse + row : nullptr, lane);
}

// Low-bit key codes for the sparse decode: one CTA of 128 threads per
// (64-token block, KV head, sequence) of a contiguous head-major bf16 cache.
// sk = max |K| over the block's valid rows / 127 (1 for an all-zero block) and
// k8 = rint(K / sk), in [-127, 127]; rows at or past the sequence's length get
// k8 = 0 and take no part in sk.
template <int D>
__global__ void __launch_bounds__(128)
    fd_quantize_keys_kernel(const __nv_bfloat16* k, const int32_t* seqlens, int Hkv, int max_len,
                            int n_blocks, int8_t* k8, float* k8_scale) {
  grid_dependency_wait();
  grid_dependents_launch();
  constexpr int PER = kTile * D / 128;      // entries per thread: half a row
  __shared__ float red[4];
  const int blk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int n = seq_length(seqlens, b, max_len);
  const int row = blk * kTile + threadIdx.x / 2;
  const int col = (threadIdx.x & 1) * PER;
  const size_t base = ((static_cast<size_t>(b) * Hkv + kvh) * max_len + row) * D + col;
  float v[PER];
  float amax = 0.f;
  if (row < n) {
#pragma unroll
    for (int w = 0; w < PER / 8; ++w) {
      const uint4 raw = *reinterpret_cast<const uint4*>(k + base + 8 * w);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h[j]);
        v[8 * w + 2 * j] = f.x;
        v[8 * w + 2 * j + 1] = f.y;
      }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(v[i]));
  } else {
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = 0.f;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float sk = amax > 0.f ? __fdiv_rn(amax, 127.f) : 1.f;
  if (threadIdx.x == 0) k8_scale[(static_cast<size_t>(b) * Hkv + kvh) * n_blocks + blk] = sk;
  if (row >= max_len) return;
#pragma unroll
  for (int w = 0; w < PER / 16; ++w) {
    uint32_t word[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t x = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = max(-127, min(127, __float2int_rn(__fdiv_rn(v[16 * w + 4 * j + e], sk))));
        x |= (static_cast<uint32_t>(c) & 0xffu) << (8 * e);
      }
      word[j] = x;
    }
    *reinterpret_cast<uint4*>(k8 + base + 16 * w) = make_uint4(word[0], word[1], word[2], word[3]);
  }
}

// Diagnostic: waits, with the kernels' bounded wait, on an mbarrier that
// nothing ever arrives on, and reports the timeout through the device error
// word as the split kernel would.  Nothing faults and nothing hangs.
__global__ void fd_wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(smem_u32(&bar), 0, limit_ns);
  if (!__all_sync(0xffffffffu, ok) && threadIdx.x == 0) raise_device_error(4u);
}

}  // namespace fd
