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
#include <cuda_fp8.h>
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
// The last step of a split: merge the CW consumer warps' states (running
// maximum and sum per head in log2 units, unnormalised accumulator rows),
// which the warps left in shared memory at L::kRedM, L::kRedL and
// L::kRedAcc, into the split's partial output and log-sum-exp (or the final
// result when the sequence has a single split).
template <int D, int NB, int MODE, int CW, class L>
__device__ __forceinline__ void split_merge(const SplitArgs& a, const float* f, int b, int h0,
                                            int split, int n_parts) {
  constexpr int NCOL = L::kNcol;
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

  split_merge<D, NB, MODE, CW, L>(a, f, b, h0, split, n_parts);
}

// The producer warp of a split CTA: streams the split's K/V tiles (or the
// listed ones) into the ring, one stage per tile, after it_base earlier ring
// uses.  Stage s holds its K tile at s * STAGE_STRIDE and its V tile
// V_OFFSET bytes further.  Contiguous caches take one TMA box per tensor and tile; paged caches
// one box per page, the page ids read from the block table 32 at a time.
// Every lane waits (the decision is made warp-uniform); lane 0 issues.
// Before returning it waits until no copy is still landing in shared memory.
template <bool PAGED, bool SPARSE, int STAGES, int STAGE_STRIDE, int V_OFFSET, int HALVES>
__device__ __forceinline__ void split_producer(const SplitArgs& a, const CUtensorMap* tmK,
                                               const CUtensorMap* tmV, uint32_t smem_base,
                                               uint32_t bar_full, uint32_t bar_empty,
                                               volatile int* cta_error, int lane, int b, int kvh,
                                               int start, int n, int n_work, int it_base,
                                               const uint16_t* list) {
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
        const uint32_t dk = smem_base + s * STAGE_STRIDE;
        const uint32_t dv = dk + V_OFFSET;
        mbar_arrive_expect_tx(bar_full + 8 * s, 2 * kTile * 128 * HALVES);
        tma_load_5d(dk, tmK, bar_full + 8 * s, 0, kvh, t0, 0, b, policy);
        tma_load_5d(dv, tmV, bar_full + 8 * s, 0, kvh, t0, 0, b, policy);
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
      const uint32_t dk = smem_base + s * STAGE_STRIDE;
      const uint32_t dv = dk + V_OFFSET;
      int pid[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) pid[j] = __shfl_sync(0xffffffffu, cur, (pg - win + j) & 31);
      if (lane == 0) {
        mbar_arrive_expect_tx(bar_full + 8 * s,
                              valid_pages * rows * 128 * HALVES * 2);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < valid_pages) {
            // page j of the tile: both column halves of `rows` rows
            const uint32_t off = j * rows * 128 * HALVES;
            tma_load_5d(dk + off, tmK, bar_full + 8 * s, 0, kvh, row0, 0, pid[j], policy);
            tma_load_5d(dv + off, tmV, bar_full + 8 * s, 0, kvh, row0, 0, pid[j], policy);
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
    split_producer<PAGED, SPARSE, STAGES, L::kStageBytes, L::kTileBytes, L::kHalves>(
        a, &tmK, &tmV, smem_base, bar_full, bar_empty, cta_error, lane, b, kvh, start, n,
        n_work, it_base, list);
  } else {
    // ------------------------------------------------------------- consumers
    split_consumers<D, NB, MODE, STAGES, FP8, SPARSE, CW>(a, smem, smem_base, bar_full, bar_empty,
                                                      cta_error, warp, lane, b, h0, split,
                                                      start, end, n_work, n_parts, list,
                                                      it_base);
  }
}

// ---------------------------------------------------------------------------
// fp8 split kernel on the fifth-generation tensor cores (tcgen05).
//
// Same work split, producer and merge as fd_split_kernel with an fp8 cache,
// but the two contractions are kind::f8f6f4 MMAs that read the e4m3 K and V
// tiles straight from the TMA-swizzled ring: no code is converted in
// registers.  Tensor memory keeps the accumulator rows of warp j of a
// warpgroup in lanes 32j .. 32j+31, the lanes that warp may read.
//
// A tcgen05 MMA costs its issuing thread about the same time whatever its
// size when it is this small, so the scores are taken four tiles at a time:
// the ring keeps its K tiles apart from its V tiles, four consecutive K
// tiles are one 256-row operand, and
//  S = Q K^T  (M = 64, N = 256 tokens, K = 128; rows 16j .. 16j+15 in lanes
//    32j .. 32j+15): the A rows 16j + r of every j hold the same 2G rows of
//    q as e4m3 pairs, so warp j reads the scores of tokens 16j .. 16j+15 of
//    each tile for all heads from its own lanes.  The warps copy their two
//    tiles' scores to registers first, which frees S for the next four.
//  O += P V  (M = 128, N = 128 = D, K = 64 tokens; row i in lane i): warp
//    j's 3G rows 32j + r of P are non-zero only in its own 16 tokens, so
//    rows 32j .. 32j+31 of O sum that warp's tokens alone, under that warp's
//    running maximum.
//
// A bf16 value x is split exactly into two e4m3 codes, x sigma = x1 + x2 / 16
// (sigma a power of two that brings max |x| to [128, 256)); q rows r < G hold
// x1 of head r and rows G + r hold x2.  The softmax weights p <= 2^8 take
// three codes, p = p1 + p2 / 16 + p3 / 256 (12 significant bits, like an f16
// weight; two codes, 8 bits, moved the log-sum-exp of a dominant token by up
// to 2^-8), in P rows r, G + r and 2G + r, and the running sum adds the
// split values, so O and l see the same weights.
// A warp rescales its O rows only when its maximum grows by more than 2^8;
// until then the weights stay relative to the older maximum.
//
// Warps: 0-7 softmax (two warpgroups that take alternate tiles, each with
// its own O in tensor memory), 8 the TMA producer, 9 the MMA issuer.
constexpr int kTcSoftmaxWarps = 8;
constexpr int kTcProducerWarp = kTcSoftmaxWarps;
constexpr int kTcMmaWarp = kTcSoftmaxWarps + 1;
constexpr int kTcThreads = (kTcSoftmaxWarps + 2) * 32;
constexpr int kTcMaxG = 8;                   // 3G rows of P per warp, at most 32
constexpr int kTcQuad = 4;                   // tiles per score MMA
constexpr uint32_t kTcCols = 512;            // TMEM columns: S of four tiles at 0 (256),
constexpr uint32_t kTcOCol = 256;            // O of warpgroup g at 256 + 128 g
constexpr float kTcRescaleLog2 = 8.f;        // weights up to 2^8 before a rescale

template <int STAGES>
struct TcSmem {
  static_assert(STAGES % kTcQuad == 0, "four consecutive K tiles are contiguous");
  static constexpr int kTileBytes = kTile * 128;          // 64 token rows of 128 codes
  static constexpr int kHalves = 1;
  static constexpr int kKRing = 0;                        // STAGES K tiles
  static constexpr int kVRing = STAGES * kTileBytes;      // STAGES V tiles
  static constexpr int kQOffset = 2 * STAGES * kTileBytes;  // 64 x 128 e4m3, 128-byte swizzle
  static constexpr int kPOffset = kQOffset + 64 * 128;    // two 128 x 64 e4m3, 8x16-byte cores
  static constexpr int kPBytes = 128 * 64;
  static constexpr int kBarOffset = kPOffset + 2 * kPBytes;
  static constexpr int kSFull = kBarOffset + 2 * STAGES * 8;  // scores of a quad ready
  static constexpr int kSFree = kSFull + 8;                   // scores of a quad copied out
  static constexpr int kPFull = kSFree + 8;                   // per warpgroup: P written
  static constexpr int kODone = kPFull + 16;                  // per warpgroup: P.V done
  static constexpr int kMmaDone = kODone + 16;                // every MMA done
  static constexpr int kTmemSlot = kMmaDone + 8;
  static constexpr int kErrorOffset = kTmemSlot + 4;
  static constexpr int kQExpOffset = kErrorOffset + 4;        // int per head
  static constexpr int kBytes = kQExpOffset + 4 * kTcMaxG;
  static constexpr int kDynamicBytes = kBytes + 1024;         // room to align to 1 KB
  // Epilogue scratch over the drained ring, in the layout split_merge reads.
  static constexpr int kNcol = 8;
  static constexpr int kAccStride = 128 + 4;
  static constexpr int kRedAcc = 0;
  static constexpr int kRedM = kRedAcc + kTcSoftmaxWarps * kNcol * kAccStride;
  static constexpr int kRedL = kRedM + kTcSoftmaxWarps * kNcol;
  static constexpr int kScratchFloats = kRedL + kTcSoftmaxWarps * kNcol;
  static_assert(kScratchFloats * 4 <= kQOffset, "epilogue scratch must fit the ring");
  static_assert(kDynamicBytes <= 227 * 1024, "shared memory per CTA");
};

// Byte offset of (row, byte k) in the 128 x 64 P operand: 8-row x 16-byte core
// matrices, 128 bytes apart along k and 512 bytes apart along the rows.
__device__ __forceinline__ uint32_t tc_p_offset(uint32_t row, uint32_t k) {
  return (row >> 3) * 512 + (k >> 4) * 128 + (row & 7) * 16 + (k & 15);
}

// Two floats to an e4m3 pair (round to nearest even, saturating), x in the
// low byte, and the values it holds.
__device__ __forceinline__ uint32_t tc_e4m3x2(float x, float y, float& xq, float& yq) {
  const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(make_float2(x, y), __NV_SATFINITE, __NV_E4M3);
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(c, __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  xq = f.x;
  yq = f.y;
  return static_cast<uint32_t>(c);
}

template <bool PAGED, int STAGES, int G>
__global__ void __launch_bounds__(kTcThreads, 1)
    fd_split_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const SplitArgs a) {
  using L = TcSmem<STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_full = smem_base + L::kBarOffset;
  const uint32_t bar_empty = bar_full + STAGES * 8;
  const uint32_t s_full = smem_base + L::kSFull;
  const uint32_t s_free = smem_base + L::kSFree;
  const uint32_t p_full = smem_base + L::kPFull;
  const uint32_t o_done = smem_base + L::kODone;
  const uint32_t mma_done = smem_base + L::kMmaDone;
  volatile int* cta_error = reinterpret_cast<volatile int*>(smem + L::kErrorOffset);
  int* qexp = reinterpret_cast<int*>(smem + L::kQExpOffset);

  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);   // released by the commit of the tile's P.V
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kTcSoftmaxWarps);
    for (int g = 0; g < 2; ++g) {
      mbar_init(p_full + 8 * g, 4);      // the four warps of the warpgroup
      mbar_init(o_done + 8 * g, 1);
    }
    mbar_init(mma_done, 1);
    *cta_error = 0;
    fence_mbar_init();
  }
  if (warp == kTcProducerWarp && lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  if constexpr (!PAGED) {
    if (warp == kTcProducerWarp && lane < a.prefetch_tiles) {
      const int tile0 = split_first_tile(a, split);
      const int t0 = (tile0 + lane) * kTile;
      if (tile0 + lane < split_first_tile(a, split + 1) && t0 < a.max_len) {
        tma_prefetch_l2_5d(&tmK, 0, kvh, t0, 0, b);
        tma_prefetch_l2_5d(&tmV, 0, kvh, t0, 0, b);
      }
    }
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(smem_base + L::kTmemSlot, kTcCols);
    tmem_relinquish();
  }
  tcgen05_fence_before();
  __syncthreads();
  tcgen05_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlot);

  grid_dependency_wait();

  const int n = seq_length(a.seqlens, b, a.max_len);
  const int start = split_first_tile(a, split) * kTile;
  const int end = min(split_first_tile(a, split + 1) * kTile, n);
  static_assert(G == 2 || G == 4 || G == 8, "group sizes of the tcgen05 kernel");
  const int h0 = kvh * G;
  const int n_tiles = start < end ? (end - start + kTile - 1) / kTile : 0;
  const int n_quads = (n_tiles + kTcQuad - 1) / kTcQuad;
  const int n_parts = (a.n_splits == 1 || (n + kTile - 1) / kTile <= a.tile_q) ? 1 : 2;

  if (n_tiles == 0) {
    if (split == 0) {  // an empty sequence: out = 0, lse = -inf
      const size_t base = (static_cast<size_t>(b) * a.Hq + h0) * 128;
      for (int i = threadIdx.x; i < G * 128; i += kTcThreads) {
        if (a.out_f32)
          a.out_f32[base + i] = 0.f;
        else
          a.out[base + i] = __float2bfloat16_rn(0.f);
      }
      if (a.lse && threadIdx.x < G) a.lse[static_cast<size_t>(b) * a.Hq + h0 + threadIdx.x] = -INFINITY;
    }
  } else {
    if (warp < kTcSoftmaxWarps) {
      // Zero the q and P operands (24 KB: 96 bytes per thread) ...
      uint4* z = reinterpret_cast<uint4*>(smem + L::kQOffset);
#pragma unroll
      for (int i = 0; i < 6; ++i) z[threadIdx.x * 6 + i] = make_uint4(0u, 0u, 0u, 0u);
      named_barrier_sync(1, kTcSoftmaxWarps * 32);
      // ... then warp g < G writes head g's pair into rows 16j + g and
      // 16j + G + g of every j; lane l holds head-dim entries 4l .. 4l+3.
      const int g = warp;
      if (g < G) {
        const uint2 raw = *reinterpret_cast<const uint2*>(
            a.q + (static_cast<size_t>(b) * a.Hq + h0 + g) * 128 + 4 * lane);
        const __nv_bfloat162 q01 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 q23 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        float x[4] = {__low2float(q01), __high2float(q01), __low2float(q23), __high2float(q23)};
        float mx = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        int e = 0;
        frexpf(mx, &e);                  // mx = f 2^e, f in [0.5, 1); 0 for mx = 0
        float r[4];
        for (int i = 0; i < 4; ++i) x[i] = ldexpf(x[i], 8 - e);   // exact
        float x1[4], x2[4];
        const uint32_t c01 = tc_e4m3x2(x[0], x[1], x1[0], x1[1]);
        const uint32_t c23 = tc_e4m3x2(x[2], x[3], x1[2], x1[3]);
        for (int i = 0; i < 4; ++i) r[i] = (x[i] - x1[i]) * 16.f;   // exact
        const uint32_t d01 = tc_e4m3x2(r[0], r[1], x2[0], x2[1]);
        const uint32_t d23 = tc_e4m3x2(r[2], r[3], x2[2], x2[3]);
        const uint32_t w1 = c01 | (c23 << 16);
        const uint32_t w2 = d01 | (d23 << 16);
        const uint32_t chunk = static_cast<uint32_t>(lane) >> 2;
        const uint32_t within = (static_cast<uint32_t>(lane) & 3) * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t r1 = 16 * j + g, r2 = 16 * j + G + g;
          *reinterpret_cast<uint32_t*>(smem + L::kQOffset + r1 * 128 + ((chunk ^ (r1 & 7)) << 4) + within) = w1;
          *reinterpret_cast<uint32_t*>(smem + L::kQOffset + r2 * 128 + ((chunk ^ (r2 & 7)) << 4) + within) = w2;
        }
        if (lane == 0) qexp[g] = e;
      }
      fence_proxy_async_smem();
    }
    __syncthreads();

    if (warp == kTcProducerWarp) {
      split_producer<PAGED, false, STAGES, L::kTileBytes, L::kVRing - L::kKRing, L::kHalves>(
          a, &tmK, &tmV, smem_base + L::kKRing, bar_full, bar_empty, cta_error, lane, b, kvh,
          start, n, n_tiles, 0, nullptr);
    } else if (warp == kTcMmaWarp) {
      if (lane == 0) {
        constexpr uint32_t kIdS = idesc_e4m3_f32(64, kTcQuad * kTile, false, false);
        constexpr uint32_t kIdPV = idesc_e4m3_f32(128, 128, false, true);
        const uint32_t qaddr = smem_base + L::kQOffset;
        bool ok = true;
        // The scores of quad q (tiles 4q .. 4q+3, stages 4q mod STAGES ..),
        // once its tiles have landed; tiles past the split give columns
        // nobody reads.
        auto issue_scores = [&](int q) -> bool {
          const int t_end = min(kTcQuad * q + kTcQuad, n_tiles);
          for (int t = kTcQuad * q; t < t_end; ++t)
            if (!mbar_wait(bar_full + 8 * (t % STAGES), (t / STAGES) & 1, kWaitLimitNs)) return false;
          tcgen05_fence_after();
          const uint32_t kaddr = smem_base + L::kKRing + ((kTcQuad * q) % STAGES) * L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_e4m3(tmem, smem_desc(qaddr + 32 * kk, 16, 1024, 2),
                     smem_desc(kaddr + 32 * kk, 16, 1024, 2), kIdS, kk > 0);
          tcgen05_commit(s_full);
          return true;
        };
        ok = issue_scores(0);
        for (int i = 0; ok && i < n_tiles; ++i) {
          const int grp = i & 1, k = i >> 1;
          if (!mbar_wait(p_full + 8 * grp, k & 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tcgen05_fence_after();
          const int s = i % STAGES;
          const uint32_t vaddr = smem_base + L::kVRing + s * L::kTileBytes;
          const uint32_t paddr = smem_base + L::kPOffset + grp * L::kPBytes;
          const uint32_t d = tmem + kTcOCol + grp * 128;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_e4m3(d, smem_desc(paddr + 256 * kk, 128, 512, 0),
                     smem_desc(vaddr + 4096 * kk, 0, 1024, 2), kIdPV, k > 0 || kk > 0);
          tcgen05_commit(o_done + 8 * grp);
          tcgen05_commit(bar_empty + 8 * s);
          // After the first P.V of a quad, the next quad's scores: every
          // softmax warp has copied this quad's out of S by then.
          const int q = i / kTcQuad;
          if (i == kTcQuad * q && q + 1 < n_quads) {
            if (!mbar_wait(s_free, q & 1, kWaitLimitNs)) {
              ok = false;
              break;
            }
            ok = issue_scores(q + 1);
          }
        }
        if (!ok) {
          raise_device_error(1u);
          *cta_error = 1;
        }
        // Nothing may still run on the tensor cores when TMEM is released.
        tcgen05_commit(mma_done);
        if (!mbar_wait(mma_done, 0, kWaitLimitNs)) raise_device_error(2u);
      }
      __syncwarp();
    } else {
      // ----------------------------------------------------------- softmax
      // After the load, lane r holds S row r (code r / G of head r mod G)
      // for the warp's 16 tokens; the scores are then spread so that lane l
      // holds tokens m TPL .. m TPL + TPL - 1 of head h = l mod G (m = l / G),
      // and every lane does a share of the exponentials and weight codes.
      constexpr int TPL = G / 2;                            // tokens per lane
      const int grp = warp >> 2, j = warp & 3;
      const uint32_t lane_base = static_cast<uint32_t>(32 * j) << 16;
      const uint32_t s_tm = tmem + lane_base + 16 * j;      // + 64 per tile of the quad
      const uint32_t o_tm = tmem + lane_base + kTcOCol + grp * 128;
      const int h = lane % G, m = lane / G;
      const float sl2 = ldexpf(a.scale_log2, qexp[h] - 8);
      uint8_t* pbuf = smem + L::kPOffset + grp * L::kPBytes;
      // This lane's P bytes: code T of head h, tokens 16j + m TPL ...
      uint32_t poff[3];
#pragma unroll
      for (int T = 0; T < 3; ++T) poff[T] = tc_p_offset(32 * j + T * G + h, 16 * j + m * TPL);
      float m_run = -INFINITY, l_run = 0.f;                 // per head (l: this lane's share)
      bool failed = false;
      int k = 0;                                            // tiles of this warpgroup so far
      for (int q = 0; q < n_quads && !failed; ++q) {
        // This warpgroup's tiles of the quad: 4q + grp and 4q + grp + 2.
        if (!__all_sync(0xffffffffu, mbar_wait(s_full, q & 1, kWaitLimitNs))) {
          failed = true;
          break;
        }
        tcgen05_fence_after();
        uint32_t raw[2][16];
        tmem_ld16(s_tm + grp * kTile, raw[0]);
        tmem_ld16(s_tm + (grp + 2) * kTile, raw[1]);
        tmem_wait_ld();
        tcgen05_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = kTcQuad * q + grp + 2 * u;
          if (i >= n_tiles) break;
          const int tile_valid = min(kTile, end - (start + i * kTile));
          float t[TPL];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float v1 = __shfl_sync(0xffffffffu, __uint_as_float(raw[u][c]), h);
            const float v2 = __shfl_sync(0xffffffffu, __uint_as_float(raw[u][c]), G + h);
            if (c / TPL == m) t[c % TPL] = (v1 + v2 * 0.0625f) * sl2;
          }
          float mx = -INFINITY;
#pragma unroll
          for (int x = 0; x < TPL; ++x) {
            if (16 * j + m * TPL + x >= tile_valid) t[x] = -INFINITY;
            mx = fmaxf(mx, t[x]);
          }
#pragma unroll
          for (int off = G; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          const float m_new = fmaxf(m_run, mx);
          const bool rescale = k > 0 && m_new > m_run + kTcRescaleLog2;
          const float al = rescale ? ex2(m_run - m_new) : 1.f;
          if (k == 0 || rescale) m_run = m_new;
          l_run *= al;
          const float mu = m_run == -INFINITY ? 0.f : m_run;
          // p = p1 + p2 / 16 + p3 / 256, each code e4m3; the residuals are
          // exact in fp32.
          uint32_t w[3] = {0u, 0u, 0u};
          float lsum = 0.f;
#pragma unroll
          for (int x = 0; x < TPL; x += 2) {
            const float p0 = ex2(t[x] - mu);
            const float p1 = TPL > 1 ? ex2(t[x + 1] - mu) : 0.f;
            float a0, a1, b0, b1, d0, d1;
            const uint32_t c1 = tc_e4m3x2(p0, p1, a0, a1);
            const float r0 = p0 - a0, r1 = p1 - a1;
            const uint32_t c2 = tc_e4m3x2(r0 * 16.f, r1 * 16.f, b0, b1);
            const float e0 = r0 - b0 * 0.0625f, e1 = r1 - b1 * 0.0625f;
            const uint32_t c3 = tc_e4m3x2(e0 * 256.f, e1 * 256.f, d0, d1);
            lsum += ((a0 + a1) + (b0 + b1) * 0.0625f) + (d0 + d1) * 0.00390625f;
            w[0] |= c1 << (8 * x);
            w[1] |= c2 << (8 * x);
            w[2] |= c3 << (8 * x);
          }
          // P.V of this warpgroup's previous tile must be done before its P
          // buffer is rewritten or O is rescaled.
          if (k > 0) {
            if (!__all_sync(0xffffffffu, mbar_wait(o_done + 8 * grp, (k - 1) & 1, kWaitLimitNs))) {
              failed = true;
              break;
            }
            tcgen05_fence_after();
          }
          if (__any_sync(0xffffffffu, rescale)) {
            // Lane r holds O row r, whose head is r mod G: this lane's own.
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
              uint32_t o[16];
              tmem_ld16(o_tm + 16 * cc, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * al);
              tmem_st16(o_tm + 16 * cc, o);
            }
            tmem_wait_st();
          }
          l_run += lsum;
#pragma unroll
          for (int T = 0; T < 3; ++T) {
            if constexpr (TPL == 4) {
              *reinterpret_cast<uint32_t*>(pbuf + poff[T]) = w[T];
            } else if constexpr (TPL == 2) {
              *reinterpret_cast<uint16_t*>(pbuf + poff[T]) = static_cast<uint16_t>(w[T]);
            } else {
              pbuf[poff[T]] = static_cast<uint8_t>(w[T]);
            }
          }
          if (tile_valid < kTile) {
            // Rows past the sequence may hold anything (NaN included): zero
            // this warp's invalid V rows so that 0 * NaN never reaches O.
            // The wait on the stage's phase, already complete, orders its
            // copies before these writes.
            if (!__all_sync(0xffffffffu, mbar_wait(bar_full + 8 * (i % STAGES), (i / STAGES) & 1,
                                                   kWaitLimitNs))) {
              failed = true;
              break;
            }
            uint8_t* vt = smem + L::kVRing + (i % STAGES) * L::kTileBytes;
            const int rr = 16 * j + (lane >> 1);
            if (rr >= tile_valid) {
              uint4* dst = reinterpret_cast<uint4*>(vt + rr * 128 + (lane & 1) * 64);
#pragma unroll
              for (int c = 0; c < 4; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
            }
          }
          fence_proxy_async_smem();
          tcgen05_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full + 8 * grp);
          ++k;
        }
      }
      // The last P.V of this warpgroup.
      if (!failed && k > 0 &&
          !__all_sync(0xffffffffu, mbar_wait(o_done + 8 * grp, (k - 1) & 1, kWaitLimitNs)))
        failed = true;
      tcgen05_fence_after();
      grid_dependents_launch();
      if (failed && lane == 0) {
        raise_device_error(1u);
        *cta_error = 1;
      }
      // Both warpgroups are past their last MMA, so the ring holds the
      // scratch: per warp and head the O row (the three weight terms summed),
      // the running maximum and sum.
      named_barrier_sync(1, kTcSoftmaxWarps * 32);
      float* f = reinterpret_cast<float*>(smem);
      const bool live = !*cta_error;
      // Sum the lanes' shares of each head's running sum.
#pragma unroll
      for (int off = G; off < 32; off <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, off);
      const bool head_lane = lane < G;
      if (live) {
        float* dst = f + L::kRedAcc + (warp * L::kNcol + h) * L::kAccStride;
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t o[16];
          if (k > 0) {
            tmem_ld16(o_tm + 16 * cc, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] = 0u;
          }
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float v = __uint_as_float(o[c]);
            const float v2 = __shfl_down_sync(0xffffffffu, v, G);
            const float v3 = __shfl_down_sync(0xffffffffu, v, 2 * G);
            if (head_lane) dst[16 * cc + c] = v + (v2 * 0.0625f + v3 * 0.00390625f);
          }
        }
        if (head_lane) {
          f[L::kRedM + warp * L::kNcol + h] = m_run;
          f[L::kRedL + warp * L::kNcol + h] = l_run;
        }
      }
      named_barrier_sync(1, kTcSoftmaxWarps * 32);
      if (live) split_merge<128, 1, kHi, kTcSoftmaxWarps, L>(a, f, b, h0, split, n_parts);
    }
  }

  // Release the tensor memory once every warp is past its last use.
  tcgen05_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tcgen05_fence_after();
    tmem_dealloc(tmem, kTcCols);
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
