/*
 * fd.h — C ABI of the B200 (sm_100a) split-KV decode attention library
 * (libfd.so).
 *
 * The operation is Flash-Decoding ("What is Flash-Decoding, and when does it
 * speed up LLMs?", slavadubrov.com: the opening paragraph and the section
 * "Why decode needs a different schedule"). One new query token per
 * sequence attends over that sequence's long cached K/V history. The history
 * is split into chunks. Each chunk gives a partial output and a log-sum-exp,
 * and a reduction merges the partials into the exact attention over the
 * whole history:
 *
 *     out[b, h, :] = softmax_j(scale * q[b, h, :] . K[b, kv, j, :]) @ V[b, kv, j, :]
 *     lse[b, h]    = ln sum_j exp(scale * q[b, h, :] . K[b, kv, j, :])
 *
 * Here kv = h / (Hq / Hkv), which covers grouped-query attention, and j runs
 * over the seqlens[b] valid cached tokens.
 *
 * Conventions shared by every entry point:
 *  - Tensor pointers are DEVICE pointers owned by the caller. The library
 *    keeps no pointer and allocates nothing; the workspace is caller-supplied.
 *  - Element types: q and out are bf16; K and V are bf16 or fp8 E4M3 codes
 *    (fd_problem.kv_dtype); lse, the workspace and scale are fp32; seqlens
 *    and block_table are int32.
 *  - Errors are return codes. No entry point aborts, throws or prints.
 *    Argument checks run on the host before anything is launched; an invalid
 *    call launches nothing.
 *  - Work is asynchronous on the caller's stream. A fault inside a kernel
 *    surfaces at the caller's next synchronisation.
 *  - There is no CPU fallback. The kernels are built for sm_100a only.
 */
#ifndef FD_H_
#define FD_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FD_API __attribute__((visibility("default")))
#else
#define FD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (struct CUstream_st*); NULL is the legacy default
 * stream. */
typedef struct CUstream_st* fd_stream_t;

typedef enum fd_status {
  FD_OK = 0,
  /* Null pointer, non-positive size, Hq % Hkv != 0, a tensor pointer not
   * 16-byte aligned (lse: 4-byte), num_splits outside [1, 1024], scale not
   * finite and positive, unknown kv_layout, shape limits exceeded. */
  FD_ERR_INVALID_ARGUMENT = -1,
  /* Head dim D not in {64, 128}, group size Hq/Hkv not in {1, 2, 4, 8, 16},
   * block_size not a power of two in [8, 256], or the device is not sm_100. */
  FD_ERR_UNSUPPORTED = -2,
  /* The chosen split count needs a workspace, and the one passed is NULL or
   * smaller than fd_workspace_bytes() reports. */
  FD_ERR_WORKSPACE = -3,
  /* A CUDA runtime or driver call failed (launch error, tensor-map encode). */
  FD_ERR_CUDA = -4,
  /* A kernel gave up on a bounded wait. Its outputs are not valid. */
  FD_ERR_DEVICE_TIMEOUT = -5
} fd_status;

/* Order of the cache dimensions (see fd_decode for the full shapes). */
typedef enum fd_kv_layout {
  /* heads outside tokens: [B, Hkv, max_len, D] or [num_blocks, Hkv, block_size, D] */
  FD_LAYOUT_HND = 0,
  /* tokens outside heads: [B, max_len, Hkv, D] or [num_blocks, block_size, Hkv, D] */
  FD_LAYOUT_NHD = 1
} fd_kv_layout;

/* Element type of the K/V cache. */
typedef enum fd_kv_dtype {
  FD_KV_BF16 = 0,     /* bf16 */
  FD_KV_FP8_E4M3 = 1  /* OCP fp8 e4m3 (bias 7, max 448, no inf); value = scale * code */
} fd_kv_dtype;

/* Tensor-core path of an fp8 cache.
 *   FD_FP8_MMA_SYNC     the default: e4m3 codes converted to f16 in registers,
 *                       both contractions on mma.sync with fp32 accumulation.
 *   FD_FP8_MMA_TCGEN05  kind::f8f6f4 tcgen05 MMAs on the codes as the TMA left
 *                       them in shared memory, accumulators in tensor memory;
 *                       q and the softmax weights enter as sums of e4m3 codes
 *                       (q exactly, the weights to 12 significant bits). Taken
 *                       where G is 2, 4 or 8 and the grid has at most one CTA
 *                       per SM; other calls run the default path. Measured
 *                       slower on B200 (CodeLlama-34B heads, 64K tokens:
 *                       40.8 against 24.2 us per call). */
typedef enum fd_fp8_mma {
  FD_FP8_MMA_SYNC = 0,
  FD_FP8_MMA_TCGEN05 = 1
} fd_fp8_mma;

/* Shape of one decode-attention call.
 *   B           sequences in the batch (1 .. 65535)
 *   Hq, Hkv     query heads and KV heads (Hkv .. 65535, Hq % Hkv == 0)
 *   D           head dimension (64 or 128)
 *   max_len     contiguous cache: rows held per (sequence, KV head);
 *               paged cache: the longest sequence the block table can hold
 *               (<= max_blocks_per_seq * block_size)
 *   block_size  0 for a contiguous cache; otherwise tokens per page
 *   num_blocks  paged cache: pages in the pool (ignored when contiguous)
 *   max_blocks_per_seq  paged cache: row length of block_table
 *   kv_layout   an fd_kv_layout value (FD_LAYOUT_HND when zero-initialised)
 *   kv_dtype    an fd_kv_dtype value (FD_KV_BF16 when zero-initialised)
 *   k_scale, v_scale
 *               fp8 caches: the real K and V are k_scale * code and
 *               v_scale * code (finite, > 0). Ignored for bf16 caches.
 *               An fp8 cache needs D = 128; on the default path the
 *               contraction runs on f16 tensor cores, so q must be finite
 *               in f16 (|q| < 65504).
 *   fp8_mma     an fd_fp8_mma value (FD_FP8_MMA_SYNC when zero-initialised);
 *               ignored for bf16 caches. */
typedef struct fd_problem {
  int32_t B;
  int32_t Hq;
  int32_t Hkv;
  int32_t D;
  int32_t max_len;
  int32_t block_size;
  int32_t num_blocks;
  int32_t max_blocks_per_seq;
  int32_t kv_layout;
  int32_t kv_dtype;
  float k_scale;
  float v_scale;
  int32_t fp8_mma;
} fd_problem;

/* Split-count planner.
 * Follows the same page's section "Why decode needs a different schedule".
 * Splitting the history creates extra work units when the batch supplies too
 * few. For a short history the partials and the reduction can cost more than
 * they save, and a large batch already supplies the work.
 * Returns S >= 1 for fd_decode's num_splits, chosen for the current device's
 * SM count. Returns 1 when B*Hkv already fills the device or the history is
 * short. Returns a negative fd_status for invalid or unsupported shapes.
 * Host only and deterministic. It reads the SM count of the current device
 * once per device and caches it. */
FD_API int fd_plan(int B, int Hq, int Hkv, int D, int max_len, int block_size);

/* The same planner with the SM count given explicitly. Pure function: no
 * CUDA call. */
FD_API int fd_plan_sm(int num_sms, int B, int Hq, int Hkv, int D, int max_len,
               int block_size);

/* Split-count planner that also sees the sequence lengths of the batch.
 * Same rule as fd_plan, with one difference. When the lengths differ,
 * splitting also evens out the work per CTA: one long sequence would
 * otherwise decide the end of the call. This planner therefore models the
 * actual per-sequence lengths instead of assuming max_len for every sequence.
 *   num_sms   SM count to plan for; <= 0 means the current device's
 *   seqlens   HOST array [B] of valid tokens per sequence, clamped to
 *             [0, max_len] as in fd_decode
 * Returns S >= 1, or a negative fd_status (a NULL seqlens is
 * FD_ERR_INVALID_ARGUMENT). Host only and deterministic. It costs O(B)
 * per candidate split count. */
FD_API int fd_plan_seqlens(int num_sms, int B, int Hq, int Hkv, int D, int max_len,
                           int block_size, const int32_t* seqlens);

/* The planner for a whole problem description: the same cost model, with
 * the cache's element type (an fp8 CTA moves half the bytes of a bf16 one
 * at the same token rate, so fp8 caches want more CTAs in flight) and, when
 * given, the lengths. fd_plan and fd_plan_seqlens plan for bf16 caches.
 *   num_sms   SM count to plan for; <= 0 means the current device's
 *   p         HOST pointer to the problem as passed to fd_decode (pointers
 *             and scales are not read)
 *   seqlens   HOST array [B] of valid tokens per sequence, or NULL when
 *             every sequence holds max_len
 * Returns S >= 1, or a negative fd_status: FD_ERR_INVALID_ARGUMENT for a
 * NULL p, a bad shape or an unknown kv_dtype; FD_ERR_UNSUPPORTED for an fp8
 * cache with D != 128. Host only and deterministic. */
FD_API int fd_plan_problem(int num_sms, const fd_problem* p, const int32_t* seqlens);

/* How a call cuts the history. With T = ceil(max_len / 64) tiles of 64
 * tokens, the effective split count is S = min(num_splits, T) (1 when
 * max_len is 0), and split s covers the tiles [floor(s*T/S),
 * floor((s+1)*T/S)) of every sequence: tokens [64*floor(s*T/S),
 * 64*floor((s+1)*T/S)), cut at the sequence's length. The splits differ by
 * at most one tile, so any split count up to T gives CTAs of balanced size.
 * Splits past a sequence's end are empty.
 * fd_split_chunk returns the largest split's tokens, 64*ceil(T/S) (64 when
 * max_len is 0); fd_effective_splits returns S. Both return a negative
 * fd_status for invalid arguments. */
FD_API int fd_split_chunk(int max_len, int num_splits);
FD_API int fd_effective_splits(int max_len, int num_splits);

/* Workspace bytes that fd_decode needs for num_splits splits. This is 0
 * when num_splits == 1. Otherwise it is the fp32 partial outputs
 * [B, Hq, S, D] followed by the fp32 partial log-sum-exps [B, Hq, S], each
 * part rounded up to 256 bytes, with S = num_splits. The effective split
 * count (fd_effective_splits) never exceeds num_splits, so this size is
 * always enough for the call.
 * Returns 0 for invalid arguments. */
FD_API size_t fd_workspace_bytes(int B, int Hq, int D, int num_splits);

/* Decode attention for one query token per sequence.
 *   p            shape (see fd_problem)
 *   q            [B, Hq, D] bf16, 16-byte aligned
 *   k_cache, v_cache
 *                (elements bf16, or fp8 e4m3 bytes when kv_dtype says so)
 *                FD_LAYOUT_HND contiguous: [B, Hkv, max_len, D];
 *                FD_LAYOUT_HND paged:      [num_blocks, Hkv, block_size, D];
 *                FD_LAYOUT_NHD contiguous: [B, max_len, Hkv, D];
 *                FD_LAYOUT_NHD paged:      [num_blocks, block_size, Hkv, D];
 *                row-major, 16-byte aligned
 *   seqlens      [B] int32 valid tokens per sequence, or NULL (all max_len).
 *                Values are clamped to [0, max_len]. Rows at or past a
 *                sequence's length are never summed; they may hold anything,
 *                NaN included. A length of 0 gives out = 0 and lse = -inf.
 *   block_table  paged only: [B, max_blocks_per_seq] int32; token t of
 *                sequence b sits in page block_table[b, t / block_size], row
 *                t % block_size. Entries are read only for pages that hold
 *                valid tokens. A page id outside [0, num_blocks) reads zeros.
 *                NULL selects the contiguous layout and needs block_size == 0.
 *   scale        softmax scale (finite, > 0), typically 1/sqrt(D)
 *   num_splits   requested split count in [1, 1024], normally fd_plan's
 *                result. The effective count is min(num_splits,
 *                ceil(max_len / 64)); see fd_split_chunk for the cut.
 *   out          [B, Hq, D] bf16, round-to-nearest-even, 16-byte aligned
 *   lse          [B, Hq] fp32 natural-log log-sum-exp of the scaled logits,
 *                or NULL to skip it
 *   workspace    fp32 scratch of at least fd_workspace_bytes(B, Hq, D, S)
 *                bytes for the effective split count S (the num_splits
 *                passed is always enough), 16-byte aligned. It may be NULL
 *                when S == 1. Its
 *                contents on entry do not matter, and it must not be shared
 *                by calls that overlap on the GPU.
 *   stream       the stream to run on
 * Results are bit-identical across repeated calls with the same inputs and
 * the same num_splits. The paged and contiguous layouts of the same logical
 * cache also give bit-identical results. */
FD_API fd_status fd_decode(const fd_problem* p, const void* q, const void* k_cache,
                    const void* v_cache, const int32_t* seqlens,
                    const int32_t* block_table, float scale, int num_splits,
                    void* out, float* lse, void* workspace,
                    size_t workspace_bytes, fd_stream_t stream);

/* Partial decode over a shard of each sequence's history, for merging
 * across GPUs (sequence-parallel decode).
 * When each GPU holds a contiguous slice of every sequence's cached tokens,
 * each GPU calls this on its own slice. The call returns the exact attention
 * over that slice: a normalised fp32 output and its log-sum-exp. After the
 * R results are gathered in one place (for example with an NCCL all-gather),
 * fd_combine merges them into the attention over the whole history. This is
 * the same log-sum-exp reduction that merges the splits of one GPU (page
 * "What is Flash-Decoding, and when does it speed up LLMs?", section "Why
 * decode needs a different schedule").
 * Arguments are those of fd_decode, except two outputs:
 *   out_f32  [B, Hq, D] fp32, 16-byte aligned (required)
 *   lse      [B, Hq] fp32 (required)
 * An empty slice gives out_f32 = 0 and lse = -inf, which weighs nothing in
 * fd_combine. */
FD_API fd_status fd_decode_partial(const fd_problem* p, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* seqlens,
                                   const int32_t* block_table, float scale, int num_splits,
                                   float* out_f32, float* lse, void* workspace,
                                   size_t workspace_bytes, fd_stream_t stream);

/* Merges R partial results into the final output. Each part covers a
 * disjoint slice of the history, for example one per GPU from
 * fd_decode_partial:
 *   m = max_r lse_r,  out = sum_r e^(lse_r - m) O_r / sum_r e^(lse_r - m),
 *   lse = m + ln sum_r e^(lse_r - m).
 *   part_o    [R, B, Hq, D] fp32, 16-byte aligned (parts outermost, as an
 *             all-gather along a new leading dimension lays them out)
 *   part_lse  [R, B, Hq] fp32
 *   out       [B, Hq, D] bf16, round-to-nearest-even, 16-byte aligned
 *   lse       [B, Hq] fp32 or NULL
 * R is in [1, 1024] and D is 64 or 128. A row whose parts are all empty gives
 * out = 0 and lse = -inf. Parts are summed in index order, so the result is
 * deterministic. It runs asynchronously on `stream`. */
FD_API fd_status fd_combine(int R, int B, int Hq, int D, const float* part_o,
                            const float* part_lse, void* out, float* lse, fd_stream_t stream);

/* fd_combine over parts placed at any stride, so that a gathered buffer is
 * merged where it lies, with no copy. Part r of row i (i = b * Hq + h) is the
 * D floats at part_o + r * o_stride + i * D and the lse at
 * part_lse[r * lse_stride + i]; fd_combine is the case o_stride = B*Hq*D,
 * lse_stride = B*Hq. One packed buffer per part, for example
 *   [O: B*Hq*D floats][lse: B*Hq floats][padding]
 * all-gathered into R consecutive buffers of P floats, is merged with
 *   part_o = buf, part_lse = buf + B*Hq*D, o_stride = lse_stride = P.
 * Strides count floats. o_stride must be a multiple of 4 and at least
 * B*Hq*D; lse_stride at least B*Hq; otherwise FD_ERR_INVALID_ARGUMENT. The
 * rest is as fd_combine. */
FD_API fd_status fd_combine_strided(int R, int B, int Hq, int D, const float* part_o,
                                    size_t o_stride, const float* part_lse, size_t lse_stride,
                                    void* out, float* lse, fd_stream_t stream);

/* Low-bit key codes for fd_decode_sparse ("Faster Than Flash: Exploiting
 * Attention Sparsity for Efficient Long-Context Decoding", abstract: a scan
 * over low-bit keys replaces metadata indices). Call it when the cache
 * changes (in a decode loop, for the blocks that tokens were appended to).
 * For every 64-token block of every (sequence, KV head):
 *   k8_scale = max |K| over the block's valid rows / 127 (1 for an all-zero
 *              block), fp32;
 *   k8       = rint(K / k8_scale) in [-127, 127], int8; rows at or past the
 *              sequence's length get 0.
 *   p         contiguous head-major bf16 cache (block_size 0, FD_LAYOUT_HND,
 *             FD_KV_BF16), D 64 or 128
 *   k_cache   [B, Hkv, max_len, D] bf16, 16-byte aligned
 *   seqlens   [B] int32 or NULL (all max_len)
 *   k8        [B, Hkv, max_len, D] int8 out, 16-byte aligned
 *   k8_scale  [B, Hkv, ceil(max_len / 64)] fp32 out
 * Returns FD_ERR_UNSUPPORTED for a paged, token-major or fp8 cache. */
FD_API fd_status fd_quantize_keys(const fd_problem* p, const void* k_cache,
                                  const int32_t* seqlens, int8_t* k8, float* k8_scale,
                                  fd_stream_t stream);

/* Sparse decode: fd_decode over the blocks a low-bit scan selects (same page,
 * abstract: a top-delta rule that filters blocks adaptively with no global
 * synchronisation, selector and computation fused in one kernel). Inside the
 * split kernel, before any K/V tile is loaded, each CTA (one split of one
 * KV head of one sequence):
 *   1. turns each query head of the group into int8: sq = max |q| / 127,
 *      q8 = rint(q / sq);
 *   2. computes for every 64-token block of its split, and every head, the
 *      largest approximate logit ((scale * sq) * k8_scale) * (q8 . k8), with
 *      the dot product exact in integers and each product rounded to fp32 in
 *      that order;
 *   3. keeps a block when some head's block maximum is >= M - delta, M being
 *      that head's largest block maximum in the split;
 *   4. runs the exact bf16 attention of fd_decode over the kept blocks only.
 * The splits then merge as in fd_decode. The result is the exact attention
 * over the union of the kept blocks. delta = +inf keeps every block and gives
 * fd_decode's result bit for bit.
 *   k8, k8_scale  from fd_quantize_keys on the same cache and lengths
 *   delta         >= 0, natural-log units (NaN is invalid)
 *   kept          [B, Hkv, ceil(max_len / 64)] uint8 out (1 = kept), or NULL.
 *                 Blocks at or past a sequence's length are not written.
 * Other arguments are those of fd_decode with a contiguous head-major bf16
 * cache and D = 128 (FD_ERR_UNSUPPORTED otherwise). The split count must make
 * the largest split (fd_split_chunk) at most 16,384 tokens
 * (FD_ERR_INVALID_ARGUMENT otherwise). The
 * codes stream through the split kernel's tile pipeline (TMA, 256 tokens per
 * stage) and the dot products run on int8 tensor cores. Results are
 * deterministic. */
FD_API fd_status fd_decode_sparse(const fd_problem* p, const void* q, const void* k_cache,
                                  const void* v_cache, const int8_t* k8,
                                  const float* k8_scale, const int32_t* seqlens, float scale,
                                  float delta, int num_splits, void* out, float* lse,
                                  uint8_t* kept, void* workspace, size_t workspace_bytes,
                                  fd_stream_t stream);

/* Largest workspace, in bytes, that fd_decode_static_workspace can use. */
#define FD_STATIC_WORKSPACE_BYTES (8u << 20)

/* fd_decode for callers that cannot allocate device memory.
 * The Flash-Decoding pages have no counterpart to this entry point; it is an
 * addition of this library. Some callers cannot call cudaMalloc at all. Examples: a plain C
 * host program that links only this library and has no device allocator of
 * its own; code inside a framework whose memory pool owns all device memory
 * and forbids raw allocations; a decode loop that must not call cudaMalloc
 * mid-step, because it can block on the device and can fail when memory runs
 * short.
 * Such callers still pass q, the caches, seqlens, block_table, out and lse,
 * exactly as for fd_decode. The workspace comes from a file-scope static
 * __device__ array of FD_STATIC_WORKSPACE_BYTES bytes, which every GPU that
 * loads this library holds until the process exits. This entry point calls
 * no cudaMalloc, cudaFree or other allocating routine.
 *  - Set-up: the first call on a device looks up the array's device address
 *    with the device current (cudaGetSymbolAddress) and caches it with the
 *    id of the device's context. Make that first call before any stream
 *    capture on that device. After a device reset (cudaDeviceReset) the
 *    device has a new context, in which the array may sit elsewhere: the
 *    next call sees the new context id and looks the address up again, so
 *    make that call, too, outside a capture.
 *  - Size limit: when the effective split count needs more than
 *    FD_STATIC_WORKSPACE_BYTES (see fd_workspace_bytes), the call returns
 *    FD_ERR_WORKSPACE and launches nothing. Pass a smaller num_splits, or use
 *    fd_decode with your own workspace.
 *  - Sharing: every call on a device uses the same array, which keeps the
 *    last call's contents. Nothing in it has to start at zero, because each
 *    call writes every partial result before reading it. Calls that overlap
 *    on the GPU, such as calls on two streams, race on the array and give
 *    wrong results: serialise them.
 * Returns the same codes as fd_decode. */
FD_API fd_status fd_decode_static_workspace(const fd_problem* p, const void* q,
                                            const void* k_cache, const void* v_cache,
                                            const int32_t* seqlens,
                                            const int32_t* block_table, float scale,
                                            int num_splits, void* out, float* lse,
                                            fd_stream_t stream);

/* Waits for `stream`, then reads and clears the current device's error word.
 * A kernel sets that word when one of its bounded waits runs out. Returns
 * FD_OK, FD_ERR_DEVICE_TIMEOUT, or FD_ERR_CUDA. */
FD_API fd_status fd_check_device_error(fd_stream_t stream);

/* Diagnostic of the failure path. Launches one warp that waits, with the
 * same bounded wait the kernels use, on an mbarrier that nothing ever
 * completes. After limit_us microseconds the wait gives up, and the kernel
 * sets the device error word the way a stalled split kernel would. The next
 * fd_check_device_error(stream) then returns FD_ERR_DEVICE_TIMEOUT and
 * clears the word. Nothing faults or hangs, and the context stays usable.
 * limit_us must be in [1, 5,000,000]. Returns FD_OK once launched. */
FD_API fd_status fd_selftest_device_timeout(unsigned int limit_us, fd_stream_t stream);

/* Static, human-readable name of a status code. */
FD_API const char* fd_status_string(fd_status status);

#ifdef __cplusplus
}
#endif

#endif /* FD_H_ */
