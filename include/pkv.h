/*
 * pkv.h -- C ABI of the B200 (sm_100a) paged-KV decode library.
 *
 * Two operations make up one decode step of one attention layer over a
 * block-structured ("paged") KV cache, the data structure the pages build
 * their serving engines around:
 *
 *   pkv_kv_append               RoPE on the new token's q (in place) and k,
 *                               then k and v written into the token's slot.
 *   pkv_paged_attention_decode  single-query attention softmax(q K^T scale) V
 *                               for every sequence and query head, reading K/V
 *                               through the sequence's block table.
 *
 * Around them: the two in one launch (pkv_decode_step); a sliding window
 * (pkv_paged_attention_decode_window); shared-prefix groups read once
 * (pkv_paged_attention_decode_cascade); chunked prefill
 * (pkv_paged_attention_prefill); an 8-bit E4M3 cache (pkv_kv_append_e4m3,
 * pkv_paged_attention_decode_e4m3, and the two in one launch,
 * pkv_decode_step_e4m3); a decode without a caller workspace
 * (pkv_paged_attention_decode_noalloc); and a host-side block manager with
 * prefix reuse (pkv_bm_*).
 *
 * Sources (page title, section):
 *   "Inference From Scratch" (book intro), "What you will build" and the
 *     chapter table: ch. 4 KV cache, ch. 8 online softmax / flash attention,
 *     ch. 9 continuous batching, ch. 10 paged attention and block tables,
 *     ch. 11 prefix caching by block reuse;
 *   "The Project: Serve Your Own LLM", milestones M2 (MHA/GQA/MQA choice of
 *     n_kv_heads), M10 (paged_gather kernel and its coalescing), M13b/M13c
 *     (paged greedy decode equals full recompute; a block pool smaller than
 *     the worst case);
 *   "LLM Inference from Scratch", Architecture overview (Llama-style decoder
 *     with RoPE and causal attention; M1 KV cache, prefill/decode
 *     equivalence);
 *   "warpllama", Milestones (static KV cache + single-token decode; fused
 *     RoPE kernel; fused attention hot path in CUDA);
 *   "Efficient LLM Inference", learning route: KV Caching (reuse, positions
 *     and windows; chunked equals full prefix), KV memory accounting,
 *     Quantization, and verifying exact execution and approximate quality
 *     separately.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.   Every tensor pointer is a DEVICE pointer (cudaMalloc, the
 *             PyTorch caching allocator, ...) unless stated otherwise.  The
 *             caller owns every buffer, including the workspace; the library
 *             never allocates device memory and keeps no pointer after a call
 *             returns.
 * Layout.     Row-major and contiguous ("[A, B, C]" means C is innermost):
 *               q            [num_tokens or num_seqs, Hq, head_dim]
 *               k_new, v_new [num_tokens, Hkv, head_dim]
 *               k/v cache    [num_blocks, Hkv, block_size, head_dim]
 *               block_tables [num_seqs, max_blocks_per_seq]  int32
 *               out          [num_seqs, Hq, head_dim]
 *             Token t of sequence b lives in physical block
 *             block_tables[b][t / block_size], row t % block_size.  A slot
 *             s names physical block s / block_size, row s % block_size.
 * Heads.      Hq must be a multiple of Hkv; query head h reads KV head
 *             h / (Hq / Hkv) (contiguous groups).
 * Supported.  head_dim in {64, 128}; block_size 16; Hq / Hkv in {1, 2, 4, 8};
 *             storage dtype fp32 or bf16 (PKV_DTYPE_*), the same for q, the
 *             new k/v and the cache; or an 8-bit E4M3 cache with bf16 q (the
 *             *_e4m3 entry points).
 * Alignment.  q, k_new, v_new, caches, out and workspace: 16-byte aligned.
 * Streams.    `stream` is a cudaStream_t (NULL = legacy default stream).  All
 *             work is enqueued asynchronously on it; a call returns as soon as
 *             its kernels are launched.
 * Errors.     Arguments are validated on the host before anything is
 *             launched; a bad argument returns a status and launches nothing.
 *             The library never reads device-resident values (slots, block
 *             ids, context lengths) on the host.  Kernels check those values
 *             themselves: an out-of-range value sets a bit in the optional
 *             device word `device_error` (PKV_DEVERR_*, OR-ed in, never
 *             cleared by the library) and the offending access is skipped --
 *             a kernel never traps and never faults on such input.  Every
 *             wait inside a kernel is bounded; a wait that runs out sets
 *             PKV_DEVERR_TIMEOUT and the kernel returns.
 * Threads.    Entry points are thread-safe; calls on one stream run in order.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pkv_status {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or shape */
    PKV_ERR_UNSUPPORTED = 2, /* valid, but outside the supported set above */
    PKV_ERR_WORKSPACE = 3,   /* workspace smaller than required */
    PKV_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    PKV_ERR_DEVICE = 5       /* pkv_get_device_error: the kernels reported a bad
                                device-resident value or a wait that ran out */
} pkv_status;

typedef enum pkv_dtype {
    PKV_DTYPE_F32 = 0,
    PKV_DTYPE_BF16 = 1,
    PKV_DTYPE_E4M3 = 2 /* 8-bit cache only: E4M3 codes x a per-tensor scale, see
                          pkv_kv_append_e4m3 / pkv_paged_attention_decode_e4m3 */
} pkv_dtype;

/* Bits OR-ed into *device_error by the kernels. */
#define PKV_DEVERR_SLOT 0x1u        /* slot_mapping[t] >= num_blocks * block_size  */
#define PKV_DEVERR_BLOCK_ID 0x2u    /* block table entry outside [0, num_blocks)   */
#define PKV_DEVERR_CONTEXT_LEN 0x4u /* context_lens[b] < 0 or > max_blocks * bs    */
#define PKV_DEVERR_TIMEOUT 0x8u     /* a bounded in-kernel wait ran out            */
#define PKV_DEVERR_PREFIX 0x10u     /* cascade: a group is malformed, or a member's
                                       shared block ids differ from its group's      */

/* Decode flags. */
#define PKV_DECODE_FORCE_SIMT 0x1u  /* bf16: use the CUDA-core kernel instead of the
                                       tensor-core one (same result within tolerance) */
#define PKV_DECODE_NO_CLUSTER 0x2u  /* never merge split contexts inside a thread-block
                                       cluster; always partials + combine kernel */

/* Upper limits of one call. */
#define PKV_MAX_SEQS_PER_CALL 4096
#define PKV_MAX_PARTITION_TOKENS 8192

/*
 * pkv_kv_append -- rotate the new tokens' q and k, write k and v into the cache.
 *
 * Source: "warpllama", Milestones (static KV cache + single-token decode,
 * fused RoPE); "LLM Inference from Scratch", Architecture overview (RoPE);
 * "Inference From Scratch", ch. 10 (block tables: a token's K/V go to the
 * physical slot its sequence's table assigns).
 *
 * For every token t < num_tokens, with p = positions[t]:
 *   q[t, h, :]   <- rope(q[t, h, :], p)                   (in place, all h < Hq)
 *   if s = slot_mapping[t] >= 0:
 *     k_cache[s / bs, h, s % bs, :] <- rope(k_new[t, h, :], p)   (h < Hkv)
 *     v_cache[s / bs, h, s % bs, :] <- v_new[t, h, :]            (bit copy)
 * rope() turns each pair (x[i], x[i + d/2]), i < d/2, by the angle
 * p * rope_theta^(-2i/d); the angle and the rotation are computed in fp64 and
 * the result is rounded once to the storage type (bf16: nearest, ties to
 * even).  A negative slot skips the cache write for that token (padding).
 *
 * Arguments
 *   q             device, [num_tokens, Hq, head_dim], dtype; read and written
 *   k_new, v_new  device, [num_tokens, Hkv, head_dim], dtype; read only
 *   positions     device, [num_tokens] int64, >= 0
 *   slot_mapping  device, [num_tokens] int64; < 0 = skip,
 *                 >= num_blocks * block_size sets PKV_DEVERR_SLOT and skips
 *   k_cache, v_cache  device, [num_blocks, Hkv, block_size, head_dim], dtype
 *   dtype         PKV_DTYPE_F32 or PKV_DTYPE_BF16
 *   rope_theta    RoPE base (> 0)
 *   device_error  device int32 or NULL
 *   stream        cudaStream_t
 * Two tokens with the same slot race; the caller gives each token its own.
 * num_tokens == 0 returns PKV_OK and launches nothing.
 */
pkv_status pkv_kv_append(void* q, const void* k_new, const void* v_new,
                         const int64_t* positions, const int64_t* slot_mapping,
                         void* k_cache, void* v_cache,
                         int64_t num_tokens, int64_t num_q_heads, int64_t num_kv_heads,
                         int64_t head_dim, int64_t num_blocks, int64_t block_size,
                         int32_t dtype, double rope_theta,
                         int32_t* device_error, void* stream);

/*
 * pkv_decode_workspace_size -- bytes of workspace pkv_paged_attention_decode
 * needs for these shapes.
 *
 * Layout: 256 bytes of work-scheduler counters, then, when contexts are
 * split, the per-partition partial results (running max, sum and output) of
 * the split-context ("flash-decoding") path: num_seqs * Hq * max_partitions *
 * (head_dim + 2) floats, where max_partitions = ceil(max_blocks_per_seq *
 * block_size / P) and P is the partition length the decode call will use
 * (partition_tokens, or the library's choice for the current device when it
 * is 0).  Pass the same shapes, dtype and partition_tokens to both calls.
 * The counters let CTAs that finish early claim more work items; they must
 * be zero before a workspace's first call (zero the first 256 bytes once,
 * e.g. with cudaMemset at allocation) and every call leaves them zero.  Host
 * only; no device memory is touched.  Returns 0 for invalid arguments.
 */
size_t pkv_decode_workspace_size(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                                 int64_t head_dim, int64_t max_blocks_per_seq,
                                 int64_t block_size, int32_t kv_dtype, int32_t partition_tokens);

/*
 * pkv_decode_launches -- how many kernels a decode call with these shapes
 * makes on the current device: 1 (one decode kernel: no context split, or
 * split contexts merged inside thread-block clusters) or 2 (the decode
 * kernel and the partition-combine kernel).  fused != 0 asks about
 * pkv_decode_step, 0 about pkv_paged_attention_decode.  Queries the current
 * device's occupancy limits (cached); launches nothing.  Returns 0 for
 * invalid arguments or when no device answers.
 */
int32_t pkv_decode_launches(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                            int64_t head_dim, int64_t max_blocks_per_seq, int64_t block_size,
                            int32_t kv_dtype, int32_t out_dtype, int32_t partition_tokens,
                            uint32_t flags, int32_t fused);

/*
 * pkv_decode_partition_tokens -- the partition length P (tokens, a multiple of
 * block_size) that a decode call with these shapes uses when its
 * partition_tokens argument is 0.  Host only.  Returns 0 for invalid
 * arguments.
 */
int32_t pkv_decode_partition_tokens(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                                    int64_t head_dim, int64_t max_blocks_per_seq,
                                    int64_t block_size, int32_t kv_dtype);

/*
 * pkv_paged_attention_decode -- one query token per sequence attends to its
 * whole cached context through its block table.
 *
 * Source: "Inference From Scratch", ch. 8 (online softmax, flash attention)
 * and ch. 10 (paged attention over block tables); "The Project: Serve Your
 * Own LLM", M2 (GQA) and M13b (paged decode equals the full-recompute
 * reference); "LLM Inference from Scratch", M1 (decode equals the last row
 * of the full-prefix causal pass, so causal attention of the newest token
 * covers every cached token and needs no mask inside the context).
 *
 * For b < num_seqs, h < Hq, with L = context_lens[b], kvh = h / (Hq / Hkv):
 *   s_t = scale * <q[b, h, :], K_b[t]>, t < L, K_b[t] the cache row of token t
 *   out[b, h, :] = sum_t exp(s_t - max s) V_b[t] / sum_t exp(s_t - max s)
 * and out[b, h, :] = 0 when L == 0.  Arithmetic is fp32 (bf16 inputs widen
 * exactly); the result is rounded once to out_dtype.
 *
 * Arguments
 *   q             device, [num_seqs, Hq, head_dim], kv_dtype
 *   k_cache, v_cache  device, [num_blocks, Hkv, block_size, head_dim], kv_dtype
 *   block_tables  device, [num_seqs, max_blocks_per_seq] int32; only the first
 *                 ceil(L / block_size) entries of a row are read
 *   context_lens  device, [num_seqs] int32 in [0, max_blocks_per_seq * block_size]
 *   out           device, [num_seqs, Hq, head_dim], out_dtype (f32 or bf16)
 *   workspace     device, >= pkv_decode_workspace_size(...) bytes, 16-byte
 *                 aligned; its first 256 bytes zero before its first call
 *                 (each call leaves them zero), the rest is clobbered.  Two
 *                 calls in flight at once need two workspaces.  May be NULL
 *                 when max_partitions is 1 (no context is split): the work
 *                 items are then dealt out round-robin instead of claimed
 *   partition_tokens  0 = library choice, else a multiple of block_size in
 *                 [block_size, PKV_MAX_PARTITION_TOKENS]: each sequence is cut
 *                 into ceil(L / P) partitions that run in parallel and are
 *                 merged by a log-sum-exp combine (any P gives the same
 *                 result up to rounding)
 *   flags         0, or PKV_DECODE_FORCE_SIMT and/or PKV_DECODE_NO_CLUSTER.
 *                 When contexts are split into 2..16 partitions and every
 *                 (sequence, kv head) can have its own cluster of that many
 *                 CTAs resident at once (small batches), the partitions of a
 *                 (sequence, kv head) run as one thread-block cluster and are
 *                 merged through distributed shared memory, without the
 *                 workspace partials and the combine kernel (same result
 *                 within tolerance); PKV_DECODE_NO_CLUSTER turns that off
 *   device_error  device int32 or NULL
 *   stream        cudaStream_t
 * num_seqs == 0 returns PKV_OK and launches nothing; num_seqs is at most
 * PKV_MAX_SEQS_PER_CALL.
 */
pkv_status pkv_paged_attention_decode(const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, const int32_t* context_lens,
                                      void* out, void* workspace, size_t workspace_bytes,
                                      int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                                      int64_t head_dim, int64_t num_blocks, int64_t block_size,
                                      int64_t max_blocks_per_seq, int32_t kv_dtype,
                                      int32_t out_dtype, float scale, int32_t partition_tokens,
                                      uint32_t flags, int32_t* device_error, void* stream);

/*
 * pkv_decode_step -- one whole decode step in ONE launch: the effect of
 * pkv_kv_append (one new token per sequence) followed by
 * pkv_paged_attention_decode.
 *
 * Source: "warpllama", Milestones (static KV cache + single-token decode;
 * fused RoPE; the attention hot path as one hand-written CUDA kernel);
 * "Inference From Scratch", ch. 4 and ch. 10 (the new token's K/V go into its
 * sequence's cache block, then the token attends to the whole cache).
 *
 * Token b of the append is sequence b's new token.  The decode kernel
 * rotates each work item's staged q once in shared memory before its MMA
 * fragments are built, and the CTA that holds a sequence's last cache page
 * rotates the new k, writes k and v into the slot and patches them into the
 * staged page, so no separate append launch and no extra pass over memory is
 * needed.  Here the angle is
 * reduced mod 2pi in fp64 but its sine, cosine and the rotation are fp32,
 * rounded once to the storage type: within one storage ulp of the fp64 result
 * pkv_kv_append produces (bit-equal in the vast majority of elements).  q itself is only read:
 * unlike pkv_kv_append, the step does not store the rotated q (it is used
 * inside the kernel only), so q can be shared by all partitions at once.
 *
 * Precondition: the new token is the last token of its context, i.e.
 * context_lens[b] >= 1 and slot_mapping[b] is the slot that block_tables[b]
 * gives token context_lens[b] - 1.  A sequence whose slot_mapping[b] is
 * negative is not appended (its cached context is attended as is); one whose
 * slot differs from that table slot gets PKV_DEVERR_SLOT and is not appended
 * either.  A context of length 0 gives an all-zero output row and the token
 * is appended as pkv_kv_append would.
 *
 * Arguments: those of the two calls (q [num_seqs, Hq, d], read only;
 * k_new, v_new [num_seqs, Hkv, d]; positions, slot_mapping
 * [num_seqs] int64), one dtype for q, the new rows and the cache.  The
 * workspace is sized and owned exactly as for pkv_paged_attention_decode.
 */
pkv_status pkv_decode_step(void* q, const void* k_new, const void* v_new,
                           const int64_t* positions, const int64_t* slot_mapping,
                           void* k_cache, void* v_cache, const int32_t* block_tables,
                           const int32_t* context_lens, void* out, void* workspace,
                           size_t workspace_bytes, int64_t num_seqs, int64_t num_q_heads,
                           int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                           int64_t block_size, int64_t max_blocks_per_seq, int32_t kv_dtype,
                           int32_t out_dtype, double rope_theta, float scale,
                           int32_t partition_tokens, uint32_t flags, int32_t* device_error,
                           void* stream);

/*
 * pkv_decode_step_window -- pkv_decode_step with a sliding window.
 *
 * Source: "Efficient LLM Inference", KV Caching: positions and windows.
 *
 * The same single launch as pkv_decode_step (the new token appended inside
 * the decode kernel), but each query attends only to the last
 * `sliding_window` tokens of its context, its own new token included, as in
 * pkv_paged_attention_decode_window: pages wholly before the window are
 * never read, and keys before it in its first page are masked.
 * sliding_window = 0 is no window (the call is then pkv_decode_step);
 * negative values return PKV_ERR_INVALID_ARG.  Every other argument,
 * precondition and error is pkv_decode_step's.
 */
pkv_status pkv_decode_step_window(void* q, const void* k_new, const void* v_new,
                                  const int64_t* positions, const int64_t* slot_mapping,
                                  void* k_cache, void* v_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, void* out, void* workspace,
                                  size_t workspace_bytes, int64_t num_seqs, int64_t num_q_heads,
                                  int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                                  int64_t block_size, int64_t max_blocks_per_seq,
                                  int32_t kv_dtype, int32_t out_dtype, double rope_theta,
                                  float scale, int32_t sliding_window, int32_t partition_tokens,
                                  uint32_t flags, int32_t* device_error, void* stream);

/* Bytes of the built-in scratch behind pkv_paged_attention_decode_noalloc.
 * Every GPU that loads the library holds this much device memory until the
 * process exits. */
#define PKV_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * pkv_paged_attention_decode_noalloc -- pkv_paged_attention_decode for callers
 * that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot hand the library a workspace.  Typical examples: a serving
 * engine that has reserved nearly all device memory for its KV block pool and
 * may not allocate on the decode path; a plugin interface that passes only
 * input and output buffers; a C host without a device allocator, for which a
 * cudaMalloc per step would also synchronise the device.
 *
 * Same arguments, layout, result and errors as pkv_paged_attention_decode,
 * minus the workspace.  The split-context scratch lives in one file-scope
 * device array of PKV_NOALLOC_SCRATCH_BYTES per GPU instead; this call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   * Shapes whose scratch need (pkv_decode_workspace_size) exceeds
 *     PKV_NOALLOC_SCRATCH_BYTES are rejected with PKV_ERR_WORKSPACE before any
 *     launch; a larger partition_tokens lowers the need.
 *   * The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress); make that first call before any stream
 *     capture.
 *   * Every call on a device shares the one array.  Its scheduler counters
 *     start at zero (static storage) and every call leaves them zero; the
 *     rest keeps the last call's partials.  Calls that can overlap on the GPU
 *     (other streams, other host threads) race on it: serialise them, or
 *     give each its own workspace through pkv_paged_attention_decode.
 */
pkv_status pkv_paged_attention_decode_noalloc(const void* q, const void* k_cache,
                                              const void* v_cache, const int32_t* block_tables,
                                              const int32_t* context_lens, void* out,
                                              int64_t num_seqs, int64_t num_q_heads,
                                              int64_t num_kv_heads, int64_t head_dim,
                                              int64_t num_blocks, int64_t block_size,
                                              int64_t max_blocks_per_seq, int32_t kv_dtype,
                                              int32_t out_dtype, float scale,
                                              int32_t partition_tokens, uint32_t flags,
                                              int32_t* device_error, void* stream);

/*
 * The 8-bit cache.
 *
 * Source: "Efficient LLM Inference", "Quantization: From Rounding Errors to
 * Model-quality Limits" (values rounded to a small set of levels with a
 * scale) and "Verify Exact Execution and Approximate Quality Separately";
 * "From KV Elements to Memory Accounting and Admission Budgets" (cache
 * bytes per token set how many requests fit).  The element format is the
 * OCP 8-bit floating point E4M3 format (1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, no infinities, largest finite 448), which the pages do
 * not name.  One scale per tensor: the cached value is code x k_scale (K) or
 * code x v_scale (V).
 *
 * Layout (uint8): one buffer kv_cache [num_blocks, Hkv, 2, block_size *
 * head_dim]; each (block, kv head) page is one contiguous region of
 * 2 x 16 x head_dim bytes:
 *   K half  [block_size][head_dim]   (rows as in the bf16 cache)
 *   V half  [head_dim][block_size]   (transposed)
 * so that one copy fetches a page's K and V (one 2 KiB request at
 * head_dim 64), and the transposed V half lets the decode's tensor-core tile
 * read the four tokens a lane needs as four consecutive bytes.  Token t of
 * block b, kv head h: K at kv_cache + ((b Hkv + h) 2 + 0) 16 d + (t % 16) d,
 * V dim i at kv_cache + ((b Hkv + h) 2 + 1) 16 d + i 16 + t % 16.
 */

/*
 * pkv_kv_append_e4m3 -- pkv_kv_append into the 8-bit cache.
 *
 * q is rotated in place and rounded to its own dtype exactly as by
 * pkv_kv_append.  For a token with slot s >= 0 and every kv head h, dim i:
 *   K half of page (s / bs, h), row s % bs, byte i  <- code(rope(k_new[t, h, :], p)[i] / k_scale)
 *   V half of page (s / bs, h), byte i * 16 + s % bs <- code(v_new[t, h, i] / v_scale)
 * where the division is fp64, its result is rounded to binary32 and code()
 * is the nearest E4M3 value of that binary32 number, ties to even,
 * saturating to +-448 (cvt.rn.satfinite).
 *
 * Arguments: those of pkv_kv_append, with
 *   dtype              PKV_DTYPE_F32 or PKV_DTYPE_BF16: q, k_new, v_new
 *   kv_cache           device uint8, the layout above (16-byte aligned)
 *   k_scale, v_scale   finite, > 0
 */
pkv_status pkv_kv_append_e4m3(void* q, const void* k_new, const void* v_new,
                              const int64_t* positions, const int64_t* slot_mapping,
                              void* kv_cache, int64_t num_tokens,
                              int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
                              int64_t num_blocks, int64_t block_size, int32_t dtype,
                              double rope_theta, float k_scale, float v_scale,
                              int32_t* device_error, void* stream);

/*
 * pkv_paged_attention_decode_e4m3 -- pkv_paged_attention_decode over the 8-bit
 * cache: the same definition with K_b[t][i] = code x k_scale and
 * V_b[t][i] = code x v_scale.
 *
 * The tensor-core tiles run as f16 MMAs: every E4M3 value is exact in f16;
 * q (bf16) is rounded to f16, which is exact for |q| in [2^-17, 65504] (q
 * entries must stay below 65504 in magnitude; smaller ones lose at most
 * 2^-25 absolutely); P is split into two f16 terms; accumulation is fp32.
 * Workspace, partitioning, cluster merging, flags (except
 * PKV_DECODE_FORCE_SIMT, which is not supported here) and errors are those of
 * pkv_paged_attention_decode; size the workspace with kv_dtype
 * PKV_DTYPE_E4M3.
 *
 * Arguments: those of pkv_paged_attention_decode, with
 *   q                  device, [num_seqs, Hq, head_dim] bf16
 *   kv_cache           device uint8, the layout above (16-byte aligned)
 *   k_scale, v_scale   finite, > 0
 *   sliding_window     0, or a window as in pkv_paged_attention_decode_window
 */
pkv_status pkv_paged_attention_decode_e4m3(const void* q, const void* kv_cache,
                                           const int32_t* block_tables,
                                           const int32_t* context_lens, void* out,
                                           void* workspace, size_t workspace_bytes,
                                           int64_t num_seqs, int64_t num_q_heads,
                                           int64_t num_kv_heads, int64_t head_dim,
                                           int64_t num_blocks, int64_t block_size,
                                           int64_t max_blocks_per_seq, int32_t out_dtype,
                                           float scale, float k_scale, float v_scale,
                                           int32_t sliding_window, int32_t partition_tokens,
                                           uint32_t flags, int32_t* device_error, void* stream);

/*
 * pkv_decode_step_e4m3 -- pkv_decode_step over the 8-bit cache: the effect of
 * pkv_kv_append_e4m3 (one new token per sequence, bf16 inputs) followed by
 * pkv_paged_attention_decode_e4m3, in ONE launch.
 *
 * Source: "warpllama", Milestones (single-token decode with the attention
 * hot path fused); "Efficient LLM Inference", Quantization (values stored as
 * a small set of levels times a scale).
 *
 * The CTA that holds a sequence's last cache page rotates the new k in fp64
 * and writes the new k and v codes into the slot and into the staged page
 * exactly as pkv_kv_append_e4m3 computes them, so the cache bytes after the
 * step equal those after the two calls.  q is only read: the kernel rotates
 * its staged copy in fp32 (angle reduced in fp64) and rounds it to bf16, as
 * the append would store it; the result is within one bf16 ulp of that q.  Preconditions, the handling of slots that differ
 * from the table's, contexts of length 0 and every error are those of
 * pkv_decode_step.
 *
 * Arguments: those of pkv_decode_step (q, k_new, v_new bf16, read only), with
 *   kv_cache           device uint8, the layout above (16-byte aligned)
 *   k_scale, v_scale   finite, > 0
 *   sliding_window     0, or a window as in pkv_decode_step_window
 * Size the workspace with kv_dtype PKV_DTYPE_E4M3.
 */
pkv_status pkv_decode_step_e4m3(void* q, const void* k_new, const void* v_new,
                                const int64_t* positions, const int64_t* slot_mapping,
                                void* kv_cache, const int32_t* block_tables,
                                const int32_t* context_lens, void* out, void* workspace,
                                size_t workspace_bytes, int64_t num_seqs, int64_t num_q_heads,
                                int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                                int64_t block_size, int64_t max_blocks_per_seq, int32_t out_dtype,
                                double rope_theta, float scale, float k_scale, float v_scale,
                                int32_t sliding_window, int32_t partition_tokens, uint32_t flags,
                                int32_t* device_error, void* stream);

/*
 * pkv_paged_attention_decode_window -- pkv_paged_attention_decode with a
 * sliding window: each sequence's query attends to the last
 * min(sliding_window, L) tokens of its context only, tokens
 * max(0, L - sliding_window) .. L - 1 (itself included).
 *
 * Source: "Efficient LLM Inference", "KV Caching: Verify Reuse, Positions and
 * Windows" (position windows on the cache; the window's exact extent is this
 * library's reading).  Pages that lie wholly before the window are not read:
 * a sequence's partitions start at the page of its window's first token, and
 * the tokens before it in that page are masked.
 *
 * Arguments: those of pkv_paged_attention_decode, plus
 *   sliding_window     >= 0; 0 = the whole context (the plain decode)
 * The workspace is sized as for pkv_paged_attention_decode (the same shapes
 * and partition_tokens).
 */
pkv_status pkv_paged_attention_decode_window(const void* q, const void* k_cache,
                                             const void* v_cache, const int32_t* block_tables,
                                             const int32_t* context_lens, void* out,
                                             void* workspace, size_t workspace_bytes,
                                             int64_t num_seqs, int64_t num_q_heads,
                                             int64_t num_kv_heads, int64_t head_dim,
                                             int64_t num_blocks, int64_t block_size,
                                             int64_t max_blocks_per_seq, int32_t kv_dtype,
                                             int32_t out_dtype, float scale,
                                             int32_t sliding_window, int32_t partition_tokens,
                                             uint32_t flags, int32_t* device_error,
                                             void* stream);

/*
 * pkv_paged_attention_decode_cascade -- pkv_paged_attention_decode for batches
 * whose sequences share prefix blocks (prefix caching): each shared prefix is
 * read once for its whole group.
 *
 * Source: "Inference From Scratch", ch. 11 (prefix caching: requests with a
 * common prefix reuse its KV blocks) and ch. 10 (paged attention through
 * block tables, which is what lets several sequences point at the same
 * physical blocks); ch. 8 (attention over a split context merges exactly
 * through (max, sum) partials).
 *
 * Groups are runs of consecutive sequences: group g is sequences
 * [group_start[g], group_start[g + 1]).  shared_tokens[b] (rounded down to
 * whole blocks and clamped to the context) is how many leading tokens of
 * sequence b lie in blocks its group shares: for j < shared_tokens[b] /
 * block_size, block_tables[b, j] must equal the entry j of the group member
 * with the most shared tokens (a mismatch sets PKV_DEVERR_PREFIX; the
 * shared pass then reads that member's blocks).  Sequences in no group use
 * shared_tokens[b] = 0 (and may be left out of every group).
 *
 * The result is that of pkv_paged_attention_decode on the same arguments
 * (same definition, up to rounding).  Work: a shared-prefix pass runs one
 * item per (group, kv head) whose rows are all the group's query heads over
 * the shared pages; the decode kernel covers each sequence's remaining
 * tokens; a combine merges both.
 *
 * Arguments: as pkv_paged_attention_decode, plus
 *   group_start   device int32 [num_groups + 1], non-decreasing, <= num_seqs
 *   shared_tokens device int32 [num_seqs]
 *   max_group_size  the largest group_start[g + 1] - group_start[g]
 *   workspace     >= pkv_decode_cascade_workspace_size(...) bytes, first 256
 *                 bytes zero before its first call (as for the decode)
 * kv_dtype must be PKV_DTYPE_BF16; num_seqs <= 256; flags 0 or
 * PKV_DECODE_FORCE_SIMT (for the per-sequence part).  q must already be
 * rotated (pkv_kv_append).
 */
pkv_status pkv_paged_attention_decode_cascade(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* context_lens, const int32_t* group_start, const int32_t* shared_tokens,
    void* out, void* workspace, size_t workspace_bytes, int64_t num_seqs, int64_t num_groups,
    int64_t max_group_size, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
    int64_t num_blocks, int64_t block_size, int64_t max_blocks_per_seq, int32_t kv_dtype,
    int32_t out_dtype, float scale, int32_t partition_tokens, uint32_t flags,
    int32_t* device_error, void* stream);

/*
 * pkv_paged_attention_decode_cascade_window -- the cascade decode with a
 * sliding window.
 *
 * Source: "Efficient LLM Inference", KV Caching: positions and windows;
 * "Inference From Scratch", ch. 11 (prefix caching by block reuse).
 *
 * The result of pkv_paged_attention_decode_window: each query attends to the
 * last `sliding_window` tokens of its context.  The shared-prefix pass gives
 * each member only the shared tokens inside its own window (none when its
 * window starts past them: its shared slot is then an empty partial), and
 * reads the group's shared pages from the first page any member's window
 * reaches; the per-sequence part starts at the later of the shared prefix's
 * end and the window's page.  sliding_window = 0 is no window (the call is
 * then pkv_paged_attention_decode_cascade); negative values return
 * PKV_ERR_INVALID_ARG.  Every other argument, precondition, the workspace and
 * every error are pkv_paged_attention_decode_cascade's.
 */
pkv_status pkv_paged_attention_decode_cascade_window(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* context_lens, const int32_t* group_start, const int32_t* shared_tokens,
    void* out, void* workspace, size_t workspace_bytes, int64_t num_seqs, int64_t num_groups,
    int64_t max_group_size, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
    int64_t num_blocks, int64_t block_size, int64_t max_blocks_per_seq, int32_t kv_dtype,
    int32_t out_dtype, float scale, int32_t sliding_window, int32_t partition_tokens,
    uint32_t flags, int32_t* device_error, void* stream);

/* Bytes of workspace pkv_paged_attention_decode_cascade needs: 256 bytes of
 * scheduler counters, then num_seqs * Hq * (NP + 1) * (head_dim + 2) floats
 * of partials.  Host only; 0 for invalid arguments. */
size_t pkv_decode_cascade_workspace_size(int64_t num_seqs, int64_t num_q_heads,
                                         int64_t num_kv_heads, int64_t head_dim,
                                         int64_t max_blocks_per_seq, int64_t block_size,
                                         int32_t kv_dtype, int32_t partition_tokens);

/*
 * pkv_paged_attention_prefill -- chunked prefill: several query tokens per
 * sequence attend causally to the paged cache.
 *
 * Source: "Efficient LLM Inference", KV Caching: Verify Reuse, Positions and
 * Windows (a prompt computed in chunks over the retained keys and values
 * must equal the full-prefix forward pass); "llm-inference-from-scratch",
 * M1 (prefill/decode equivalence); "Inference From Scratch", ch. 8 and
 * ch. 10 (online softmax; paged attention through block tables).
 *
 * The chunk of sequence b is its last C = chunk_tokens context tokens: their
 * K/V are already in the cache (appended with pkv_kv_append, e.g. with
 * positions L_b - C .. L_b - 1), and their rotated queries are q[b, 0..C-1].
 * For b < num_seqs, i < C, h < Hq, with L = context_lens[b], kvh = h / G:
 *   out[b, i, h, :] = sum_{t <= L-C+i} exp(s_t - max s) V_b[t] / sum_t exp(s_t - max s),
 *   s_t = scale * <q[b, i, h, :], K_b[t]>,
 * i.e. pkv_paged_attention_decode of query i with context length L - C + i + 1.
 * With sliding_window = W > 0 the sum runs over L-C+i-W < t <= L-C+i only
 * (query i's last W tokens, as in pkv_paged_attention_decode_window); pages
 * before the chunk's first window are not read.
 * fp32 arithmetic (bf16 inputs widen exactly), P applied as a two-term bf16
 * split on the tensor cores, the result rounded once to out_dtype.
 *
 * Arguments
 *   q             device, [num_seqs, C, Hq, head_dim] bf16
 *   k_cache, v_cache  device, [num_blocks, Hkv, block_size, head_dim] bf16
 *   block_tables  device, [num_seqs, max_blocks_per_seq] int32
 *   context_lens  device, [num_seqs] int32 in [C, max_blocks_per_seq * block_size],
 *                 the chunk included (a shorter one sets PKV_DEVERR_CONTEXT_LEN
 *                 and its rows are not written)
 *   out           device, [num_seqs, C, Hq, head_dim], f32 or bf16
 *   workspace     device, >= pkv_prefill_workspace_size(...) bytes (NULL when
 *                 that is 0); contents need no initialisation
 *   sliding_window  0 (whole causal prefix) or W > 0 (the last W tokens)
 *   partition_tokens  0 = library choice (pkv_prefill_partition_tokens), else a
 *                 multiple of block_size in [block_size, PKV_MAX_PARTITION_TOKENS]
 * kv_dtype must be PKV_DTYPE_BF16.  num_seqs == 0 returns PKV_OK and launches
 * nothing.  Errors as for pkv_paged_attention_decode.
 */
pkv_status pkv_paged_attention_prefill(const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, const int32_t* context_lens,
                                       void* out, void* workspace, size_t workspace_bytes,
                                       int64_t num_seqs, int64_t chunk_tokens,
                                       int64_t num_q_heads, int64_t num_kv_heads,
                                       int64_t head_dim, int64_t num_blocks, int64_t block_size,
                                       int64_t max_blocks_per_seq, int32_t kv_dtype,
                                       int32_t out_dtype, float scale, int32_t sliding_window,
                                       int32_t partition_tokens, int32_t* device_error,
                                       void* stream);

/* Bytes of workspace pkv_paged_attention_prefill needs (partition partials:
 * num_seqs * C * Hq * NP * (head_dim + 2) floats when NP > 1, else 0).  Host
 * only; 0 also for invalid arguments. */
size_t pkv_prefill_workspace_size(int64_t num_seqs, int64_t chunk_tokens, int64_t num_q_heads,
                                  int64_t num_kv_heads, int64_t head_dim,
                                  int64_t max_blocks_per_seq, int64_t block_size,
                                  int32_t partition_tokens);

/* The partition length a prefill call with partition_tokens = 0 uses.  Host
 * only; 0 for invalid arguments. */
int32_t pkv_prefill_partition_tokens(int64_t num_seqs, int64_t chunk_tokens, int64_t num_q_heads,
                                     int64_t num_kv_heads, int64_t head_dim,
                                     int64_t max_blocks_per_seq, int64_t block_size);

/*
 * Block manager: the host side of a paged KV cache -- which physical blocks
 * each sequence owns, with prefix caching and eviction.
 *
 * Source: "Inference From Scratch", ch. 10 (block pool, block tables, slot
 * mapping) and ch. 11 (prefix caching, hash-based reuse of the KV blocks of
 * a common prefix); "The Project: Serve Your Own LLM", M13c (a pool smaller
 * than the worst case, so the engine must preempt).
 *
 * A full block (block_size tokens) is published under its tokens and the
 * blocks before it; a later sequence whose prompt starts with the same
 * tokens reuses those blocks (exact token comparison: no false sharing).
 * Blocks are reference counted; a published block nobody uses stays cached
 * until the pool needs it (least recently released first).  A partial last
 * block is always private.  Host memory only, no CUDA; not thread safe.
 * Statuses: PKV_ERR_INVALID_ARG (bad handle, unknown or duplicate sequence,
 * short output buffer), PKV_ERR_WORKSPACE (out of blocks: free a sequence,
 * i.e. preempt, and retry; nothing was allocated).
 */
typedef struct pkv_block_manager pkv_block_manager;

/* A manager of num_blocks blocks of block_size tokens; NULL on error. */
pkv_block_manager* pkv_bm_create(int32_t num_blocks, int32_t block_size);
void pkv_bm_destroy(pkv_block_manager* bm);

/* Admit a sequence with its prompt's token ids (host memory).  Cached blocks
 * covering the longest run of whole prompt blocks are reused;
 * *shared_tokens (may be NULL) receives the number of prompt tokens they
 * hold, whose K/V need not be computed again. */
pkv_status pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                               int64_t num_tokens, int32_t* shared_tokens);

/* Cache slot (block * block_size + row) of every prompt token of seq_id, -1
 * for tokens in reused blocks (pkv_kv_append skips negative slots). */
pkv_status pkv_bm_prompt_slots(const pkv_block_manager* bm, int64_t seq_id, int64_t* slots,
                               int64_t max_tokens);

/* Append one generated token: *slot receives its cache slot (a new block is
 * taken when the last one is full; a block that becomes full is published). */
pkv_status pkv_bm_append(pkv_block_manager* bm, int64_t seq_id, int32_t token, int64_t* slot);

/* Release a finished or preempted sequence's blocks. */
pkv_status pkv_bm_free_sequence(pkv_block_manager* bm, int64_t seq_id);

/* The sequence's block table row (padded with -1 to max_blocks), its block
 * count and token count; table may be NULL to query the counts. */
pkv_status pkv_bm_block_table(const pkv_block_manager* bm, int64_t seq_id, int32_t* table,
                              int32_t max_blocks, int32_t* num_blocks, int64_t* num_tokens);

/* Prompt tokens the sequence found in cached blocks (-1: unknown sequence). */
int32_t pkv_bm_shared_tokens(const pkv_block_manager* bm, int64_t seq_id);

/* Blocks available to new tokens (free + cached but unused), and cached
 * (published) blocks; -1 for a NULL handle. */
int32_t pkv_bm_free_blocks(const pkv_block_manager* bm);
int32_t pkv_bm_cached_blocks(const pkv_block_manager* bm);

/*
 * KV memory accounting, before any allocation ("Efficient LLM Inference",
 * From KV Elements to Memory Accounting and Admission Budgets).  Host only.
 *
 * pkv_kv_request_bytes: cache bytes a request of `tokens` tokens occupies
 * over `num_layers` layers: ceil(tokens / block_size) blocks, each
 * num_layers * 2 (K and V) * num_kv_heads * block_size * head_dim elements
 * of kv_dtype (PKV_DTYPE_F32 / _BF16 / _E4M3).  E.g. 16 layers, 8 kv heads,
 * head_dim 64, bf16: 32 KiB per token, 64 MiB for 2048 tokens.
 *
 * pkv_kv_admission_capacity: how many such requests fit in `pool_bytes`
 * (floor).
 *
 * Both return -1 for invalid arguments (or an overflowing size).
 */
int64_t pkv_kv_request_bytes(int64_t num_layers, int64_t num_kv_heads, int64_t head_dim,
                             int64_t block_size, int64_t tokens, int32_t kv_dtype);
int64_t pkv_kv_admission_capacity(int64_t pool_bytes, int64_t num_layers, int64_t num_kv_heads,
                                  int64_t head_dim, int64_t block_size, int64_t tokens,
                                  int32_t kv_dtype);

/*
 * pkv_get_device_error -- wait for a stream and read the device error word.
 *
 * Source: "Inference From Scratch", ch. 10 (block tables: every id a kernel
 * reads comes from the table, so a bad entry must be reported, not followed).
 *
 * Waits until all work enqueued on `stream` so far has finished (a
 * cudaStreamSynchronize: call it between steps, not inside a captured
 * graph), then copies the word at `device_error` (the int32 device word the
 * kernels OR their PKV_DEVERR_* bits into) to *code_out.  The word is left as
 * it is; the caller clears it (e.g. cudaMemsetAsync) when it wants a fresh
 * one.
 *
 * Arguments
 *   device_error  int32 device word (required).
 *   stream        cudaStream_t the kernels ran on (NULL = legacy default).
 *   code_out      HOST int32, receives the word.
 * Returns PKV_OK when the word is 0, PKV_ERR_DEVICE when it is not (the bits
 * are in *code_out and named by pkv_last_error), PKV_ERR_INVALID_ARG for a
 * null pointer, PKV_ERR_CUDA when the copy or the synchronisation fails
 * (e.g. a fault of earlier work on the stream).
 */
pkv_status pkv_get_device_error(const int32_t* device_error, void* stream, int32_t* code_out);

/*
 * pkv_selftest_bounded_wait -- run the kernels' bounded wait until it gives up.
 *
 * A diagnostic with no counterpart in the pages.  Every in-kernel wait of
 * this library (the page pipeline's shared-memory barriers) gives up after a
 * bounded time, sets PKV_DEVERR_TIMEOUT and lets the kernel return, so a
 * stalled copy can never hang a GPU.  This launches one warp that waits, with
 * that same code, on a barrier nothing ever completes, for `limit_us`
 * microseconds (1 .. 2 000 000), then ORs PKV_DEVERR_TIMEOUT into
 * *device_error and, if `waited_ns` is not NULL, stores the waited time
 * (int64 device word, nanoseconds).  Asynchronous on `stream`.
 * Returns PKV_ERR_INVALID_ARG for a limit outside the range or a null
 * device_error, PKV_ERR_CUDA if the launch fails.
 */
pkv_status pkv_selftest_bounded_wait(uint32_t limit_us, int32_t* device_error,
                                     uint64_t* waited_ns, void* stream);

/* Short text for a status code (static storage). */
const char* pkv_status_string(int32_t status);

/* Detail of the last non-OK status returned on the calling thread (static,
 * thread-local storage; empty when none). */
const char* pkv_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
