/*
 * libdkv -- quantize-on-commit and bidirectional block attention over a
 * low-bit block-diffusion KV cache, for NVIDIA B200 (sm_100a).
 *
 * The operations follow three passages of the source pages:
 *   - "SoloQ: Calibration-Free Quantization for Diffusion Language Models",
 *     block-diffusion paragraph: the cache is quantized when a block is
 *     committed and not before, the block under denoising keeps full
 *     precision, and K is quantized per channel on an asymmetric grid, as in
 *     KIVI.
 *   - "KV Cache Quantization for Diffusion Language Models" (Tai et al.,
 *     Findings of EMNLP 2026), abstract: KIVI carried over to prefix-cache
 *     reuse; KProtect holds a chosen set of K entries in high precision
 *     while V is stored at low bit width.
 *   - MaskAhead / Q-MaskAhead abstract: every denoising step of a block
 *     model reads the whole committed cache, and the quantized variant runs
 *     that attention on the low-bit cache itself.
 *
 * Quantizer of one group (b bits): s = fp16((max - min) / (2^b - 1)),
 * z = fp16(min), q = clamp(rint((x - z) / s), 0, 2^b - 1), all fp32 with
 * round-to-nearest-even; dequantized value q * s + z.  K groups are
 * k_group consecutive tokens of one channel (positions aligned to 0); V
 * groups are v_group consecutive channels of one token.  Protected K
 * positions are left out of their group's min/max, get code 0, and keep
 * their bf16 vector in a side table.
 *
 * Conventions for every call:
 *   - Return value: DKV_OK (0) or a DKV_ERR_* code.  On an error detected on
 *     the host no state changes and nothing is launched; dkv_last_error()
 *     gives a message (thread-local, valid until the next call).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Commit and
 *     attention are asynchronous and stream-ordered; alloc, free, status and
 *     export synchronize `stream`.
 *   - Caller buffers are device memory (cudaMalloc or torch), contiguous,
 *     16-byte aligned, bf16 = IEEE bfloat16 bit patterns.  The library keeps
 *     no caller pointer past the call.  Commit and attention calls run on the
 *     current CUDA device, which must be the one the cache was allocated on
 *     (else DKV_ERR_INVALID_ARG).
 *   - Errors found while kernels run (protected side table full, committed
 *     value out of fp16 range) are sticky flags read by dkv_cache_status.
 */
#ifndef DKV_H
#define DKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  DKV_OK = 0,
  DKV_ERR_INVALID_ARG = 1, /* NULL/misaligned pointer, bad size */
  DKV_ERR_UNSUPPORTED = 2, /* shape or bit width outside the built set */
  DKV_ERR_CAPACITY = 3,    /* len + block would exceed max_tokens */
  DKV_ERR_CUDA = 4         /* a CUDA runtime call failed */
};

/* sticky device-side flags (dkv_cache_status) */
enum {
  DKV_FLAG_CAPACITY = 0x1, /* side table full: later protected tokens were quantized normally */
  DKV_FLAG_RANGE = 0x2,    /* a committed K/V value was NaN/Inf or |x| > 65504; the
                              quantizer used NaN -> 0 and clamped to +-65504 */
  DKV_FLAG_TIMEOUT = 0x4,  /* an attention CTA gave up waiting on one of its own
                              pipeline stages (bounded wait, about 1 s); that call's
                              output is undefined */
  DKV_FLAG_BOUNDS = 0x8    /* bounds-checking build only (libdkv_bc.so, compiled
                              with DKV_BOUNDS_CHECK): an index or copy range failed
                              its check against its buffer and the access was
                              skipped; that call's results are undefined */
};

/* Cache shape.  Supported: head_dim == 128; block a multiple of 32, <= 128;
 * q_heads a multiple of kv_heads with (q_heads/kv_heads)*block <= 256;
 * k_bits, v_bits in {2, 3, 4, 16} (16 = store bf16, quantization off);
 * k_group in {32, 64, 128} with k_group % block == 0 or block % k_group == 0;
 * v_group in {32, 64, 128}; max_tokens a multiple of max(k_group, block). */
typedef struct dkv_config {
  int32_t batch;         /* B: sequences, at most 512 (each has its own committed
                            length; they stay equal unless dkv_commit_block_seqs or
                            dkv_cache_truncate_seq make them differ) */
  int32_t q_heads;       /* Hq */
  int32_t kv_heads;      /* Hkv; query head h reads kv-head h / (Hq/Hkv) */
  int32_t head_dim;      /* d */
  int32_t block;         /* blk: tokens per committed / active block */
  int32_t k_bits;        /* bK */
  int32_t v_bits;        /* bV */
  int32_t k_group;       /* GK: tokens per K group (per channel) */
  int32_t v_group;       /* GV: channels per V group (per token) */
  int32_t max_protected; /* side-table capacity per (sequence, kv-head) */
  int64_t max_tokens;    /* capacity per sequence */
  int32_t sink_tokens;   /* attention sink: positions [0, sink_tokens) of every
                            sequence stay in full precision -- K protected (a
                            side-table entry each, counted in max_protected),
                            V kept as bf16 beside its codes.  0 = none; at
                            most 256 and max_tokens.  At 2-bit KV keeping the
                            sink in full precision matters (SoloQ, KV-only
                            paragraph). */
  int32_t reserved;      /* must be 0 */
} dkv_config;

typedef struct dkv_cache dkv_cache; /* opaque; owns its device memory */

/* Allocate an empty cache (len = 0) on the current device.  Device memory is
 * owned by the handle until dkv_cache_free.  Synchronizes `stream`. */
int dkv_cache_alloc(const dkv_config* cfg, void* stream, dkv_cache** out);

/* Release the handle and its device memory (synchronizes the device). */
int dkv_cache_free(dkv_cache* cache);

/* Commit one block: k, v are bf16 [B, Hkv, block, d]; protect_words is a
 * device array uint32 [B, Hkv, block/32] whose bit t marks token t of the
 * block as a protected K position, or NULL for none.  V is quantized per
 * token at once; K tokens wait in a bf16 tail until their K group is
 * complete, then the group is quantized.  len grows by `block` (host side,
 * at once).  Returns DKV_ERR_CAPACITY if len + block > max_tokens. */
int dkv_commit_block(dkv_cache* cache, const void* k, const void* v,
                     const uint32_t* protect_words, void* stream);

/* Per-sequence lengths (sequences of one batch finish their blocks at
 * different denoising steps -- SoloQ, block-diffusion paragraph: each block is
 * quantized when it is committed).  Commit one block to the sequences listed
 * in `seqs` (host int32 array of n_seqs distinct indices in [0, B); n_seqs = 0
 * does nothing): each appends at its own committed length.  k, v and
 * protect_words have the shapes of dkv_commit_block; the rows of sequences not
 * listed are not read.  DKV_ERR_CAPACITY if a listed sequence would pass
 * max_tokens (nothing changes).  Attention then runs every sequence over its
 * own committed tokens plus its active block. */
int dkv_commit_block_seqs(dkv_cache* cache, const void* k, const void* v,
                          const uint32_t* protect_words, const int32_t* seqs,
                          int32_t n_seqs, void* stream);

/* Committed tokens of every sequence: lens is a host array of B entries
 * (host mirror, no synchronization). */
int dkv_cache_seq_lens(const dkv_cache* cache, int64_t* lens);

/* dkv_cache_truncate for one sequence: roll sequence `seq` back to new_len
 * (same rules as dkv_cache_truncate, against that sequence's length). */
int dkv_cache_truncate_seq(dkv_cache* cache, int32_t seq, int64_t new_len, void* stream);

/* One denoising-step attention: q bf16 [B, Hq, block, d], the active block
 * k_act, v_act bf16 [B, Hkv, block, d] (kept in full precision), out bf16
 * [B, Hq, block, d].  Every query attends to every committed token and every
 * active-block token (bidirectional, no mask): out = softmax(softmax_scale *
 * q K^T) V with K, V the dequantized cache, the bf16 K tail and the active
 * block; fp32 softmax, bf16 (round-to-nearest-even) output.  q, k_act,
 * v_act must hold values within the fp16 range. */
int dkv_block_attention(dkv_cache* cache, const void* q, const void* k_act,
                        const void* v_act, float softmax_scale, void* out,
                        void* stream);

/* Q-MaskAhead selection (MaskAhead / Q-MaskAhead abstract: the queries of the
 * block being denoised score the cached entries by their expected share of
 * the attention output, the block attends to the best-scored ones, and the
 * quantized variant scores and attends on the low-bit cache).  The abstract
 * gives no formula; the reading taken here: for every (sequence, kv-head)
 * unit and committed token j,
 *   c_j = (sum over the unit's query rows i of p_ij) * ||v_hat_j||_2,
 * p_ij the softmax weight of token j for row i in the full attention of this
 * call (committed tokens and active block, from the dequantized cache);
 * the min(budget, len) tokens of largest c_j are kept (equal scores: the
 * lower position first), and every query row attends to them plus the
 * whole active block: out = softmax(softmax_scale * q K_sel^T) V_sel, bf16.
 * Arguments as in dkv_block_attention, and:
 *   budget    tokens kept per unit, 0 <= budget <= max_tokens
 *   selected  device int32 [B, Hkv, budget], or NULL: the kept positions of
 *             each unit in increasing order, -1 after the last
 *   scores    device fp32 [B, Hkv, max_tokens], or NULL: c_j at [.., j] for
 *             j < the sequence's length
 * Launches: the split attention kernel (for each row's softmax max and sum),
 * a scoring kernel, a per-unit top-k kernel (radix select), the mma.sync
 * attention over the gathered tokens, and the combine when it splits.  The
 * first call on a handle allocates its workspace ([B*Hkv, max_tokens] x 3
 * fp32/int32 words); make it before any stream capture.  Not available on a
 * rotated-V cache (DKV_ERR_UNSUPPORTED); query groups must be a multiple of
 * 16 rows. */
int dkv_block_attention_selected(dkv_cache* cache, const void* q, const void* k_act,
                                 const void* v_act, float softmax_scale, int32_t budget,
                                 void* out, int32_t* selected, float* scores, void* stream);

/* Dual-cache attention (the prefix and dual cache reuse of Fast-dLLM-style
 * decoding that "KV Cache Quantization for Diffusion Language Models"
 * quantizes, abstract): the active block's queries attend to `prefix` (the
 * committed tokens before the block), the active block, and `suffix`, a second
 * cache holding the KV of the region after the block (for instance the masked
 * tokens of later blocks, refreshed with dkv_cache_truncate(suffix, 0) and new
 * commits).  out = softmax over all three segments, bidirectional, no mask;
 * each cache is dequantized with its own bit widths and groups (a bf16 suffix
 * uses bits = 16).  Arguments as in dkv_block_attention.  The two caches must
 * be on the same device and have the same batch, heads, head_dim and block
 * (else DKV_ERR_INVALID_ARG); neither may rotate V
 * (DKV_ERR_UNSUPPORTED), the suffix may not have a sink.  An empty suffix
 * gives exactly dkv_block_attention.  Launches: the split attention kernel on
 * each cache (the suffix with its own DKV_OPT_* choices) writing into the
 * prefix cache's split workspace, then one combine; no allocation.  Device
 * flags raised while reading the suffix are reported by the suffix handle. */
int dkv_block_attention_dual(dkv_cache* prefix, dkv_cache* suffix, const void* q,
                             const void* k_act, const void* v_act, float softmax_scale,
                             void* out, void* stream);

/* Rotated V (K-RPBH, "SoloQ: Calibration-Free Quantization for Diffusion
 * Language Models", K-RPBH paragraph and the KV-cache paragraph): committed V
 * rows are rotated by an orthogonal map R before their per-token
 * quantization, the active block's V is rotated the same way (and rounded to
 * bf16), and the attention output is rotated back, so the result is still
 * softmax(...) V in the original basis; only the quantization error changes.
 * For a row x of d = 128 channels and blocks of b channels (k = d / b):
 *   y[i] = x[perm[i]];  each block of y <- (block) H_b / sqrt(b) with H_b the
 *   Sylvester Hadamard matrix;  w[r*b + i] = sum_c mix[r*k + c] * y[c*b + i].
 * Evaluated in fp32 in a fixed order (butterflies over strides 1, 2, ...,
 * b/2; one multiply by fp32(1/sqrt(b)); the mix summed over c = 0..k-1 from
 * 0; no fused multiply-add), so the stored codes are reproducible bit for bit.
 *   perm  host int32 [128], a permutation of 0..127 (the caller's random draw)
 *   mix   host fp32 [k * k], row-major, orthogonal (|mix mix^T - I| <= 1e-4)
 *   block b in {16, 32, 64, 128}; block = 0 (perm, mix NULL) turns it off.
 * Call before the first commit (len == 0) of a cache with v_bits < 16 and
 * sink_tokens == 0.  The library copies the arguments (synchronously) and
 * allocates a [B, Hkv, block, d] bf16 buffer for the rotated active block,
 * so two attention calls on one handle must not overlap on the GPU.  Each
 * attention call then also launches a small rotation kernel and always the
 * combine kernel (which applies the inverse rotation in fp32).
 * Errors: DKV_ERR_INVALID_ARG (len > 0, NULL or non-permutation perm, NULL,
 * non-finite or non-orthogonal mix), DKV_ERR_UNSUPPORTED (block not in the
 * set, v_bits == 16, sink_tokens > 0), DKV_ERR_CUDA; nothing changes on an
 * error. */
int dkv_cache_set_v_rotation(dkv_cache* cache, const int32_t* perm, const float* mix,
                             int32_t block);

/* Roll the cache back to its first new_len committed tokens (for instance to
 * reuse a shared prefix, the prefix-cache reuse of the Tai et al. abstract).
 * new_len must be a multiple of `block` and, when k_bits < 16, of k_group, so
 * that no incomplete K group remains; 0 <= new_len <= len.  The side table
 * keeps the entries of the surviving groups.  len changes at once on the
 * host.  Every sequence is rolled back (new_len must not exceed any
 * sequence's length).  No kernel runs here: the device-side count of side-table entries
 * and the tail mask are reset by the next dkv_commit_block, or by
 * dkv_cache_export if that comes first (on its stream), which is all that
 * reads them; dkv_block_attention reads neither.  `stream` is unused. */
int dkv_cache_truncate(dkv_cache* cache, int64_t new_len, void* stream);

/* dkv_block_attention for callers that cannot call cudaMalloc -- code that
 * runs while a CUDA stream capture is active (cudaMalloc is a prohibited call
 * there and would invalidate the capture), or a plugin inside a host
 * application that owns and budgets all device memory.  The pages have no
 * counterpart to this call; it computes exactly what dkv_block_attention
 * computes, with the same arguments, launch plan and error codes, but takes
 * its split scratch (the per-split partial outputs merged by the combine
 * kernel) from a fixed buffer compiled into the library instead of the
 * handle's workspace, and allocates nothing: no cudaMalloc, cudaFree or
 * allocating library routine.  The cache handle is an input created
 * beforehand (dkv_cache_alloc).
 *   - The buffer is a static __device__ array of DKV_NOALLOC_SCRATCH_BYTES
 *     (16 MiB); every GPU that loads libdkv holds it until the process exits.
 *   - A plan needing more scratch than that (B*Hkv * splits *
 *     (q_heads/kv_heads)*block * (2*head_dim + 8) bytes, whenever the
 *     combine kernel runs: splits > 1, or a rotated-V cache) returns
 *     DKV_ERR_UNSUPPORTED with a message; lower DKV_OPT_SPLITS.
 *   - A rotated-V cache rotates the active block's V into the buffer the
 *     handle allocated in dkv_cache_set_v_rotation (no allocation here).
 *   - The first call on each device looks up the buffer's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - Every call on a device shares the one buffer, which keeps the last
 *     call's contents (each call overwrites what it reads).  Calls that
 *     overlap on the GPU -- on different streams without ordering between
 *     them -- race on it; serialize them. */
#define DKV_NOALLOC_SCRATCH_BYTES (16u << 20)
int dkv_block_attention_noalloc(dkv_cache* cache, const void* q, const void* k_act,
                                const void* v_act, float softmax_scale, void* out,
                                void* stream);

/* Committed tokens of the longest sequence (host mirror, no synchronization);
 * the committed length of every sequence when they are all equal. */
int dkv_cache_len(const dkv_cache* cache, int64_t* len);

/* Synchronize `stream`, return the sticky DKV_FLAG_* bits and clear them. */
int dkv_cache_status(dkv_cache* cache, void* stream, uint32_t* flags);

/* Host copies of the committed state in the canonical layout (U = B*Hkv
 * units, u = b*Hkv + h; L = len; Lq = tokens whose K group is complete,
 * = L when k_bits == 16; nG = Lq / k_group).  Every pointer is a host buffer
 * owned by the caller, or NULL to skip that array.  Synchronizes `stream`.
 *   k_codes   uint32 [U, nG, d, k_group*k_bits/32]  codes of one (group,
 *             channel) packed along its tokens, a little-endian bit stream:
 *             token t at bits [k_bits*t, +k_bits) of the stream, where bit i
 *             is bit i mod 32 of word i/32 (at 3 bits codes 10 and 21 of
 *             every 32 straddle two words)
 *   k_sz      uint16 [U, nG, d, 2]    fp16 (scale, zero) per (group, channel)
 *   k_raw     uint16 [U, L, d]        bf16 K when k_bits == 16
 *   k_tail    uint16 [U, L - Lq, d]   bf16 K of the incomplete group
 *   tail_mask uint32 [U, ceil(k_group/32)]  protect bits of the tail slots
 *   v_codes   uint32 [U, L, d*v_bits/32]    per token, packed along channels
 *   v_sz      uint16 [U, L, d/v_group, 2]   fp16 (scale, zero)
 *   v_raw     uint16 [U, L, d]        bf16 V when v_bits == 16
 *   prot_count  int32 [U]             side-table entries in use
 *   prot_pos    int32 [U, max_protected]    their positions, ascending
 *               (unused slots: -1)
 *   prot_k      uint16 [U, max_protected, d] their bf16 K vectors
 *   prot_gstart int32 [U, nG + 1]     entries stored before group j */
typedef struct dkv_export {
  uint32_t* k_codes;
  uint16_t* k_sz;
  uint16_t* k_raw;
  uint16_t* k_tail;
  uint32_t* tail_mask;
  uint32_t* v_codes;
  uint16_t* v_sz;
  uint16_t* v_raw;
  int32_t* prot_count;
  int32_t* prot_pos;
  uint16_t* prot_k;
  int32_t* prot_gstart;
  uint16_t* v_sink;      /* [U][min(sink_tokens, len)][d] bf16 (v_bits < 16) */
} dkv_export;

int dkv_cache_export(dkv_cache* cache, void* stream, dkv_export* out);

/* dkv_cache_export of one sequence: its Hkv units (U = kv_heads, in kv-head
 * order) at its own committed length.  dkv_cache_export itself requires all
 * sequences to have the same length (else DKV_ERR_INVALID_ARG). */
int dkv_cache_export_seq(dkv_cache* cache, int32_t seq, void* stream, dkv_export* out);

/* Tuning knobs (testing and benchmarking).  Values persist on the handle.
 *   DKV_OPT_SPLITS: token splits per (sequence, kv-head) in attention;
 *     0 = chosen from the SM count (default).  Results agree within fp32
 *     rounding for any split count.
 *   DKV_OPT_ATTN_KERNEL: 0 = best available (default: 2 where the shape has a
 *     tcgen05 variant, else 1), 1 = warp-level mma.sync kernel, 2 = tcgen05
 *     tensor-memory kernel with query-row blocks of up to 128 rows, 3 =
 *     tcgen05 with the tokens on the TMEM lanes, for 32-row query groups only
 *     (DKV_ERR_UNSUPPORTED for 2 and 3 where the shape has no such variant).
 *   DKV_OPT_TEST_STALL: bounds-checking build (libdkv_bc.so) only, else
 *     DKV_ERR_UNSUPPORTED.  A test of the bounded waits: value t >= 0 makes the
 *     tcgen05 kernel's loader withhold the copies of tile t (0 = the first
 *     tile of each CTA's token range), so the waits on that stage run out;
 *     while it is set every bounded wait gives up after 2 ms instead of about
 *     1 s.  The call then raises DKV_FLAG_TIMEOUT, every CTA leaves its
 *     loops, waits for its own copies and MMAs in flight and frees its tensor
 *     memory; the output is undefined.  -1 (default) turns it off. */
enum { DKV_OPT_SPLITS = 1, DKV_OPT_ATTN_KERNEL = 2, DKV_OPT_PROFILE = 3, DKV_OPT_TEST_STALL = 4 };
int dkv_cache_set_option(dkv_cache* cache, int32_t key, int64_t value);

/* With DKV_OPT_PROFILE = 1, every kernel launch on this handle (outside CUDA
 * graph capture) is bracketed by CUDA events recorded on its stream.  This
 * call waits for them and returns, per kernel kind, the summed device time in
 * milliseconds and the launch count since the last read, then resets them.
 * kind: DKV_KERNEL_ATTENTION (the split attention kernel; for
 * dkv_block_attention_selected also its scoring and top-k kernels and the
 * attention over the kept tokens), DKV_KERNEL_COMBINE,
 * DKV_KERNEL_COMMIT, DKV_KERNEL_TRUNCATE. */
enum { DKV_KERNEL_ATTENTION = 0, DKV_KERNEL_COMBINE = 1, DKV_KERNEL_COMMIT = 2,
       DKV_KERNEL_TRUNCATE = 3 };
int dkv_profile_read(dkv_cache* cache, int32_t kind, double* total_ms, int64_t* launches);

/* Launch description of the last dkv_block_attention (or
 * dkv_block_attention_dual, recorded on the prefix handle) on this handle:
 * the kernel used (1 = mma.sync, 2 or 3 = tcgen05 as in DKV_OPT_ATTN_KERNEL;
 * the prefix's for a dual call),
 * the split count (prefix + suffix splits for a dual call), and how many
 * kernels it launched (attention, plus the combine unless one split wrote
 * the output directly, plus the active-block rotation of a rotated-V cache;
 * 3 for a dual call). */
int dkv_last_attention_plan(const dkv_cache* cache, int32_t* kernel,
                            int32_t* splits, int32_t* launches);

/* Message of the last error on this thread ("" if none). */
const char* dkv_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* DKV_H */
