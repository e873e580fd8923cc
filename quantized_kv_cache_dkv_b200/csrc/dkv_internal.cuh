// Internal declarations shared by the host API and the kernels of libdkv.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dkv.h"

#include <nvtx3/nvToolsExt.h>

namespace dkv {

// Bounds checks of the bounds-checking build (DKV_BOUNDS_CHECK, built as
// libdkv_bc.so): DKV_IN_BOUNDS(cond, status) is `cond`, and records
// DKV_FLAG_BOUNDS in the sticky status when it fails, so the caller can skip
// the access.  In the normal build it is `true` and costs nothing.
#ifdef DKV_BOUNDS_CHECK
#define DKV_IN_BOUNDS(cond, status) \
  ((cond) ? true : (atomicOr((status), uint32_t(DKV_FLAG_BOUNDS)), false))
#else
#define DKV_IN_BOUNDS(cond, status) true
#endif

// Programmatic dependent launch.  Every kernel of the library is launched
// with launch_pdl, so the GPU may schedule it while the previous kernel of its
// stream is still running; it calls pdl_wait() before its first global memory
// access (the wait returns once the previous grid has completed and its
// writes are visible) and then pdl_trigger(), which lets the next kernel be
// scheduled as soon as every CTA of this grid has reached it.  What overlaps
// is only launch latency and setup that touches no global memory (shared
// memory barriers, TMEM allocation).  A dependent is scheduled only after all
// CTAs of its predecessor are resident, so early CTAs cannot starve it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KParams, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KParams...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Host-side NVTX range around one library call (header-only NVTX: it costs a
// few nanoseconds unless a profiler is attached, which then shows each call
// on the timeline).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kHeadDim = 128;
constexpr int kChunk = 32;  // token granularity of every segment boundary

// Device-side view of one cache.  Array layouts are the canonical ones of
// dkv.h with the capacity (not the length) as the token extent.
struct CacheView {
  int32_t B, Hq, Hkv, d, blk, g, rows;
  int32_t kb, vb, GK, GV, P;
  int64_t cap;     // tokens per unit
  int64_t nG;      // cap / GK (K groups per unit)
  int32_t kw;      // uint32 words per (K group, channel) = GK*kb/32
  int32_t vw;      // uint32 words per V token = d*vb/32
  int32_t vgroups; // d / GV
  int32_t twords;  // ceil(GK/32)
  int32_t U;

  uint32_t* k_codes;    // [U][nG][d][kw]
  __half2* k_sz;        // [U][nG][d]
  uint16_t* k_raw;      // [U][cap][d]          (kb == 16)
  uint16_t* k_tail;     // [U][GK][d]
  uint32_t* tail_mask;  // [U][twords]
  uint32_t* v_codes;    // [U][cap][vw]
  __half2* v_sz;        // [U][cap][vgroups]
  uint16_t* v_raw;      // [U][cap][d]          (vb == 16)
  int32_t* prot_count;  // [U]
  int32_t* prot_pos;    // [U][P]
  uint16_t* prot_k;     // [U][P][d]
  int32_t* prot_gstart; // [U][nG + 1]
  uint32_t* status;     // sticky DKV_FLAG_* bits
  int32_t sink;         // positions [0, sink) in full precision (K protected, V bf16)
  uint16_t* v_sink;     // [U][sink][d] bf16 V rows of the sink positions (vb < 16)
  // K-RPBH rotation of V (0: none): V rows are quantized in the rotated basis
  int32_t vrot_b;             // Hadamard block b in {16, 32, 64, 128}
  float vrot_norm;            // fp32(1 / sqrt(b))
  const int32_t* vrot_perm;   // [d] permutation: y[i] = x[perm[i]]
  const float* vrot_mix;      // [k][k] orthogonal mix, k = d / b
};

// Committed tokens of every sequence, passed by value to each launch (the
// host keeps the lengths; a CUDA graph captures them with the launch).
constexpr int kMaxSeqs = 512;
struct SeqLens {
  int32_t len[kMaxSeqs];
};

// Arguments of one attention call.
struct AttnArgs {
  CacheView c;
  SeqLens lens;           // committed tokens per sequence
  int32_t with_active;    // 1: the active block follows each sequence's tokens
  const uint16_t* q;      // [B][Hq][blk][d] bf16
  const uint16_t* k_act;  // [B][Hkv][blk][d] bf16
  const uint16_t* v_act;  // [B][Hkv][blk][d] bf16
  uint16_t* out;          // [B][Hq][blk][d] bf16
  __half* part_o;         // [U][nsplit][rows][d] fp16: the split's output divided by its row sum
  float2* part_ml;        // [U][nsplit][rows] (running max in log2 units, sum)
  float scale_log2;       // softmax_scale * log2(e)
  int64_t L;              // committed tokens of the longest sequence (planning)
  int64_t Lq;             // its tokens whose K is in complete groups (or raw)
  int64_t n_tok;          // L + blk (L without the active block)
  int32_t nsplit;
  int32_t tiles_per_split;  // in units of the kernel's token tile
  int32_t final_out;        // 1: the attention kernel writes bf16 out (one split,
                            // no rotation); 0: fp16 partials for combine_kernel
  int32_t part_base;        // split sp of unit u writes partial u*part_stride +
  int32_t part_stride;      // part_base + sp (one call: 0 and nsplit)
  // Attention over selected committed tokens (mma.sync kernel, gather = 1):
  // slot i < min(budget, L) of unit u is token sel[u * sel_ld + i]
  const int32_t* sel;
  int32_t sel_ld;
  int32_t budget;
  int32_t gather;
  int32_t tc_layout;        // tcgen05 kernel: 0 query-row blocks, 1 tokens on lanes (32 rows)
  uint64_t wait_limit_ns;   // limit of one bounded wait in the tcgen05 kernel
  int32_t test_stall_tile;  // bounds-checking build: tile whose copies the
                            // tcgen05 loader withholds (-1: none)
};

// Token counts of one unit (u = b * Hkv + h) in one attention call: L
// committed, Lq of them with K in complete groups (or raw), n_tok attended
// (L plus the active block when there is one).  Capacities are at most 2^30
// tokens, so 32 bits hold them.
struct UnitLen {
  int32_t L, Lq, n_tok;
};
__device__ __forceinline__ UnitLen unit_len(const AttnArgs& a, int u) {
  const int32_t L = a.lens.len[u / a.c.Hkv];
  UnitLen r;
  if (a.gather) {
    // the selected slots take the place of the committed tokens
    r.L = r.Lq = L < a.budget ? L : a.budget;
  } else {
    r.L = L;
    r.Lq = a.c.kb < 16 ? (L / a.c.GK) * a.c.GK : L;
  }
  r.n_tok = r.L + (a.with_active ? a.c.blk : 0);
  return r;
}

// One commit launch: the sequences that append a block (bit b of commit[]),
// each at its own position p0.len[b]; trunc[] marks sequences with a
// roll-back recorded since their last commit.
struct CommitArgs {
  SeqLens p0;
  uint32_t commit[kMaxSeqs / 32];
  uint32_t trunc[kMaxSeqs / 32];
};
cudaError_t launch_commit(const CacheView& c, const uint16_t* k, const uint16_t* v,
                          const uint32_t* pw, const CommitArgs& ca, cudaStream_t s);
// Applies recorded roll-backs (sequences with a trunc bit, to lens) to the
// side-table count and tail mask.
cudaError_t launch_truncate(const CacheView& c, const CommitArgs& ca, cudaStream_t s);
// The active block's V [U][blk][d] bf16 rotated like committed V rows (same
// fp32 order) and rounded to bf16 into dst (c.vrot_b > 0).
cudaError_t launch_rotate_v_rows(const CacheView& c, const uint16_t* src, uint16_t* dst,
                                 cudaStream_t s);

// mma.sync kernel: token tile of 64.
constexpr int kMmaTile = 64;
cudaError_t launch_attention_mma(const AttnArgs& a, cudaStream_t s);
cudaError_t launch_combine(const AttnArgs& a, cudaStream_t s);
// Q-MaskAhead selection (mma.sync kernels).  Scores: for every committed
// token j of unit u and row block rb, part[(u * nrb + rb) * ld + j] = (sum
// over the block's rows i of p_ij) * ||v_hat_j||, with p_ij the softmax weight
// of the whole call, from the split partials a.part_ml (a.with_active = 0).
int score_row_blocks(const CacheView& c);
cudaError_t launch_scores(const AttnArgs& a, float* part, int64_t ld, cudaStream_t s);
// Per unit: scores[u * ld + j] = sum over row blocks of part, then the
// min(budget, L) largest (ties: lower position) into sel[u * sel_ld + ...]
// in increasing position order, -1 after them.
cudaError_t launch_topk(const AttnArgs& a, const float* part, int64_t ld, float* scores,
                        int32_t* sel, cudaStream_t s);

// tcgen05 kernel: token tile of 128, rows == 128.
constexpr int kTcTile = 128;
bool tc_supported(const CacheView& c);
cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t s);

// Split workspace of one attention call: fp16 partial outputs (each split's
// output divided by its row sum) [U][splits][rows][d], then (max, sum)
// pairs in fp32 [U][splits][rows],
// starting at the next 256-byte boundary.  The handle's workspace and the
// no-allocation entry point's static buffer are both sized by these.
inline size_t split_o_bytes(int64_t U, int64_t splits, int64_t rows) {
  return (size_t(U) * size_t(splits) * size_t(rows) * kHeadDim * sizeof(__half) + 255) &
         ~size_t(255);
}
inline size_t split_ml_bytes(int64_t U, int64_t splits, int64_t rows) {
  return size_t(U) * size_t(splits) * size_t(rows) * sizeof(float2);
}

// Read-only view of a cache handle, and the thread-local error message, for
// entry points defined outside dkv_api.cu.
struct CacheInfo {
  CacheView v;
  int64_t len;       // the longest sequence's committed tokens
  SeqLens lens;      // every sequence's
  int device;  // CUDA device the cache was allocated on
  int num_sms;
  int32_t opt_splits, opt_kernel, max_splits;
  int32_t opt_test_stall;  // DKV_OPT_TEST_STALL (bounds-checking build), -1 = off
  uint16_t* vrot_act;  // [U][blk][d] rotated active-block V (when c.v.vrot_b > 0)
};
bool cache_info(const dkv_cache* c, CacheInfo* out);

// Launch plan of one attention call (kernel, split count, tiles per split);
// fills a->L, Lq, n_tok, nsplit, tiles_per_split.  Returns DKV_OK or an error
// code with *err set.
// with_active = false: the tokens are the committed ones only (no active
// block; the suffix cache of a dual-cache call).
int plan_attention(const CacheInfo& ci, AttnArgs* a, int* kernel, const char** err,
                   bool with_active = true);
int report_error(int code, const char* msg);
// DKV_OK when the current CUDA device is the cache's, else DKV_ERR_INVALID_ARG
// (or DKV_ERR_CUDA) with the error message set.
int check_device(const CacheInfo& ci);

}  // namespace dkv
