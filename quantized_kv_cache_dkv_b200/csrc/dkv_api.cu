// C-ABI entry points of libdkv: argument checks, device memory, split
// planning and kernel launches.  Every step of the path runs in the kernels
// of commit.cu, attn_mma.cu and attn_tc.cu; this file only plans and launches.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "dkv_internal.cuh"

namespace {
// CUDA events bracketing kernel launches (DKV_OPT_PROFILE)
struct ProfRecord {
  cudaEvent_t start, stop;
  int kind;
};
}  // namespace

struct dkv_cache {
  dkv_config cfg;
  dkv::CacheView v;
  int device = 0;
  int num_sms = 148;
  std::vector<int64_t> lens;       // committed tokens per sequence (the host is the authority)
  std::vector<char> trunc;         // a roll-back of that sequence not yet applied on the device
  void* arena = nullptr;
  size_t arena_bytes = 0;
  __half* part_o = nullptr;
  float2* part_ml = nullptr;
  void* sel_mem = nullptr;       // selection workspace (first dkv_block_attention_selected)
  void* vrot_mem = nullptr;      // rotation parameters + rotated active block (V rotation)
  uint16_t* vrot_act = nullptr;  // [U][blk][d] bf16
  int32_t max_splits = 1;
  int32_t opt_splits = 0;
  int32_t opt_kernel = 0;
  int32_t opt_test_stall = -1;
  int32_t last_kernel = 0, last_splits = 0, last_launches = 0;
  bool profile = false;
  std::vector<ProfRecord> prof;  // event pool; the first prof_used are pending
  size_t prof_used = 0;
};

namespace {

thread_local std::string g_err;

int fail(int code, const std::string& msg) {
  g_err = msg;
  return code;
}

#define DKV_CUDA(expr)                                                              \
  do {                                                                              \
    cudaError_t e_ = (expr);                                                        \
    if (e_ != cudaSuccess)                                                          \
      return fail(DKV_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(e_)); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int check_config(const dkv_config* c) {
  if (!c) return fail(DKV_ERR_INVALID_ARG, "config is NULL");
  if (c->batch < 1 || c->q_heads < 1 || c->kv_heads < 1 || c->head_dim < 1 || c->block < 1 ||
      c->max_tokens < 1 || c->max_protected < 0)
    return fail(DKV_ERR_INVALID_ARG, "non-positive size in config");
  if (c->batch > dkv::kMaxSeqs)
    return fail(DKV_ERR_UNSUPPORTED, "batch must be <= " + std::to_string(dkv::kMaxSeqs));
  if (c->q_heads % c->kv_heads)
    return fail(DKV_ERR_INVALID_ARG, "q_heads must be a multiple of kv_heads");
  if (c->head_dim != dkv::kHeadDim) return fail(DKV_ERR_UNSUPPORTED, "head_dim must be 128");
  if (c->block % 32 || c->block > 128)
    return fail(DKV_ERR_UNSUPPORTED, "block must be a multiple of 32 and <= 128");
  if ((c->q_heads / c->kv_heads) * c->block > 256)
    return fail(DKV_ERR_UNSUPPORTED, "(q_heads/kv_heads)*block must be <= 256");
  auto okbits = [](int b) { return b == 2 || b == 3 || b == 4 || b == 16; };
  if (!okbits(c->k_bits) || !okbits(c->v_bits))
    return fail(DKV_ERR_UNSUPPORTED, "k_bits/v_bits must be 2, 3, 4 or 16");
  auto okgrp = [](int g) { return g == 32 || g == 64 || g == 128; };
  if (c->k_bits < 16) {
    if (!okgrp(c->k_group)) return fail(DKV_ERR_UNSUPPORTED, "k_group must be 32, 64 or 128");
    if (c->k_group % c->block && c->block % c->k_group)
      return fail(DKV_ERR_UNSUPPORTED, "k_group and block must divide one another");
  }
  if (c->v_bits < 16 && !okgrp(c->v_group))
    return fail(DKV_ERR_UNSUPPORTED, "v_group must be 32, 64 or 128");
  int64_t unit = c->block;
  if (c->k_bits < 16) unit = std::max<int64_t>(unit, c->k_group);
  if (c->max_tokens % unit)
    return fail(DKV_ERR_INVALID_ARG, "max_tokens must be a multiple of max(k_group, block)");
  if (c->max_tokens > (int64_t(1) << 30))
    return fail(DKV_ERR_INVALID_ARG, "max_tokens too large (limit 2^30)");
  if (c->sink_tokens < 0 || c->sink_tokens > 256 || c->sink_tokens > c->max_tokens)
    return fail(DKV_ERR_INVALID_ARG, "sink_tokens must be in [0, min(256, max_tokens)]");
  if (c->reserved != 0) return fail(DKV_ERR_INVALID_ARG, "reserved must be 0");
  return DKV_OK;
}

// Runs `launch` on stream s; when profiling (and s is not capturing a graph)
// records a pair of events around it.
template <class F>
cudaError_t timed_launch(dkv_cache* c, int kind, cudaStream_t s, F&& launch) {
  bool rec = c->profile;
  if (rec) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &st) != cudaSuccess || st != cudaStreamCaptureStatusNone) rec = false;
  }
  if (!rec) return launch();
  if (c->prof_used == c->prof.size()) {
    ProfRecord r{};
    cudaError_t e = cudaEventCreate(&r.start);
    if (e == cudaSuccess) e = cudaEventCreate(&r.stop);
    if (e != cudaSuccess) return e;
    c->prof.push_back(r);
  }
  ProfRecord& r = c->prof[c->prof_used++];
  r.kind = kind;
  cudaError_t e = cudaEventRecord(r.start, s);
  if (e == cudaSuccess) e = launch();
  if (e == cudaSuccess) e = cudaEventRecord(r.stop, s);
  return e;
}

int64_t max_len(const dkv_cache* c) {
  int64_t m = 0;
  for (int64_t l : c->lens) m = std::max(m, l);
  return m;
}

bool any_trunc(const dkv_cache* c) {
  for (char t : c->trunc)
    if (t) return true;
  return false;
}

// lengths, commit set and roll-back marks of one commit / truncate launch
dkv::CommitArgs commit_args(const dkv_cache* c, const std::vector<char>& commits) {
  dkv::CommitArgs ca;
  std::memset(&ca, 0, sizeof(ca));
  for (size_t b = 0; b < c->lens.size(); ++b) {
    ca.p0.len[b] = int32_t(c->lens[b]);
    if (commits[b]) ca.commit[b >> 5] |= 1u << (b & 31);
    if (c->trunc[b]) ca.trunc[b >> 5] |= 1u << (b & 31);
  }
  return ca;
}

int split_cap(int U, int sms) {
  int64_t s = ceil_div(int64_t(8) * sms, U);
  return int(std::min<int64_t>(64, std::max<int64_t>(4, s)));
}

}  // namespace

namespace dkv {

bool cache_info(const dkv_cache* c, CacheInfo* out) {
  if (!c || !out) return false;
  out->v = c->v;
  out->len = max_len(c);
  std::memset(&out->lens, 0, sizeof(out->lens));
  for (size_t b = 0; b < c->lens.size(); ++b) out->lens.len[b] = int32_t(c->lens[b]);
  out->device = c->device;
  out->num_sms = c->num_sms;
  out->opt_splits = c->opt_splits;
  out->opt_kernel = c->opt_kernel;
  out->opt_test_stall = c->opt_test_stall;
  out->max_splits = c->max_splits;
  out->vrot_act = c->vrot_act;
  return true;
}

int report_error(int code, const char* msg) { return fail(code, msg); }

int check_device(const CacheInfo& ci) {
  int dev = -1;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev != ci.device)
    return fail(DKV_ERR_INVALID_ARG, "the current CUDA device (" + std::to_string(dev) +
                                         ") is not the cache's device (" + std::to_string(ci.device) + ")");
  return DKV_OK;
}

int plan_attention(const CacheInfo& ci, AttnArgs* a, int* kernel_out, const char** err,
                   bool with_active) {
  const CacheView& v = ci.v;
  a->L = ci.len;
  a->Lq = v.kb < 16 ? (ci.len / v.GK) * v.GK : ci.len;
  a->n_tok = ci.len + (with_active ? v.blk : 0);
  a->lens = ci.lens;
  a->with_active = with_active ? 1 : 0;
  if (a->n_tok <= 0) {
    *err = "no tokens to attend to";
    return DKV_ERR_INVALID_ARG;
  }
  // kernel 2: tcgen05 with query-row blocks; 3: tcgen05 with the tokens on
  // the TMEM lanes (32-row query groups only)
  int kernel = ci.opt_kernel;
  if (kernel == 0) kernel = tc_supported(v) ? 2 : 1;
  if ((kernel >= 2 && !tc_supported(v)) || (kernel == 3 && v.rows != 32)) {
    *err = "no tcgen05 attention variant for this shape";
    return DKV_ERR_UNSUPPORTED;
  }
  a->tc_layout = kernel == 3 ? 1 : 0;
  const int tile = kernel >= 2 ? kTcTile : kMmaTile;
  const int64_t n_tiles = ceil_div(a->n_tok, tile);
  const int64_t nrb = kernel >= 2 ? (v.rows + 127) / 128 : 1;
  const int64_t cap = std::max<int64_t>(1, std::min<int64_t>(n_tiles, ci.max_splits));
  int64_t ns;
  if (ci.opt_splits > 0) {
    ns = std::min<int64_t>(ci.opt_splits, cap);
  } else {
    // minimise waves x (tiles per split + 2 tiles of per-CTA overhead) plus
    // the combine's traffic (U*rows*(4d+8) bytes per split, ~5.2 MB per tile
    // time), one CTA per SM
    const double comb = double(v.U) * v.rows * (4.0 * v.d + 8.0) / 5.2e6;
    double best = 1e300;
    ns = 1;
    for (int64_t s = 1; s <= cap; ++s) {
      const int64_t tps = ceil_div(n_tiles, s);
      const int64_t se = ceil_div(n_tiles, tps);
      if (se != s) continue;
      const int64_t waves = ceil_div(v.U * nrb * se, ci.num_sms);
      const double cost = double(waves) * double(tps + 2) + (se > 1 ? comb * se : 0.0);
      if (cost < best - 1e-9) {
        best = cost;
        ns = se;
      }
    }
  }
  const int64_t tps = ceil_div(n_tiles, ns);
  a->nsplit = int(ceil_div(n_tiles, tps));  // no empty split
  a->tiles_per_split = int(tps);
  // a rotated-V cache always goes through the combine kernel (inverse rotation)
  a->final_out = (a->nsplit == 1 && v.vrot_b == 0) ? 1 : 0;
  a->part_base = 0;
  a->part_stride = a->nsplit;
  // bounded waits give up after about 1 s; the stall test hook shortens that
  a->test_stall_tile = ci.opt_test_stall;
  a->wait_limit_ns = ci.opt_test_stall >= 0 ? 2000000ull : 1000000000ull;
  *kernel_out = kernel;
  return DKV_OK;
}

}  // namespace dkv

extern "C" {

const char* dkv_last_error(void) { return g_err.c_str(); }

int dkv_cache_alloc(const dkv_config* cfg, void* stream, dkv_cache** out) {
  dkv::NvtxRange nvtx_range("dkv_cache_alloc");
  g_err.clear();
  if (!out) return fail(DKV_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  int rc = check_config(cfg);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  dkv_cache* c = new (std::nothrow) dkv_cache();
  if (!c) return fail(DKV_ERR_INVALID_ARG, "host allocation failed");
  c->cfg = *cfg;
  c->lens.assign(size_t(cfg->batch), 0);
  c->trunc.assign(size_t(cfg->batch), 0);
  dkv::CacheView& v = c->v;
  v.B = cfg->batch;
  v.Hq = cfg->q_heads;
  v.Hkv = cfg->kv_heads;
  v.d = cfg->head_dim;
  v.blk = cfg->block;
  v.g = v.Hq / v.Hkv;
  v.rows = v.g * v.blk;
  v.kb = cfg->k_bits;
  v.vb = cfg->v_bits;
  v.GK = cfg->k_bits < 16 ? cfg->k_group : cfg->block;
  v.GV = cfg->v_bits < 16 ? cfg->v_group : 32;
  v.P = cfg->k_bits < 16 ? cfg->max_protected : 0;
  v.cap = cfg->max_tokens;
  v.nG = v.cap / v.GK;
  v.kw = v.kb < 16 ? v.GK * v.kb / 32 : 0;
  v.vw = v.vb < 16 ? v.d * v.vb / 32 : 0;
  v.vgroups = v.d / v.GV;
  v.twords = (v.GK + 31) / 32;
  v.U = v.B * v.Hkv;
  v.sink = cfg->sink_tokens;
  const size_t U = size_t(v.U);

  cudaError_t e = cudaGetDevice(&c->device);
  if (e == cudaSuccess)
    e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
  if (e != cudaSuccess) {
    delete c;
    return fail(DKV_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  }
  c->max_splits = split_cap(v.U, c->num_sms);

  // one arena; 256-byte aligned regions
  struct Region { size_t off, bytes; };
  size_t off = 0;
  auto take = [&](size_t bytes) {
    Region r{off, bytes};
    off = align256(off + bytes);
    return r;
  };
  const bool kq = v.kb < 16, vq = v.vb < 16;
  Region r_kc = take(kq ? U * v.nG * v.d * v.kw * 4 : 0);
  Region r_ksz = take(kq ? U * v.nG * v.d * 4 : 0);
  Region r_kraw = take(kq ? 0 : U * v.cap * v.d * 2);
  Region r_tail = take(kq ? U * v.GK * v.d * 2 : 0);
  Region r_tm = take(U * v.twords * 4);
  Region r_vc = take(vq ? U * v.cap * v.vw * 4 : 0);
  Region r_vsz = take(vq ? U * v.cap * v.vgroups * 4 : 0);
  Region r_vraw = take(vq ? 0 : U * v.cap * v.d * 2);
  Region r_pc = take(U * 4);
  Region r_pp = take(U * size_t(v.P) * 4);
  Region r_pk = take(U * size_t(v.P) * v.d * 2);
  Region r_pg = take(U * (v.nG + 1) * 4);
  Region r_st = take(4);
  Region r_po = take(dkv::split_o_bytes(v.U, c->max_splits, v.rows));
  Region r_pml = take(dkv::split_ml_bytes(v.U, c->max_splits, v.rows));
  Region r_vsink = take(vq ? U * size_t(v.sink) * v.d * 2 : 0);
  c->arena_bytes = off;

  e = cudaMalloc(&c->arena, c->arena_bytes);
  if (e != cudaSuccess) {
    delete c;
    return fail(DKV_ERR_CUDA, std::string("cudaMalloc: ") + cudaGetErrorString(e));
  }
  char* base = static_cast<char*>(c->arena);
  auto at = [&](const Region& r) -> void* { return r.bytes ? base + r.off : nullptr; };
  v.k_codes = static_cast<uint32_t*>(at(r_kc));
  v.k_sz = static_cast<__half2*>(at(r_ksz));
  v.k_raw = static_cast<uint16_t*>(at(r_kraw));
  v.k_tail = static_cast<uint16_t*>(at(r_tail));
  v.tail_mask = static_cast<uint32_t*>(at(r_tm));
  v.v_codes = static_cast<uint32_t*>(at(r_vc));
  v.v_sz = static_cast<__half2*>(at(r_vsz));
  v.v_raw = static_cast<uint16_t*>(at(r_vraw));
  v.prot_count = static_cast<int32_t*>(at(r_pc));
  v.prot_pos = static_cast<int32_t*>(at(r_pp));
  v.prot_k = static_cast<uint16_t*>(at(r_pk));
  v.prot_gstart = static_cast<int32_t*>(at(r_pg));
  v.status = static_cast<uint32_t*>(at(r_st));
  c->part_o = static_cast<__half*>(at(r_po));
  c->part_ml = static_cast<float2*>(at(r_pml));
  v.v_sink = static_cast<uint16_t*>(at(r_vsink));

  // zero everything that carries state (counters, masks, status) -- and the
  // rest, so exports of unused slots are deterministic; prot_pos unused = -1
  e = cudaMemsetAsync(c->arena, 0, r_po.off, s);
  if (e == cudaSuccess && r_pp.bytes) e = cudaMemsetAsync(base + r_pp.off, 0xFF, r_pp.bytes, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cudaFree(c->arena);
    delete c;
    return fail(DKV_ERR_CUDA, std::string("cache init: ") + cudaGetErrorString(e));
  }
  *out = c;
  return DKV_OK;
}

int dkv_cache_free(dkv_cache* c) {
  dkv::NvtxRange nvtx_range("dkv_cache_free");
  g_err.clear();
  if (!c) return fail(DKV_ERR_INVALID_ARG, "cache is NULL");
  cudaError_t e = cudaDeviceSynchronize();
  cudaError_t e2 = cudaFree(c->arena);
  for (void* m : {c->vrot_mem, c->sel_mem}) {
    if (!m) continue;
    const cudaError_t e3 = cudaFree(m);
    if (e2 == cudaSuccess) e2 = e3;
  }
  for (auto& r : c->prof) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  delete c;
  if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("sync: ") + cudaGetErrorString(e));
  if (e2 != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("cudaFree: ") + cudaGetErrorString(e2));
  return DKV_OK;
}

int dkv_cache_len(const dkv_cache* c, int64_t* len) {
  g_err.clear();
  if (!c || !len) return fail(DKV_ERR_INVALID_ARG, "NULL argument");
  *len = max_len(c);
  return DKV_OK;
}

int dkv_cache_seq_lens(const dkv_cache* c, int64_t* lens) {
  g_err.clear();
  if (!c || !lens) return fail(DKV_ERR_INVALID_ARG, "NULL argument");
  for (size_t b = 0; b < c->lens.size(); ++b) lens[b] = c->lens[b];
  return DKV_OK;
}

static int check_truncate(const dkv_cache* c, int64_t cur, int64_t new_len) {
  if (new_len < 0 || new_len > cur || new_len % c->v.blk)
    return fail(DKV_ERR_INVALID_ARG, "new_len must be a multiple of block within [0, len]");
  if (c->v.kb < 16 && new_len % c->v.GK)
    return fail(DKV_ERR_INVALID_ARG, "new_len must be a multiple of k_group");
  return DKV_OK;
}

// The device side (side-table count, tail mask) is read only by the next
// commit and by export, so a roll-back is recorded here and applied by
// whichever of them comes first: no launch of its own.
int dkv_cache_truncate(dkv_cache* c, int64_t new_len, void* stream) {
  dkv::NvtxRange nvtx_range("dkv_cache_truncate");
  g_err.clear();
  if (!c) return fail(DKV_ERR_INVALID_ARG, "cache is NULL");
  for (int64_t l : c->lens) {
    const int rc = check_truncate(c, l, new_len);
    if (rc != DKV_OK) return rc;
  }
  (void)stream;
  for (size_t b = 0; b < c->lens.size(); ++b) {
    if (c->v.kb < 16) c->trunc[b] = 1;
    c->lens[b] = new_len;
  }
  return DKV_OK;
}

int dkv_cache_truncate_seq(dkv_cache* c, int32_t seq, int64_t new_len, void* stream) {
  dkv::NvtxRange nvtx_range("dkv_cache_truncate_seq");
  g_err.clear();
  if (!c) return fail(DKV_ERR_INVALID_ARG, "cache is NULL");
  if (seq < 0 || seq >= c->v.B) return fail(DKV_ERR_INVALID_ARG, "seq out of range");
  const int rc = check_truncate(c, c->lens[size_t(seq)], new_len);
  if (rc != DKV_OK) return rc;
  (void)stream;
  if (c->v.kb < 16) c->trunc[size_t(seq)] = 1;
  c->lens[size_t(seq)] = new_len;
  return DKV_OK;
}

// Applies recorded roll-backs to the device state (export without an
// intervening commit).
static int apply_pending_truncate(dkv_cache* c, cudaStream_t s) {
  if (!any_trunc(c)) return DKV_OK;
  const dkv::CommitArgs ca = commit_args(c, std::vector<char>(c->lens.size(), 0));
  cudaError_t e = timed_launch(c, DKV_KERNEL_TRUNCATE, s,
                               [&] { return dkv::launch_truncate(c->v, ca, s); });
  if (e != cudaSuccess)
    return fail(DKV_ERR_CUDA, std::string("truncate launch: ") + cudaGetErrorString(e));
  std::fill(c->trunc.begin(), c->trunc.end(), 0);
  return DKV_OK;
}

static int commit_some(dkv_cache* c, const void* k, const void* v, const uint32_t* protect_words,
                       const std::vector<char>& commits, void* stream) {
  if (!k || !v) return fail(DKV_ERR_INVALID_ARG, "NULL cache, k or v");
  if (!aligned16(k) || !aligned16(v) ||
      (reinterpret_cast<uintptr_t>(protect_words) & 3u))
    return fail(DKV_ERR_INVALID_ARG, "k and v must be 16-byte aligned, protect_words 4-byte");
  for (size_t b = 0; b < c->lens.size(); ++b)
    if (commits[b] && c->lens[b] + c->v.blk > c->v.cap)
      return fail(DKV_ERR_CAPACITY, "len + block exceeds max_tokens");
  {
    dkv::CacheInfo ci;
    dkv::cache_info(c, &ci);
    const int drc = dkv::check_device(ci);
    if (drc != DKV_OK) return drc;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dkv::CommitArgs ca = commit_args(c, commits);
  cudaError_t e = timed_launch(c, DKV_KERNEL_COMMIT, s, [&] {
    return dkv::launch_commit(c->v, static_cast<const uint16_t*>(k),
                              static_cast<const uint16_t*>(v), protect_words, ca, s);
  });
  if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("commit launch: ") + cudaGetErrorString(e));
  for (size_t b = 0; b < c->lens.size(); ++b)
    if (commits[b]) {
      c->trunc[b] = 0;
      c->lens[b] += c->v.blk;
    }
  return DKV_OK;
}

int dkv_commit_block(dkv_cache* c, const void* k, const void* v, const uint32_t* protect_words,
                     void* stream) {
  dkv::NvtxRange nvtx_range("dkv_commit_block");
  g_err.clear();
  if (!c) return fail(DKV_ERR_INVALID_ARG, "NULL cache, k or v");
  return commit_some(c, k, v, protect_words, std::vector<char>(c->lens.size(), 1), stream);
}

int dkv_commit_block_seqs(dkv_cache* c, const void* k, const void* v,
                          const uint32_t* protect_words, const int32_t* seqs, int32_t n_seqs,
                          void* stream) {
  dkv::NvtxRange nvtx_range("dkv_commit_block_seqs");
  g_err.clear();
  if (!c) return fail(DKV_ERR_INVALID_ARG, "NULL cache, k or v");
  if (n_seqs < 0 || (n_seqs > 0 && !seqs)) return fail(DKV_ERR_INVALID_ARG, "bad sequence list");
  std::vector<char> commits(c->lens.size(), 0);
  for (int32_t i = 0; i < n_seqs; ++i) {
    if (seqs[i] < 0 || seqs[i] >= c->v.B) return fail(DKV_ERR_INVALID_ARG, "sequence index out of range");
    if (commits[size_t(seqs[i])]) return fail(DKV_ERR_INVALID_ARG, "sequence listed twice");
    commits[size_t(seqs[i])] = 1;
  }
  if (n_seqs == 0) return DKV_OK;
  return commit_some(c, k, v, protect_words, commits, stream);
}

int dkv_block_attention(dkv_cache* c, const void* q, const void* k_act, const void* v_act,
                        float softmax_scale, void* out, void* stream) {
  dkv::NvtxRange nvtx_range("dkv_block_attention");
  g_err.clear();
  if (!c || !q || !k_act || !v_act || !out) return fail(DKV_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(q) || !aligned16(k_act) || !aligned16(v_act) || !aligned16(out))
    return fail(DKV_ERR_INVALID_ARG, "q, k_act, v_act and out must be 16-byte aligned");
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return fail(DKV_ERR_INVALID_ARG, "softmax_scale must be finite");
  const dkv::CacheView& v = c->v;
  dkv::AttnArgs a{};
  a.c = v;
  a.q = static_cast<const uint16_t*>(q);
  a.k_act = static_cast<const uint16_t*>(k_act);
  a.v_act = static_cast<const uint16_t*>(v_act);
  a.out = static_cast<uint16_t*>(out);
  a.part_o = c->part_o;
  a.part_ml = c->part_ml;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  dkv::CacheInfo ci;
  dkv::cache_info(c, &ci);
  const int drc = dkv::check_device(ci);
  if (drc != DKV_OK) return drc;
  int kernel = 0;
  const char* perr = nullptr;
  const int prc = dkv::plan_attention(ci, &a, &kernel, &perr);
  if (prc != DKV_OK) return fail(prc, perr);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int launches = 1;
  if (v.vrot_b) {
    // the active block's V into the rotated basis of the cache's V rows
    cudaError_t e = dkv::launch_rotate_v_rows(v, a.v_act, c->vrot_act, s);
    if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("rotation launch: ") + cudaGetErrorString(e));
    a.v_act = c->vrot_act;
    ++launches;
  }
  cudaError_t e = timed_launch(c, DKV_KERNEL_ATTENTION, s, [&] {
    return kernel >= 2 ? dkv::launch_attention_tc(a, s) : dkv::launch_attention_mma(a, s);
  });
  if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("attention launch: ") + cudaGetErrorString(e));
  if (!a.final_out) {
    e = timed_launch(c, DKV_KERNEL_COMBINE, s, [&] { return dkv::launch_combine(a, s); });
    if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("combine launch: ") + cudaGetErrorString(e));
    ++launches;
  }
  c->last_kernel = kernel;
  c->last_splits = a.nsplit;
  c->last_launches = launches;
  return DKV_OK;
}

int dkv_block_attention_dual(dkv_cache* c, dkv_cache* sfx, const void* q, const void* k_act,
                             const void* v_act, float softmax_scale, void* out, void* stream) {
  dkv::NvtxRange nvtx_range("dkv_block_attention_dual");
  g_err.clear();
  if (!c || !sfx || !q || !k_act || !v_act || !out) return fail(DKV_ERR_INVALID_ARG, "NULL argument");
  const dkv::CacheView& v = c->v;
  const dkv::CacheView& vs = sfx->v;
  if (vs.B != v.B || vs.Hq != v.Hq || vs.Hkv != v.Hkv || vs.d != v.d || vs.blk != v.blk)
    return fail(DKV_ERR_INVALID_ARG, "prefix and suffix caches must share batch, heads, head_dim and block");
  if (sfx->device != c->device)
    return fail(DKV_ERR_INVALID_ARG, "prefix and suffix caches must be on the same device");
  if (v.vrot_b || vs.vrot_b)
    return fail(DKV_ERR_UNSUPPORTED, "dual-cache attention with rotated V is not supported");
  if (vs.sink > 0) return fail(DKV_ERR_UNSUPPORTED, "the suffix cache cannot have an attention sink");
  if (max_len(sfx) == 0) {
    // nothing after the active block: the single-cache call
    const int rc = dkv_block_attention(c, q, k_act, v_act, softmax_scale, out, stream);
    return rc;
  }
  if (!aligned16(q) || !aligned16(k_act) || !aligned16(v_act) || !aligned16(out))
    return fail(DKV_ERR_INVALID_ARG, "q, k_act, v_act and out must be 16-byte aligned");
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return fail(DKV_ERR_INVALID_ARG, "softmax_scale must be finite");

  // prefix + active block: splits [0, n1); suffix: splits [n1, n1 + n2) of the
  // prefix cache's partial workspace (room for max_splits per unit)
  dkv::AttnArgs a1{}, a2{};
  for (dkv::AttnArgs* a : {&a1, &a2}) {
    a->q = static_cast<const uint16_t*>(q);
    a->k_act = static_cast<const uint16_t*>(k_act);
    a->v_act = static_cast<const uint16_t*>(v_act);
    a->out = static_cast<uint16_t*>(out);
    a->part_o = c->part_o;
    a->part_ml = c->part_ml;
    a->scale_log2 = softmax_scale * 1.4426950408889634f;
  }
  a1.c = v;
  a2.c = vs;
  dkv::CacheInfo ci1, ci2;
  dkv::cache_info(c, &ci1);
  dkv::cache_info(sfx, &ci2);
  const int drc = dkv::check_device(ci1);
  if (drc != DKV_OK) return drc;
  ci1.max_splits = c->max_splits - 1;
  int k1 = 0, k2 = 0;
  const char* perr = nullptr;
  int prc = dkv::plan_attention(ci1, &a1, &k1, &perr, true);
  if (prc != DKV_OK) return fail(prc, perr);
  ci2.max_splits = c->max_splits - a1.nsplit;
  prc = dkv::plan_attention(ci2, &a2, &k2, &perr, false);
  if (prc != DKV_OK) return fail(prc, perr);
  const int total = a1.nsplit + a2.nsplit;
  a1.final_out = a2.final_out = 0;
  a1.part_base = 0;
  a2.part_base = a1.nsplit;
  a1.part_stride = a2.part_stride = total;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = timed_launch(c, DKV_KERNEL_ATTENTION, s, [&] {
    return k1 >= 2 ? dkv::launch_attention_tc(a1, s) : dkv::launch_attention_mma(a1, s);
  });
  if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("attention launch: ") + cudaGetErrorString(e));
  e = timed_launch(c, DKV_KERNEL_ATTENTION, s, [&] {
    return k2 >= 2 ? dkv::launch_attention_tc(a2, s) : dkv::launch_attention_mma(a2, s);
  });
  if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("suffix attention launch: ") + cudaGetErrorString(e));
  dkv::AttnArgs ac = a1;
  ac.nsplit = total;
  e = timed_launch(c, DKV_KERNEL_COMBINE, s, [&] { return dkv::launch_combine(ac, s); });
  if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("combine launch: ") + cudaGetErrorString(e));
  c->last_kernel = k1;
  c->last_splits = total;
  c->last_launches = 3;
  return DKV_OK;
}

int dkv_block_attention_selected(dkv_cache* c, const void* q, const void* k_act,
                                 const void* v_act, float softmax_scale, int32_t budget, void* out,
                                 int32_t* selected, float* scores, void* stream) {
  dkv::NvtxRange nvtx_range("dkv_block_attention_selected");
  g_err.clear();
  if (!c || !q || !k_act || !v_act || !out) return fail(DKV_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(q) || !aligned16(k_act) || !aligned16(v_act) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(selected) & 3u) || (reinterpret_cast<uintptr_t>(scores) & 3u))
    return fail(DKV_ERR_INVALID_ARG, "q, k_act, v_act and out must be 16-byte aligned, "
                                     "selected and scores 4-byte aligned");
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return fail(DKV_ERR_INVALID_ARG, "softmax_scale must be finite");
  const dkv::CacheView& v = c->v;
  if (budget < 0 || budget > v.cap) return fail(DKV_ERR_INVALID_ARG, "budget must be in [0, max_tokens]");
  if (v.vrot_b) return fail(DKV_ERR_UNSUPPORTED, "selection over a rotated-V cache is not supported");
  if (v.rows % 16) return fail(DKV_ERR_UNSUPPORTED, "(q_heads/kv_heads)*block must be a multiple of 16");
  dkv::CacheInfo ci;
  dkv::cache_info(c, &ci);
  const int drc = dkv::check_device(ci);
  if (drc != DKV_OK) return drc;
  // workspace, [U][cap] each: row-block shares of the scores, scores, selection
  const int nrb = dkv::score_row_blocks(v);
  const size_t cells = size_t(v.U) * size_t(v.cap);
  const size_t part_b = align256(cells * nrb * 4), sc_b = align256(cells * 4);
  if (!c->sel_mem) DKV_CUDA(cudaMalloc(&c->sel_mem, part_b + sc_b + cells * 4));
  float* part = static_cast<float*>(c->sel_mem);
  float* sc = scores ? scores : reinterpret_cast<float*>(static_cast<char*>(c->sel_mem) + part_b);
  int32_t* sel = selected ? selected
                          : reinterpret_cast<int32_t*>(static_cast<char*>(c->sel_mem) + part_b + sc_b);
  const int32_t sel_ld = selected ? budget : int32_t(v.cap);

  dkv::AttnArgs a{};
  a.c = v;
  a.q = static_cast<const uint16_t*>(q);
  a.k_act = static_cast<const uint16_t*>(k_act);
  a.v_act = static_cast<const uint16_t*>(v_act);
  a.out = static_cast<uint16_t*>(out);
  a.part_o = c->part_o;
  a.part_ml = c->part_ml;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  int kernel = 0;
  const char* perr = nullptr;
  int prc = dkv::plan_attention(ci, &a, &kernel, &perr);
  if (prc != DKV_OK) return fail(prc, perr);
  a.final_out = 0;  // the first pass keeps every row's (max, sum) in the split partials
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = timed_launch(c, DKV_KERNEL_ATTENTION, s, [&] {
    return kernel >= 2 ? dkv::launch_attention_tc(a, s) : dkv::launch_attention_mma(a, s);
  });
  if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("attention launch: ") + cudaGetErrorString(e));
  // contributions of the committed tokens, then the selection
  dkv::AttnArgs sa = a;
  sa.with_active = 0;
  sa.sel = sel;
  sa.sel_ld = sel_ld;
  sa.budget = budget;
  e = timed_launch(c, DKV_KERNEL_ATTENTION, s, [&] { return dkv::launch_scores(sa, part, v.cap, s); });
  if (e == cudaSuccess)
    e = timed_launch(c, DKV_KERNEL_ATTENTION, s,
                     [&] { return dkv::launch_topk(sa, part, v.cap, sc, sel, s); });
  if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("selection launch: ") + cudaGetErrorString(e));
  // attention over the selected tokens and the active block (mma.sync gather)
  dkv::CacheInfo cg = ci;
  cg.len = std::min<int64_t>(budget, ci.len);
  cg.opt_kernel = 1;
  dkv::AttnArgs ga = a;
  prc = dkv::plan_attention(cg, &ga, &kernel, &perr);
  if (prc != DKV_OK) return fail(prc, perr);
  ga.lens = ci.lens;  // unit_len takes min(budget, each sequence's length)
  ga.gather = 1;
  ga.sel = sel;
  ga.sel_ld = sel_ld;
  ga.budget = budget;
  e = timed_launch(c, DKV_KERNEL_ATTENTION, s, [&] { return dkv::launch_attention_mma(ga, s); });
  if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("selected attention launch: ") + cudaGetErrorString(e));
  int launches = 4;
  if (!ga.final_out) {
    e = timed_launch(c, DKV_KERNEL_COMBINE, s, [&] { return dkv::launch_combine(ga, s); });
    if (e != cudaSuccess) return fail(DKV_ERR_CUDA, std::string("combine launch: ") + cudaGetErrorString(e));
    ++launches;
  }
  c->last_kernel = 1;
  c->last_splits = ga.nsplit;
  c->last_launches = launches;
  return DKV_OK;
}

int dkv_cache_status(dkv_cache* c, void* stream, uint32_t* flags) {
  dkv::NvtxRange nvtx_range("dkv_cache_status");
  g_err.clear();
  if (!c || !flags) return fail(DKV_ERR_INVALID_ARG, "NULL argument");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DKV_CUDA(cudaStreamSynchronize(s));
  DKV_CUDA(cudaMemcpy(flags, c->v.status, 4, cudaMemcpyDeviceToHost));
  DKV_CUDA(cudaMemset(c->v.status, 0, 4));
  return DKV_OK;
}

// Host copies of units [u0, u0 + nU), all of committed length L.
static int export_units(dkv_cache* c, size_t u0, size_t nU, int64_t L, void* stream,
                        dkv_export* o) {
  const dkv::CacheView& v = c->v;
  const int trc = apply_pending_truncate(c, static_cast<cudaStream_t>(stream));
  if (trc != DKV_OK) return trc;
  DKV_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  const int64_t Lq = v.kb < 16 ? (L / v.GK) * v.GK : L;
  const int64_t nGq = v.kb < 16 ? Lq / v.GK : 0;
  // row = one unit: `width` bytes of a unit's `pitch`-byte region
  auto copy2d = [&](void* dst, const void* src, size_t width, size_t pitch) -> cudaError_t {
    if (!dst || !src || width == 0) return cudaSuccess;
    return cudaMemcpy2D(dst, width, static_cast<const char*>(src) + u0 * pitch, pitch, width, nU,
                        cudaMemcpyDeviceToHost);
  };
  if (v.kb < 16) {
    DKV_CUDA(copy2d(o->k_codes, v.k_codes, nGq * v.d * v.kw * 4, v.nG * v.d * v.kw * 4));
    DKV_CUDA(copy2d(o->k_sz, v.k_sz, nGq * v.d * 4, v.nG * v.d * 4));
    DKV_CUDA(copy2d(o->k_tail, v.k_tail, (L - Lq) * v.d * 2, size_t(v.GK) * v.d * 2));
    DKV_CUDA(copy2d(o->tail_mask, v.tail_mask, v.twords * 4, v.twords * 4));
    // Only the words of the occupied tail slots are meaningful (the commit
    // kernel writes a slot's word when tokens enter the tail and leaves it
    // when their group completes): the canonical view has the rest zero.
    if (o->tail_mask)
      for (size_t uu = 0; uu < nU; ++uu)
        for (int w = int((L - Lq) / 32); w < v.twords; ++w) o->tail_mask[uu * v.twords + w] = 0u;
    DKV_CUDA(copy2d(o->prot_count, v.prot_count, 4, 4));
    DKV_CUDA(copy2d(o->prot_pos, v.prot_pos, size_t(v.P) * 4, size_t(v.P) * 4));
    DKV_CUDA(copy2d(o->prot_k, v.prot_k, size_t(v.P) * v.d * 2, size_t(v.P) * v.d * 2));
    DKV_CUDA(copy2d(o->prot_gstart, v.prot_gstart, (nGq + 1) * 4, (v.nG + 1) * 4));
  } else {
    DKV_CUDA(copy2d(o->k_raw, v.k_raw, L * v.d * 2, v.cap * v.d * 2));
    if (o->prot_count) std::memset(o->prot_count, 0, nU * 4);
  }
  if (v.vb < 16) {
    DKV_CUDA(copy2d(o->v_codes, v.v_codes, L * v.vw * 4, v.cap * v.vw * 4));
    DKV_CUDA(copy2d(o->v_sz, v.v_sz, L * v.vgroups * 4, v.cap * v.vgroups * 4));
    const int64_t ns = std::min<int64_t>(v.sink, L);
    if (ns > 0) DKV_CUDA(copy2d(o->v_sink, v.v_sink, ns * v.d * 2, size_t(v.sink) * v.d * 2));
  } else {
    DKV_CUDA(copy2d(o->v_raw, v.v_raw, L * v.d * 2, v.cap * v.d * 2));
  }
  return DKV_OK;
}

int dkv_cache_export(dkv_cache* c, void* stream, dkv_export* o) {
  dkv::NvtxRange nvtx_range("dkv_cache_export");
  g_err.clear();
  if (!c || !o) return fail(DKV_ERR_INVALID_ARG, "NULL argument");
  for (int64_t l : c->lens)
    if (l != c->lens[0])
      return fail(DKV_ERR_INVALID_ARG,
                  "sequences have different lengths: export them with dkv_cache_export_seq");
  return export_units(c, 0, size_t(c->v.U), c->lens[0], stream, o);
}

int dkv_cache_export_seq(dkv_cache* c, int32_t seq, void* stream, dkv_export* o) {
  dkv::NvtxRange nvtx_range("dkv_cache_export_seq");
  g_err.clear();
  if (!c || !o) return fail(DKV_ERR_INVALID_ARG, "NULL argument");
  if (seq < 0 || seq >= c->v.B) return fail(DKV_ERR_INVALID_ARG, "seq out of range");
  return export_units(c, size_t(seq) * size_t(c->v.Hkv), size_t(c->v.Hkv), c->lens[size_t(seq)],
                      stream, o);
}

int dkv_cache_set_v_rotation(dkv_cache* c, const int32_t* perm, const float* mix,
                             int32_t block) {
  dkv::NvtxRange nvtx_range("dkv_cache_set_v_rotation");
  g_err.clear();
  if (!c) return fail(DKV_ERR_INVALID_ARG, "cache is NULL");
  if (max_len(c) != 0) return fail(DKV_ERR_INVALID_ARG, "set the V rotation before the first commit");
  if (block == 0) {
    if (c->vrot_mem) {
      DKV_CUDA(cudaDeviceSynchronize());
      DKV_CUDA(cudaFree(c->vrot_mem));
    }
    c->vrot_mem = nullptr;
    c->vrot_act = nullptr;
    c->v.vrot_b = 0;
    c->v.vrot_perm = nullptr;
    c->v.vrot_mix = nullptr;
    return DKV_OK;
  }
  if (block != 16 && block != 32 && block != 64 && block != 128)
    return fail(DKV_ERR_UNSUPPORTED, "rotation block must be 16, 32, 64 or 128");
  if (c->v.vb == 16) return fail(DKV_ERR_UNSUPPORTED, "V rotation needs quantized V (v_bits < 16)");
  if (c->v.sink > 0) return fail(DKV_ERR_UNSUPPORTED, "V rotation with an attention sink is not supported");
  if (!perm || !mix) return fail(DKV_ERR_INVALID_ARG, "perm and mix must not be NULL");
  const int d = dkv::kHeadDim, k = d / block;
  std::vector<char> seen(d, 0);
  for (int i = 0; i < d; ++i) {
    if (perm[i] < 0 || perm[i] >= d || seen[perm[i]])
      return fail(DKV_ERR_INVALID_ARG, "perm must be a permutation of 0..127");
    seen[perm[i]] = 1;
  }
  for (int i = 0; i < k * k; ++i)
    if (!std::isfinite(mix[i])) return fail(DKV_ERR_INVALID_ARG, "mix must be finite");
  for (int r = 0; r < k; ++r)
    for (int q = 0; q < k; ++q) {
      double dot = 0.0;
      for (int j = 0; j < k; ++j) dot += double(mix[r * k + j]) * double(mix[q * k + j]);
      if (std::fabs(dot - (r == q ? 1.0 : 0.0)) > 1e-4)
        return fail(DKV_ERR_INVALID_ARG, "mix must be orthogonal (|mix mix^T - I| <= 1e-4)");
    }
  // [perm d int32][mix k*k fp32] at 0, the rotated active block at 1024
  const size_t act_bytes = size_t(c->v.U) * size_t(c->v.blk) * size_t(d) * 2;
  void* mem = nullptr;
  DKV_CUDA(cudaMalloc(&mem, 1024 + act_bytes));
  std::vector<unsigned char> host(1024, 0);
  std::memcpy(host.data(), perm, size_t(d) * 4);
  std::memcpy(host.data() + size_t(d) * 4, mix, size_t(k) * k * 4);
  cudaError_t e = cudaMemcpy(mem, host.data(), host.size(), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(mem);
    return fail(DKV_ERR_CUDA, std::string("cudaMemcpy: ") + cudaGetErrorString(e));
  }
  if (c->vrot_mem) {
    DKV_CUDA(cudaDeviceSynchronize());
    DKV_CUDA(cudaFree(c->vrot_mem));
  }
  c->vrot_mem = mem;
  unsigned char* base = static_cast<unsigned char*>(mem);
  c->vrot_act = reinterpret_cast<uint16_t*>(base + 1024);
  c->v.vrot_b = block;
  c->v.vrot_norm = float(1.0 / std::sqrt(double(block)));
  c->v.vrot_perm = reinterpret_cast<const int32_t*>(base);
  c->v.vrot_mix = reinterpret_cast<const float*>(base + size_t(d) * 4);
  return DKV_OK;
}

int dkv_cache_set_option(dkv_cache* c, int32_t key, int64_t value) {
  g_err.clear();
  if (!c) return fail(DKV_ERR_INVALID_ARG, "cache is NULL");
  switch (key) {
    case DKV_OPT_SPLITS:
      if (value < 0 || value > c->max_splits)
        return fail(DKV_ERR_INVALID_ARG, "splits must be in [0, " + std::to_string(c->max_splits) + "]");
      c->opt_splits = int32_t(value);
      return DKV_OK;
    case DKV_OPT_ATTN_KERNEL:
      if (value < 0 || value > 3) return fail(DKV_ERR_INVALID_ARG, "kernel must be 0, 1, 2 or 3");
      if ((value >= 2 && !dkv::tc_supported(c->v)) || (value == 3 && c->v.rows != 32))
        return fail(DKV_ERR_UNSUPPORTED, "no tcgen05 attention variant for this shape");
      c->opt_kernel = int32_t(value);
      return DKV_OK;
    case DKV_OPT_TEST_STALL:
#ifdef DKV_BOUNDS_CHECK
      if (value < -1 || value > (int64_t(1) << 30))
        return fail(DKV_ERR_INVALID_ARG, "test stall tile must be -1 (off) or a tile index");
      c->opt_test_stall = int32_t(value);
      return DKV_OK;
#else
      return fail(DKV_ERR_UNSUPPORTED, "DKV_OPT_TEST_STALL exists only in the bounds-checking build");
#endif
    case DKV_OPT_PROFILE:
      if (value != 0 && value != 1) return fail(DKV_ERR_INVALID_ARG, "profile must be 0 or 1");
      c->profile = value == 1;
      return DKV_OK;
    default:
      return fail(DKV_ERR_INVALID_ARG, "unknown option key");
  }
}

int dkv_profile_read(dkv_cache* c, int32_t kind, double* total_ms, int64_t* launches) {
  g_err.clear();
  if (!c || !total_ms || !launches) return fail(DKV_ERR_INVALID_ARG, "NULL argument");
  double ms = 0.0;
  int64_t n = 0;
  for (size_t i = 0; i < c->prof_used; ++i) {
    ProfRecord& r = c->prof[i];
    DKV_CUDA(cudaEventSynchronize(r.stop));
    if (r.kind != kind) continue;
    float t = 0.f;
    DKV_CUDA(cudaEventElapsedTime(&t, r.start, r.stop));
    ms += t;
    ++n;
  }
  // records of other kinds stay readable: compact them to the front
  size_t keep = 0;
  for (size_t i = 0; i < c->prof_used; ++i)
    if (c->prof[i].kind != kind) std::swap(c->prof[keep++], c->prof[i]);
  c->prof_used = keep;
  *total_ms = ms;
  *launches = n;
  return DKV_OK;
}

int dkv_last_attention_plan(const dkv_cache* c, int32_t* kernel, int32_t* splits,
                            int32_t* launches) {
  g_err.clear();
  if (!c) return fail(DKV_ERR_INVALID_ARG, "cache is NULL");
  if (kernel) *kernel = c->last_kernel;
  if (splits) *splits = c->last_splits;
  if (launches) *launches = c->last_launches;
  return DKV_OK;
}

}  // extern "C"
