// dkv_block_attention_noalloc: block attention whose split scratch lives in a
// static device buffer of this file, so the call allocates nothing.  For
// callers that cannot call cudaMalloc (inside CUDA stream capture, or in a
// host application that owns all device memory).  The computation, launch
// plan and kernels are those of dkv_block_attention.
#include <algorithm>
#include <cstdint>
#include <mutex>
#include <string>

#include "dkv_internal.cuh"

namespace {

constexpr size_t kScratchBytes = DKV_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Split partials: [U][splits][rows][d] fp32, then [U][splits][rows] float2.
// Host code must not use this name as an address: it is a host-side stand-in.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};  // device address per device ordinal

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int dkv_block_attention_noalloc(dkv_cache* cache, const void* q, const void* k_act,
                                           const void* v_act, float softmax_scale, void* out,
                                           void* stream) {
  using dkv::report_error;
  dkv::CacheInfo ci;
  if (!dkv::cache_info(cache, &ci) || !q || !k_act || !v_act || !out)
    return report_error(DKV_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(q) || !aligned16(k_act) || !aligned16(v_act) || !aligned16(out))
    return report_error(DKV_ERR_INVALID_ARG, "q, k_act, v_act and out must be 16-byte aligned");
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return report_error(DKV_ERR_INVALID_ARG, "softmax_scale must be finite");

  // once per device, with that device current: the buffer's device address
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return report_error(DKV_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return report_error(DKV_ERR_UNSUPPORTED, "device ordinal >= 64");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess)
        return report_error(DKV_ERR_CUDA, (std::string("cudaGetSymbolAddress: ") +
                                           cudaGetErrorString(e)).c_str());
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }

  const dkv::CacheView& v = ci.v;
  dkv::AttnArgs a{};
  a.c = v;
  a.q = static_cast<const uint16_t*>(q);
  a.k_act = static_cast<const uint16_t*>(k_act);
  a.v_act = static_cast<const uint16_t*>(v_act);
  a.out = static_cast<uint16_t*>(out);
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.L = ci.len;
  a.Lq = v.kb < 16 ? (ci.len / v.GK) * v.GK : ci.len;
  a.n_tok = ci.len + v.blk;

  // the launch plan of dkv_block_attention
  int kernel = ci.opt_kernel;
  if (kernel == 0) kernel = dkv::tc_supported(v) ? 2 : 1;
  if (kernel == 2 && !dkv::tc_supported(v))
    return report_error(DKV_ERR_UNSUPPORTED, "no tcgen05 attention variant for this shape");
  const int tile = kernel == 2 ? dkv::kTcTile : dkv::kMmaTile;
  const int64_t n_tiles = ceil_div(a.n_tok, tile);
  int64_t ns;
  if (ci.opt_splits > 0) {
    ns = ci.opt_splits;
  } else {
    ns = ceil_div(int64_t(2) * ci.num_sms, v.U);
    ns = std::min<int64_t>(ns, std::max<int64_t>(1, n_tiles / 2));
  }
  ns = std::max<int64_t>(1, std::min<int64_t>({ns, n_tiles, int64_t(ci.max_splits)}));
  const int64_t tps = ceil_div(n_tiles, ns);
  ns = ceil_div(n_tiles, tps);
  a.nsplit = int(ns);
  a.tiles_per_split = int(tps);

  if (a.nsplit > 1) {
    const size_t rows_total = size_t(v.U) * size_t(a.nsplit) * size_t(v.rows);
    const size_t o_bytes = align256(rows_total * size_t(dkv::kHeadDim) * sizeof(float));
    const size_t need = o_bytes + rows_total * sizeof(float2);
    if (need > kScratchBytes)
      return report_error(
          DKV_ERR_UNSUPPORTED,
          ("this plan needs " + std::to_string(need) + " bytes of split scratch; the static buffer "
           "holds " + std::to_string(kScratchBytes) + ": lower DKV_OPT_SPLITS or use "
           "dkv_block_attention").c_str());
    a.part_o = static_cast<float*>(scratch);
    a.part_ml = reinterpret_cast<float2*>(static_cast<unsigned char*>(scratch) + o_bytes);
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  e = kernel == 2 ? dkv::launch_attention_tc(a, s) : dkv::launch_attention_mma(a, s);
  if (e != cudaSuccess)
    return report_error(DKV_ERR_CUDA, (std::string("attention launch: ") + cudaGetErrorString(e)).c_str());
  if (a.nsplit > 1) {
    e = dkv::launch_combine(a, s);
    if (e != cudaSuccess)
      return report_error(DKV_ERR_CUDA, (std::string("combine launch: ") + cudaGetErrorString(e)).c_str());
  }
  report_error(DKV_OK, "");
  return DKV_OK;
}
