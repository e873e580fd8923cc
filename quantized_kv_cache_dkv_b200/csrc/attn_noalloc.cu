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

// Split partials, laid out as the handle's workspace (split_o_bytes of fp16
// partial outputs, then split_ml_bytes of (max, sum) pairs).  Host code must
// not use this name as an address: it is a host-side stand-in.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};  // device address per device ordinal

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int dkv_block_attention_noalloc(dkv_cache* cache, const void* q, const void* k_act,
                                           const void* v_act, float softmax_scale, void* out,
                                           void* stream) {
  dkv::NvtxRange nvtx_range("dkv_block_attention_noalloc");
  using dkv::report_error;
  dkv::CacheInfo ci;
  if (!dkv::cache_info(cache, &ci) || !q || !k_act || !v_act || !out)
    return report_error(DKV_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(q) || !aligned16(k_act) || !aligned16(v_act) || !aligned16(out))
    return report_error(DKV_ERR_INVALID_ARG, "q, k_act, v_act and out must be 16-byte aligned");
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return report_error(DKV_ERR_INVALID_ARG, "softmax_scale must be finite");

  // the call runs on the cache's device, which must be the current one (the
  // static buffer exists once per device)
  const int drc = dkv::check_device(ci);
  if (drc != DKV_OK) return drc;
  const int dev = ci.device;
  if (dev < 0 || dev >= kMaxDevices) return report_error(DKV_ERR_UNSUPPORTED, "device ordinal >= 64");
  cudaError_t e = cudaSuccess;
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

  // the launch plan of dkv_block_attention
  int kernel = 0;
  const char* perr = nullptr;
  const int prc = dkv::plan_attention(ci, &a, &kernel, &perr);
  if (prc != DKV_OK) return report_error(prc, perr);

  if (!a.final_out) {
    const size_t o_bytes = dkv::split_o_bytes(v.U, a.nsplit, v.rows);
    const size_t need = o_bytes + dkv::split_ml_bytes(v.U, a.nsplit, v.rows);
    if (need > kScratchBytes)
      return report_error(
          DKV_ERR_UNSUPPORTED,
          ("this plan needs " + std::to_string(need) + " bytes of split scratch; the static buffer "
           "holds " + std::to_string(kScratchBytes) + ": lower DKV_OPT_SPLITS or use "
           "dkv_block_attention").c_str());
    a.part_o = static_cast<__half*>(scratch);
    a.part_ml = reinterpret_cast<float2*>(static_cast<unsigned char*>(scratch) + o_bytes);
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (v.vrot_b) {
    // the active block's V into the cache's rotated basis (cache-owned buffer)
    e = dkv::launch_rotate_v_rows(v, a.v_act, ci.vrot_act, s);
    if (e != cudaSuccess)
      return report_error(DKV_ERR_CUDA, (std::string("rotation launch: ") + cudaGetErrorString(e)).c_str());
    a.v_act = ci.vrot_act;
  }
  e = kernel >= 2 ? dkv::launch_attention_tc(a, s) : dkv::launch_attention_mma(a, s);
  if (e != cudaSuccess)
    return report_error(DKV_ERR_CUDA, (std::string("attention launch: ") + cudaGetErrorString(e)).c_str());
  if (!a.final_out) {
    e = dkv::launch_combine(a, s);
    if (e != cudaSuccess)
      return report_error(DKV_ERR_CUDA, (std::string("combine launch: ") + cudaGetErrorString(e)).c_str());
  }
  report_error(DKV_OK, "");
  return DKV_OK;
}
