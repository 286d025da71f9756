// fq_attn_decode_noalloc: the fused decode-attention step for callers that cannot allocate
// device memory.
//
// fq_attn_decode needs a caller-owned workspace for its split-softmax partials.  Some callers
// cannot provide one: code embedded in a host application whose allocator owns all device
// memory and offers no hook for library scratch, or a decode loop that must not call
// cudaMalloc because allocation may synchronise the device and has unbounded latency.  For
// them this entry point keeps the partials in a fixed array that lives in the library's own
// device memory (a file-scope __device__ array, FQ_ATTN_NOALLOC_SCRATCH_BYTES bytes on every
// GPU that loads the library, held until the process exits).
//
// The array's name is only a host-side stand-in in host code; its device address is fetched
// once per device with cudaGetSymbolAddress (with that device current) the first time the
// entry point runs there, and that address is what the kernels receive.
#include <mutex>

#include "fq_internal.h"

namespace fq {
namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_attn_noalloc_scratch[FQ_ATTN_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
fq_status scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_noalloc_scratch) != cudaSuccess || p == nullptr)
      return FQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FQ_OK;
}

}  // namespace
}  // namespace fq

extern "C" fq_status fq_attn_decode_noalloc(
    const uint16_t* q, int B, int Hq, int Hkv, int64_t T, int d, const uint8_t* k_codes,
    const uint16_t* k_norms, int kK, int NK, const float* rotK, const float* cbK,
    const uint8_t* v_codes, const uint16_t* v_norms, int kV, int NV, const float* rotV,
    const float* cbV, float scale, float* out, void* stream) {
  // The same validation as fq_attn_decode comes first, so that a bad call is refused with its
  // own status before the scratch array is looked up.
  fq::AttnArgs a;
  size_t need = 0;
  fq_status st = fq::attn_prepare(q, B, Hq, Hkv, T, d, k_codes, k_norms, kK, NK, rotK, cbK,
                                  v_codes, v_norms, kV, NV, rotV, cbV, scale, out, &a, &need);
  if (st != FQ_OK) return st;
  // Sizes beyond the fixed scratch are refused before anything is enqueued.
  if (need > (size_t)FQ_ATTN_NOALLOC_SCRATCH_BYTES) return FQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    st = fq::scratch_on_current_device(&scratch);
    if (st != FQ_OK) return st;
  }
  // Same kernels and results as fq_attn_decode, with the fixed array as workspace (T = 0 needs
  // none: the output is zeroed).
  return fq_attn_decode(q, B, Hq, Hkv, T, d, k_codes, k_norms, kK, NK, rotK, cbK, v_codes,
                        v_norms, kV, NV, rotV, cbV, scale, out, scratch,
                        (size_t)FQ_ATTN_NOALLOC_SCRATCH_BYTES, stream);
}
