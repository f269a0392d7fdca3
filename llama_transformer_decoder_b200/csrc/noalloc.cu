// Decode attention for callers that cannot let the library allocate device
// memory. The split partials that llama_attention_decode keeps in
// library-allocated scratch live here in one file-scope static device array
// instead, and the call's device-side errors go to a static status word next
// to it, so the call itself never allocates or frees device memory. The
// array starts zeroed, as the decode kernel's work counters in its last 16
// bytes must (the kernel re-arms them at the end of every launch).
#include <map>
#include <mutex>

#include "kernels.h"
#include "llama_b200.h"

namespace {

constexpr size_t kScratchBytes = 8u << 20;   // 8 MiB, held by every GPU that loads the library

static __device__ __align__(256) float g_decode_scratch[kScratchBytes / sizeof(float)];
static __device__ int g_noalloc_status;

// Device addresses of the two symbols, per device. In host code a __device__
// symbol's name is only a host-side stand-in, so each address is looked up
// (cudaGetSymbolAddress) with the device current and passed to the kernels.
// The lookup is redone when the device's context changed since (e.g. after
// cudaDeviceReset, which unloads the module and may move the array).
struct Addrs {
  uint64_t ctx_id = 0;
  float* scratch = nullptr;
  int* status = nullptr;
};
std::mutex g_mu;
std::map<int, Addrs> g_addrs;

// lookup == false: only return what an earlier call set up on this device
// (nothing when no call ran here, or the context changed since).
int addresses(Addrs* out, bool lookup) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LLAMA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  const uint64_t id = llama::context_key();
  auto it = g_addrs.find(dev);
  if (it != g_addrs.end() && !(id >> 63) && it->second.ctx_id == id) {
    *out = it->second;
    return LLAMA_OK;
  }
  if (!lookup) {
    *out = Addrs{};
    return LLAMA_OK;
  }
  Addrs a;
  void* p = nullptr;
  void* s = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr ||
      cudaGetSymbolAddress(&s, g_noalloc_status) != cudaSuccess || s == nullptr) {
    cudaGetLastError();
    return LLAMA_ERR_CUDA;
  }
  a.scratch = static_cast<float*>(p);
  a.status = static_cast<int*>(s);
  a.ctx_id = llama::context_key();   // the lookup made the device's context current if it was not
  g_addrs[dev] = a;
  *out = a;
  return LLAMA_OK;
}

}  // namespace

namespace llama {

// Reads and clears the status word of the no-allocation calls on the current
// device (synchronous copies; nothing is allocated). 0 when no such call ran.
int noalloc_take_status(int* out) {
  *out = 0;
  Addrs a;
  const int rc = addresses(&a, false);
  if (rc != LLAMA_OK) return rc;
  if (!a.status) return LLAMA_OK;
  int s = 0;
  if (cudaMemcpy(&s, a.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(a.status, 0, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return LLAMA_ERR_CUDA;
  }
  *out = s;
  return LLAMA_OK;
}

}  // namespace llama

extern "C" int llama_attention_decode_noalloc(const void* q, const void* kc, const void* vc, const int32_t* len,
                                              void* o, int32_t B, int32_t cmax, int32_t H, int32_t Hk, int32_t d,
                                              int32_t dtype, void* stream) {
  if (!q || !kc || !vc || !len || !o) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || cmax <= 0 || H <= 0 || Hk <= 0 || H % Hk != 0) return LLAMA_ERR_SHAPE;
  if (dtype != LLAMA_F32 && dtype != LLAMA_BF16 && dtype != LLAMA_F16) return LLAMA_ERR_INVALID_ARG;
  const size_t need = llama::decode_scratch_floats(cmax, B, H, Hk, d, dtype);
  if (need * sizeof(float) > kScratchBytes) return LLAMA_ERR_SHAPE;
  Addrs a;
  const int rc = addresses(&a, true);
  if (rc != LLAMA_OK) return rc;
  llama::DecodeScratch ds{a.scratch, kScratchBytes / sizeof(float)};
  return llama::attention_decode(q, kc, vc, len, 0, o, B, cmax, H, Hk, d, cmax, dtype, &ds, a.status,
                                 static_cast<cudaStream_t>(stream));
}
