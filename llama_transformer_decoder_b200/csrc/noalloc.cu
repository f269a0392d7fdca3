// Decode attention for callers that cannot let the library allocate device
// memory. The split partials that llama_attention_decode keeps in
// library-allocated scratch live here in one file-scope static device array
// instead, so the call itself never allocates or frees device memory.
#include <mutex>

#include "kernels.h"
#include "llama_b200.h"

namespace {

constexpr size_t kScratchBytes = 4u << 20;   // 4 MiB, held by every GPU that loads the library
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_decode_scratch[kScratchBytes / sizeof(float)];

// Device address of g_decode_scratch per device. In host code the symbol is
// only a host-side stand-in, so the address is looked up once per device, with
// that device current, and passed to the kernels.
std::mutex g_mu;
float* g_addr[kMaxDevices] = {};

int scratch_address(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LLAMA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return LLAMA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return LLAMA_ERR_CUDA;
    }
    g_addr[dev] = static_cast<float*>(p);
  }
  *out = g_addr[dev];
  return LLAMA_OK;
}

}  // namespace

extern "C" int llama_attention_decode_noalloc(const void* q, const void* kc, const void* vc, const int32_t* len,
                                              void* o, int32_t B, int32_t cmax, int32_t H, int32_t Hk, int32_t d,
                                              int32_t dtype, void* stream) {
  if (!q || !kc || !vc || !len || !o) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || cmax <= 0 || H <= 0 || Hk <= 0 || H % Hk != 0) return LLAMA_ERR_SHAPE;
  if (dtype != LLAMA_F32 && dtype != LLAMA_BF16 && dtype != LLAMA_F16) return LLAMA_ERR_INVALID_ARG;
  const size_t need = llama::decode_scratch_floats(cmax, B, H, Hk, d, dtype);
  if (need * sizeof(float) > kScratchBytes) return LLAMA_ERR_SHAPE;
  float* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != LLAMA_OK) return rc;
  llama::DecodeScratch ds{scratch, kScratchBytes / sizeof(float)};
  return llama::attention_decode(q, kc, vc, len, 0, o, B, cmax, H, Hk, d, cmax, dtype, &ds, nullptr,
                                 static_cast<cudaStream_t>(stream));
}
