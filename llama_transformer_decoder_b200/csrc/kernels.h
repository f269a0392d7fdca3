// Internal launch interface between the C-ABI host code (model.cu) and the
// kernels. Not part of the public header.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace llama {

struct EpiArgs;
struct KvLayout;
struct ChainJobDesc;

// Launch with programmatic stream serialization (the kernel must call
// pdl_wait() before reading its predecessor's output). Disabled when the
// environment variable LLAMA_NO_PDL is set.
bool pdl_enabled();
// Process-wide count of kernel launches made by the library.
void count_launches(unsigned long long n);
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  count_launches(1);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

enum GemmVariant { GEMM_AUTO = 0, GEMM_WIDE = 1, GEMM_SKINNY = 2 };

// Scratch of the split-tile fixups: one fp32 share slot per CTA and one
// counter per split tile (counters start at zero; the kernels leave them zero).
struct GemmScratch {
  float* ws;
  size_t ws_floats;
  int* tickets;
  int n_tickets;
};

// Identity of the calling thread's current CUDA context (unique over the
// process lifetime; a device reset gives a new one). Falls back to a key of
// the device ordinal when no context is current.
uint64_t context_key();
// SM count of the current device (cached per device).
int num_sms();
// Raises the dynamic shared-memory limit of `kern` to `bytes` on the current
// device, once per device (thread-safe). LLAMA_OK or LLAMA_ERR_CUDA.
int ensure_smem_attr(const void* kern, int bytes);

// How a wide (prefill) GEMM is spread over the SMs: tiles [0, T_dp) in
// data-parallel waves, the rest stream-K over G_sk CTAs (see gemm_tc.cu).
struct WideSplit {
  int tiles, sk_tiles, T_dp, G_sk, grid;
};
WideSplit wide_split(int M, int N, int K);
// Partial-tile workspace (floats) a wide GEMM needs for its stream-K tiles
// (plus sk_tiles tickets).
size_t wide_workspace_floats();
int make_tmap_16(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t pitch, int box_rows,
                 bool is_f16);
// Scratch of the stream-K skinny GEMM for M rows: two partial tiles per CTA.
size_t skinny_workspace_floats(int M);

// True when an automatic 16-bit GEMM of this shape runs the CTA-pair kernel.
bool gemm16_uses_pair(int M, int N, int K);
// Up to four CTA-pair GEMMs (each gemm16_uses_pair) in one persistent launch,
// later jobs waiting only for the row blocks of earlier jobs they read (see
// ChainJobDesc in epilogue.cuh). elt = LLAMA_BF16 or LLAMA_F16.
int gemm16_chain(const ChainJobDesc* jobs, int n, int elt, int* status, cudaStream_t st);
// 16-bit GEMM; elt = LLAMA_BF16 or LLAMA_F16 (element type of A, W and 16-bit outputs).
int gemm16(const void* A, int M, int K, int lda, const void* W, int N, int ldw, int elt, int kind, const EpiArgs& e,
           int variant, GemmScratch* scratch, int* status, cudaStream_t st);
int gemm_f32(const float* A, int M, int K, int lda, const float* W, int N, int ldw, int kind, const EpiArgs& e,
             int* status, cudaStream_t st);

// Elementwise / reductions. dtype: LLAMA_F32, LLAMA_BF16 or LLAMA_F16 (of `y` / tables).
int launch_embed(const int32_t* tokens, int M, const void* table, int V, int D, int dtype, float* x, int* status,
                 cudaStream_t st);
// y[r] = rmsnorm(x[row(r)]) * g; row(r) = r, or (r+1)*S-1 when last_of_S > 0.
// 16-bit outputs that are not finite latch LLAMA_ERR_RANGE in *status (if given).
int launch_rmsnorm(const float* x, const float* g, void* y, int rows, int D, float eps, int last_of_S, int dtype,
                   cudaStream_t st, int* status = nullptr);
int launch_argmax(const float* logits, int32_t* out, int B, int V, cudaStream_t st);
// y = x * g (16-bit) and ss[r*ss_n + 0] = sum of x[r]^2 (other slots 0): the
// inputs of a GEMM that applies the RMSNorm in its epilogue.
int launch_norm_prep(const float* x, const float* g, void* y, float* ss, int rows, int D, int ss_n, int dtype,
                     cudaStream_t st, int* status = nullptr);
int launch_add_lengths(int32_t* len, int B, int add, cudaStream_t st);

// Attention. q [B][H][S][d]; K/V cache [B][Hk][Smax][d] (this layer);
// o [B*S][H*d]; pos0[b] = position of the call's first query (null = 0).
// Caches: contiguous [B][Hk][Smax][d] (kv_table == nullptr), or paged: pages
// [kv_pages][Hk][128][d] with page j of sequence b at kv_table[b*kv_max_pages + j]
// (16-bit, d = 128 only; Smax is then the per-sequence capacity).
int attention_prefill(const void* q, const void* kc, const void* vc, void* o, const int32_t* pos0, int B, int S,
                      int H, int Hk, int d, int Smax, int dtype, int* status, cudaStream_t st,
                      const int32_t* kv_table = nullptr, int kv_max_pages = 0, int kv_pages = 0);
// tcgen05 flash attention for 16-bit q/k/v (elt = LLAMA_BF16 or LLAMA_F16), d = 128.
int attention_prefill_tc(const void* q, const void* kc, const void* vc, void* o, const int32_t* pos0, int B, int S,
                         int H, int Hk, int Smax, int elt, int* status, cudaStream_t st,
                         const int32_t* kv_table = nullptr, int kv_max_pages = 0, int kv_pages = 0);
// Decode: q [B][H][d]; keys 0 .. nkeys[b]-1 (+ add) of the cache; o [B][H*d].
struct DecodeScratch {
  float* part;  // [B][H][splits][d + 2]
  size_t floats;
};
size_t decode_scratch_floats(int cmax, int B, int H, int Hk, int d, int dtype);
int attention_decode(const void* q, const void* kc, const void* vc, const int32_t* nkeys, int add_keys, void* o,
                     int B, int cmax, int H, int Hk, int d, int Smax, int dtype, DecodeScratch* scratch,
                     int* status, cudaStream_t st, const int32_t* kv_table = nullptr, int kv_max_pages = 0,
                     int kv_pages = 0);

// Status word of llama_attention_decode_noalloc on the current device: read
// and cleared (0 when that call never ran on the device). Allocates nothing.
int noalloc_take_status(int* out);

// Seeded generator: SplitMix64 counter streams + Box-Muller from IEEE basic ops.
// Logical element i = ((o * rows + r) * cols + c) of a [outer][rows][cols]
// tensor lands at  o*outer_stride + (r*row_mult + row_off)*row_stride + c.
struct FillLayout {
  int64_t outer, rows, cols;
  int64_t outer_stride, row_stride;
  int row_mult, row_off;
};
// dtype: element type of dst; round_bf16 rounds each value to bf16 first (bf16
// values kept in an fp16 buffer).
int launch_fill_normal(void* dst, const FillLayout& L, uint64_t seed, uint64_t stream_id, float std, int dtype,
                       cudaStream_t st, bool round_bf16 = false);
int launch_convert_2d(void* dst, int64_t dpitch, int dst_elt, const void* src, int64_t spitch, int src_elt,
                      int64_t rows, int64_t cols, cudaStream_t st);
int launch_fill_const(float* dst, int64_t n, float v, cudaStream_t st);
// One kernel whose bounded wait can never complete (kind 0: mbarrier, 1:
// device counter); it gives up after limit_ns and latches a timeout.
int launch_wait_selftest(int kind, uint64_t limit_ns, int* status, cudaStream_t st);
// N(0, std^2) draws of stream `stream_id` in the logical order [B][Hk][c][d]
// (the cache generator's order), written through a cache layout.
int launch_fill_kv(void* dst, const KvLayout& L, int B, int Hk, int c, int d, uint64_t seed, uint64_t stream_id,
                   float std, int dtype, bool round_bf16, cudaStream_t st);
// Cache (through L) <- src [B][Hk][c][d], converting src_elt -> dst_elt.
int launch_kv_scatter(void* dst, int dst_elt, const KvLayout& L, int B, int Hk, int c, int d, const void* src,
                      int src_elt, cudaStream_t st);

}  // namespace llama
