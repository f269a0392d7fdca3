/*
 * llama_b200.h — C ABI of the Llama-3 decoder forward pass on B200 (sm_100a).
 *
 * What is computed follows the Llama-3 walkthrough "250行代码从头搭建Llama 3，
 * GitHub一天4.6k星！Karpathy大赞" (ai02.cc), cited below as [W] with its section:
 * token embedding (分词器与编码), RMSNorm (构建Transformer层), per-head Q/K/V
 * projections (查询向量, 键向量, 值向量), rotary position embedding on adjacent
 * pairs (位置编码), causal grouped-query attention (查询和键相乘, 掩码,
 * 多头注意力), the Wo projection plus residual (相加与归一化), the SwiGLU
 * feed-forward plus residual (前馈神经网络层), the layer stack, the final
 * norm, last-token logits and greedy argmax (预测下一个输出). The KV cache is
 * the one described by "Deepdive-llama3-from-scratch" (KV-Cache chapter) and
 * sized up front by max_seq_len x max_batch_size as the Hacker News thread
 * "Llama 3 implemented in pure NumPy" explains.
 *
 * Conventions for every call:
 *  - Return value: LLAMA_OK (0) or a negative LLAMA_ERR_* code. No call throws
 *    or aborts. Errors detected inside a kernel (bad token id, timeout of a
 *    bounded wait) are latched in a device status word and returned by the
 *    next llama_sync_status() (model calls) or llama_status() (stateless
 *    calls).
 *  - Pointers named "device" are CUDA device pointers; the caller owns them
 *    and the library never frees them. `stream` is a cudaStream_t passed as
 *    void* (NULL = legacy default stream); calls are asynchronous on it
 *    unless stated otherwise.
 *  - Matrices are row-major and contiguous. Weights use the checkpoint's
 *    [out, in] convention and y = x W^T ([W] 查询向量).
 *  - dtype: LLAMA_F32 computes everything in fp32 on the CUDA cores.
 *    LLAMA_F16 stores weights, activations and the cache in fp16 and
 *    accumulates in fp32 on the tensor cores (tcgen05), with an fp32 residual
 *    stream and fp32 logits. LLAMA_BF16 takes bf16 weights (and bf16 K/V in
 *    llama_set_kv) at the boundary and runs the LLAMA_F16 path on them: each
 *    bf16 value is stored as the fp16 nearest to it (exact for
 *    2^-14 <= |w| <= 65504; smaller magnitudes keep an absolute error below
 *    2^-25, larger ones overflow), and activations are rounded to fp16, whose
 *    three extra mantissa bits keep the logits of a 32-layer stack within
 *    2e-2 (relative L2) of the exact result, which bf16 rounding of the
 *    activations does not. llama_get_weight returns bf16 again.
 *  - A model and its buffers belong to the device that was current at
 *    llama_create; make that device current before every later call.
 *    Kernel attributes and scratch of the stateless calls are kept per device.
 *    cudaDeviceReset frees everything the library holds on that device:
 *    models created before it must not be used after it.
 */
#ifndef LLAMA_B200_H
#define LLAMA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LLAMA_OK 0
#define LLAMA_ERR_INVALID_ARG (-1)   /* null pointer, bad enum, misaligned buffer */
#define LLAMA_ERR_SHAPE (-2)         /* sizes violate the model or the call's limits */
#define LLAMA_ERR_OOM (-3)           /* device allocation failed */
#define LLAMA_ERR_CUDA (-4)          /* a CUDA runtime/driver call failed */
#define LLAMA_ERR_DEVICE_TIMEOUT (-5)/* a bounded device-side wait gave up */
#define LLAMA_ERR_DEVICE_BOUNDS (-6) /* an index checked on the device was out of range */
#define LLAMA_ERR_UNSUPPORTED (-7)   /* combination not implemented (e.g. 16-bit model with head_dim != 128) */
#define LLAMA_ERR_RANGE (-8)         /* a 16-bit activation was not finite after rounding (fp16 overflows above
                                        65504): latched by the kernel that rounded it; the outputs are garbage */

typedef enum { LLAMA_F32 = 0, LLAMA_BF16 = 1, LLAMA_F16 = 2 } llama_dtype;

/* Model statement: the fields of params.json ([W] 下载并读取模型权重) plus the
 * cache sizing of the Hacker News thread (max_batch, max_seq). */
typedef struct llama_config {
  int32_t dim;                /* 4096 for the 8B model */
  int32_t n_layers;           /* 32 */
  int32_t n_heads;            /* 32; head_dim = dim / n_heads */
  int32_t n_kv_heads;         /* 8; n_heads % n_kv_heads == 0 */
  int32_t vocab_size;         /* 128256 */
  int32_t ffn_hidden;         /* SwiGLU width; 0 = derive with llama_ffn_hidden */
  int32_t multiple_of;        /* 1024 */
  float ffn_dim_multiplier;   /* 1.3; <= 0 means none */
  float norm_eps;             /* 1e-5 */
  float rope_theta;           /* 500000 */
  int32_t max_batch;          /* sequences held in the KV cache */
  int32_t max_seq;            /* positions per sequence in the KV cache */
  int32_t max_tokens;         /* largest B*S of one prefill call; 0 = min(max_batch*max_seq, 16384) */
  int32_t dtype;              /* llama_dtype */
  int32_t kv_page_size;       /* 0: contiguous cache [n_layers][max_batch][n_kv_heads][max_seq][head_dim];
                                 128: paged cache [n_layers][kv_pages][n_kv_heads][128][head_dim] with a block
                                 table (16-bit models; pages are taken from a pool as sequences grow and
                                 returned by llama_reset / llama_set_lengths) */
  int32_t kv_pages;           /* paged: pages in the pool; 0 = max_batch * ceil(max_seq / 128) */
  int32_t act_dtype;          /* 16-bit models: element type of activations, KV cache and P. 0 = LLAMA_F16
                                 (the default policy described above); LLAMA_BF16 (bf16 models only) keeps
                                 weights, activations, cache and P in bf16 as the pages compute (logits of a
                                 deep stack drift further from the exact result: see the dtype note) */
} llama_config;

typedef struct llama_model llama_model; /* opaque: weights, KV cache, lengths, workspace */

/* SwiGLU width from params.json: multiple_of * ceil(int(mult * floor(8*dim/3)) / multiple_of),
 * the multiplier step skipped when mult <= 0. ([W] 下载并读取模型权重 prints multiple_of and
 * ffn_dim_multiplier only; this reading gives 14336 for dim 4096.) */
int32_t llama_ffn_hidden(int32_t dim, int32_t multiple_of, float ffn_dim_multiplier);

/* Validates cfg, allocates weights, KV cache ([n_layers][max_batch][n_kv_heads][max_seq][head_dim]
 * for K and for V), the RoPE table and the workspace on the current device. Weights are zero until
 * llama_init_weights or llama_set_weight. All sequence lengths start at 0. Synchronous. */
int llama_create(const llama_config* cfg, llama_model** out);
void llama_destroy(llama_model* m);
/* Copy of the resolved configuration (ffn_hidden and max_tokens filled in). */
int llama_get_config(const llama_model* m, llama_config* out);
/* Bytes of device memory held by the model. */
size_t llama_device_bytes(const llama_model* m);

/* Seeded synthetic weights: every matrix N(0, std^2) from the counter-based generator
 * (SplitMix64 streams + Box-Muller, one stream per checkpoint key in the key order of
 * [W] 下载并读取模型权重), rounded to the model dtype (bf16 models: rounded to bf16, then held
 * as fp16); every norm weight 1.0. Produces the same values as the host generator in the
 * repository's seeded_inputs module. */
int llama_init_weights(llama_model* m, uint64_t seed, float std, void* stream);

/* Copy one checkpoint tensor in or out, by its checkpoint name ("tok_embeddings.weight",
 * "layers.{i}.attention.wq.weight", ..., "norm.weight", "output.weight"), in the checkpoint's
 * [out, in] layout and in the model dtype (norm weights are always fp32). nbytes must equal the
 * tensor's size. on_device: 1 if src/dst is device memory, 0 for host memory. */
int llama_set_weight(llama_model* m, const char* name, const void* src, size_t nbytes, int on_device, void* stream);
int llama_get_weight(llama_model* m, const char* name, void* dst, size_t nbytes, int on_device, void* stream);

/* Prefill: tokens (device int32 [B][S]) are appended to sequences 0..B-1 at positions
 * len[b] .. len[b]+S-1, their post-RoPE K and V written to the cache, and the last token's
 * logits of each sequence kept ([W] 预测下一个输出: final norm once, final_embedding[-1] @
 * output^T). Requires B <= max_batch, B*S <= max_tokens, len[b]+S <= max_seq. len[b] += S.
 * On a non-default stream the step is replayed from a CUDA graph kept per (B, S): the first call
 * for a shape runs eagerly, the second is captured, later calls replay it. Tokens are first
 * copied into a model-owned buffer, and positions and the block table are read from device
 * memory, so a replay always computes the current call. The default stream, profiling and the
 * environment variable LLAMA_NO_GRAPH keep every call eager. Graphs are kept until
 * llama_destroy, one per shape seen twice: a workload with many distinct prompt lengths should
 * prefill on the default stream (or set LLAMA_NO_GRAPH). A model must not be used from two host
 * threads at once. */
int llama_prefill(llama_model* m, const int32_t* tokens, int32_t B, int32_t S, void* stream);

/* One decode step: token b (device int32 [B]) is processed at position len[b] of sequence b,
 * attending to keys 0..len[b] through the cache; len[b] += 1. Logits are kept as for prefill.
 * Replayed from CUDA graphs as for prefill, one graph per (B, cache bound), the cache bound
 * being the longest sequence rounded up to 512 positions. */
int llama_decode_step(llama_model* m, const int32_t* tokens, int32_t B, void* stream);

/* fp32 logits [B][vocab] (device) of the last prefill or decode step. */
int llama_logits(llama_model* m, float* dst, void* stream);
/* Greedy next token of each sequence (device int32 [B]): the largest logit, the lowest index
 * among equal maxima ([W] 预测下一个输出: torch.argmax). */
int llama_argmax(llama_model* m, int32_t* dst, void* stream);

/* End to end from host memory: copies tokens (host int32 [B][S]) to the device, prefills, then
 * runs n_new greedy decode steps feeding each argmax back, and copies the B*(n_new+1) chosen
 * tokens ([B][n_new+1], host) back. Synchronizes the stream before returning. */
int llama_generate(llama_model* m, const int32_t* host_tokens, int32_t B, int32_t S, int32_t n_new,
                   int32_t* host_out, void* stream);

/* One decoder block on given hidden states: x (device fp32 [B][S][dim]) is the residual stream
 * entering layer `layer` at positions len[b]..len[b]+S-1; y (device fp32, same shape) receives
 * its output. The layer's cache entries are written; lengths are NOT advanced. */
int llama_block_forward(llama_model* m, int32_t layer, const float* x, float* y, int32_t B, int32_t S,
                        void* stream);

/* Cache and length control. llama_fill_kv_random writes N(0,1) K and V entries (taken as
 * already rotated) for positions 0..c-1 of every layer and every sequence < max_batch from the
 * seeded generator (layer l: stream 2^21+2l for K, +1 for V, element order [b][g][t][d]) and
 * sets every length to c (rounded as the weights are). llama_set_kv copies caller K/V (device, model dtype,
 * [B][n_kv_heads][c][head_dim]) into layer `layer`, positions 0..c-1. Lengths are host-visible
 * state: set_lengths takes host int32 [B] (B <= max_batch); reset sets all to 0. */
int llama_fill_kv_random(llama_model* m, uint64_t seed, int32_t c, void* stream);
int llama_set_kv(llama_model* m, int32_t layer, const void* k, const void* v, int32_t B, int32_t c, void* stream);
int llama_set_lengths(llama_model* m, const int32_t* host_len, int32_t B, void* stream);
int llama_get_lengths(const llama_model* m, int32_t* host_len, int32_t B);
/* Paged models: the block table of sequences 0..B-1 (host int32 [B][ceil(max_seq/128)]): the pool page
 * holding positions 128j .. 128j+127 of sequence b, -1 past its pages. LLAMA_ERR_UNSUPPORTED when the
 * cache is contiguous. */
int llama_get_block_table(const llama_model* m, int32_t* host_table, int32_t B);
int llama_reset(llama_model* m, void* stream);

/* Per-kernel timing of eager model calls: while enabled (1), an event is recorded on the
 * launching stream before every kernel launch of prefill/decode/argmax (CUDA-graph replay is
 * bypassed). llama_profile_read synchronizes, then fills ms[k] (summed time from the launch's
 * event to the next one) and launches[k] for kinds k < n_kinds, clears the record and returns
 * the number of kinds (embed, rmsnorm, gemm_qkv_rope, attention_prefill, attention_decode,
 * gemm_wo_residual, gemm_w13_swiglu, gemm_w2_residual, gemm_lm_head, other, gemm_chain: one prefill
 * launch running a layer's Wo, w1/w3 and w2 projections and the next layer's QKV projection). */
int llama_profile(llama_model* m, int enable);
int llama_profile_read(llama_model* m, double* ms, int64_t* launches, int n_kinds);
const char* llama_profile_kind_name(int kind);
/* Kernels launched by this library in this process so far (CUDA-graph replays count the
 * kernels they contain). */
uint64_t llama_kernel_launches(void);

/* Synchronizes `stream`, then returns and clears the model's latched device status. */
int llama_sync_status(llama_model* m, void* stream);
const char* llama_status_string(int status);

/* ---------------------------------------------------------------- stateless kernels
 * Same kernels as the model, on caller buffers (device pointers, dtype = element type of
 * q/k/v/o/x/w). They use library-owned scratch on the current device, allocated on first use. */

/* Causal GQA attention for prefill ([W] 查询和键相乘, 掩码, 多头注意力): q [B][H][S][d],
 * k, v [B][Hk][S][d] (already rotated), o [B][S][H*d]; query s sees keys 0..s; head h reads kv
 * head h / (H/Hk); scores scaled by 1/sqrt(d). bf16 and fp16 require d = 128; fp32 takes d in
 * {32,64,128}. */
int llama_attention_prefill(const void* q, const void* k, const void* v, void* o, int32_t B, int32_t S, int32_t H,
                            int32_t Hk, int32_t d, int32_t dtype, void* stream);

/* Single-query attention over a cache (decode): q [B][H][d]; kc, vc [B][Hk][cmax][d]; len
 * (device int32 [B], 1 <= len[b] <= cmax) = number of valid keys of sequence b; o [B][H*d].
 * Split over the key range, merged with the log-sum-exp rule. d in {64,128} (bf16, fp16) or
 * {32,64,128} (fp32); H/Hk <= 8. A len[b] outside [1, cmax] gives a NaN row for sequence b (the
 * other rows are computed normally) and latches LLAMA_ERR_DEVICE_BOUNDS for llama_status(). */
int llama_attention_decode(const void* q, const void* kc, const void* vc, const int32_t* len, void* o, int32_t B,
                           int32_t cmax, int32_t H, int32_t Hk, int32_t d, int32_t dtype, void* stream);

/* llama_attention_decode for callers that cannot let this library allocate device memory.
 * Some programs own all of the GPU's memory through their own allocator or pool (a serving
 * engine's preallocated cache pool, a framework's caching allocator that has reserved most of
 * the card): a cudaMalloc made behind their back can fail or fragment that pool, and a
 * cudaMalloc/cudaFree inside a latency-critical loop synchronizes the whole device. This call
 * never allocates or frees device memory; everything else is the same as
 * llama_attention_decode (arguments, layouts, results, bit for bit).
 * Its split partials live in one static 8 MiB device array that every GPU which loads this
 * library keeps until the process exits. Calls needing more than 8 MiB of partials return
 * LLAMA_ERR_SHAPE: for bf16 or fp16 with d = 128 the partials take at most
 * (B*Hk + 12*SMs) * (H/Hk) * (d+2) * 4 + 16 bytes (SMs = 148 on B200; (B*Hk + 4*SMs) * ... when
 * B*Hk*ceil(cmax/32) < 512*SMs), so with H = 32, Hk = 8 every B up to 280 fits whatever cmax.
 * Device-side errors of the call (a len[b] outside [1, cmax], which also gives a NaN row; a
 * bounded wait that gave up) are latched in a static status word of its own, next to the
 * array; llama_status() returns and clears it, and allocates nothing when only this call ran.
 * The first call on a device looks up the array's and the status word's device addresses for
 * that device (cudaGetSymbolAddress); make that first call before any stream capture begins.
 * The lookup is repeated after the device's context changed (cudaDeviceReset).
 * Every call uses the same array and status word, so calls that may run at the same time on
 * the GPU (e.g. on two streams) race: order them. Nothing has to be cleared between calls,
 * since every partial is written before it is read.
 * The pages have no counterpart of this entry point: it exists for deployment only. */
int llama_attention_decode_noalloc(const void* q, const void* kc, const void* vc, const int32_t* len, void* o,
                                   int32_t B, int32_t cmax, int32_t H, int32_t Hk, int32_t d, int32_t dtype,
                                   void* stream);

/* Paged-cache forms (16-bit, d = 128): k_pages, v_pages [n_pages][Hk][128][d]; table (device int32
 * [B][max_pages]) gives page j of sequence b (keys 128j .. 128j+127); entries must lie in [-1, n_pages),
 * -1 marking an unused slot, else LLAMA_ERR_SHAPE (the table is read back to the host to check it).
 * Prefill: q [B][H][S][d]; sequence b's S queries sit at positions pos0[b] .. pos0[b]+S-1 (pos0 device
 * int32 [B], NULL = all 0) and see keys 0 .. their own position, which the caller has already written into
 * the pages; o [B][S][H*d]. Decode: q [B][H][d], len (device int32 [B]) keys per sequence, o [B][H*d].
 * Same kernels as the model's paged cache ([W] 查询和键相乘, 掩码; [H]: the cache sized by max_seq_len). */
int llama_attention_prefill_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* table,
                                  int32_t max_pages, int32_t n_pages, const int32_t* pos0, void* o, int32_t B,
                                  int32_t S, int32_t H, int32_t Hk, int32_t d, int32_t dtype, void* stream);
int llama_attention_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* table,
                                 int32_t max_pages, int32_t n_pages, const int32_t* len, void* o, int32_t B,
                                 int32_t H, int32_t Hk, int32_t d, int32_t dtype, void* stream);

/* y = x W^T: x [M][K], w [N][K] (dtype), y fp32 [M][N]. variant 0 = automatic, 1 = the wide
 * persistent tcgen05 kernel, 2 = the skinny split-K tcgen05 kernel (M <= 256); fp32 ignores it.
 * bf16 and fp16 require K % 8 == 0 and 16-byte aligned x and w. */
int llama_linear(const void* x, const void* w, float* y, int32_t M, int32_t N, int32_t K, int32_t dtype,
                 int32_t variant, void* stream);

/* y = x * rsqrt(mean(x^2) + eps) * g per row ([W] 构建Transformer层): x fp32 [M][D], g fp32 [D],
 * y [M][D] in dtype. */
int llama_rmsnorm(const float* x, const float* g, void* y, int32_t M, int32_t D, float eps, int32_t dtype,
                  void* stream);

/* Row-wise argmax of fp32 logits [B][V] into int32 [B], lowest index among equal maxima. */
int llama_argmax_rows(const float* logits, int32_t* out, int32_t B, int32_t V, void* stream);

/* n draws of N(0, std^2) of stream `stream_id` under `seed` (the weight generator) into dst
 * (device, dtype; fp16 rounds the fp32 draw to fp16 directly). */
int llama_fill_normal(void* dst, int64_t n, uint64_t seed, uint64_t stream_id, float std, int32_t dtype,
                      void* stream);

/* Failure-detection self test. Every spin-wait of the library's kernels (on an mbarrier, or on a
 * counter other CTAs increment) is bounded: after its limit (2 s in the kernels) it latches
 * LLAMA_ERR_DEVICE_TIMEOUT in the status word and the kernel returns, so a stuck wait never hangs
 * the GPU and the context stays usable. This call runs one such wait that can never complete
 * (kind 0: the first phase of an mbarrier nobody arrives on; kind 1: a device counter nobody
 * increments) with the limit limit_ns (1 .. 10^10); llama_status() then returns
 * LLAMA_ERR_DEVICE_TIMEOUT. Not part of the pages' method: it tests the library's failure handling. */
int llama_wait_selftest(int32_t kind, uint64_t limit_ns, void* stream);

/* Synchronizes `stream`, then returns and clears the status word of the stateless calls on the
 * current device (the first non-zero of theirs and llama_attention_decode_noalloc's). */
int llama_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LLAMA_B200_H */
