// Bandwidth-bound kernels around the GEMMs: embedding gather, RMSNorm,
// greedy argmax, per-sequence length update, and the seeded generator that
// stands in for checkpoint weights and synthetic inputs.
#include "common.cuh"
#include "kernels.h"

namespace llama {

namespace {

// ------------------------------------------------------------- embedding
// x[m, :] = table[tokens[m], :] widened to fp32 (row gather of tok_embeddings).
template <typename T>
__global__ void embed_kernel(const int32_t* __restrict__ tokens, const T* __restrict__ table, int V, int D,
                             float* __restrict__ x, int* status) {
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x;
  const int tok = tokens[m];
  float* dst = x + (size_t)m * D;
  if (tok < 0 || tok >= V) {
    if (threadIdx.x == 0) set_status(status, LLAMA_ERR_DEVICE_BOUNDS);
    for (int i = threadIdx.x; i < D; i += blockDim.x) dst[i] = 0.f;
    return;
  }
  const T* src = table + (size_t)tok * D;
  for (int i = threadIdx.x; i < D; i += blockDim.x) dst[i] = to_f<T>(src[i]);
}

// ---------------------------------------------------------------- RMSNorm
// y = x * rsqrt(mean(x^2) + eps) * g over one row of D fp32 values.
template <typename T>
__device__ __forceinline__ void store4(T* p, float a, float b, float c, float d) {
  if constexpr (sizeof(T) == 2) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack2<T>(a, b), pack2<T>(c, d));
  } else {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
  }
}

// One row per 256-thread block. Rows with D % 4 == 0 and D <= 8192 stay in
// registers between the sum of squares and the scaling (x is read once) and
// are written with 8- or 16-byte stores.
template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                                      T* __restrict__ y, int D, float eps, int last_of_S,
                                                      int* status) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x;
  const size_t src_row = last_of_S > 0 ? (size_t)(r + 1) * last_of_S - 1 : (size_t)r;
  const float* xr = x + src_row * D;
  T* yr = y + (size_t)r * D;
  __shared__ float red[8];
  constexpr int NV = 8;  // float4 per thread in the register path
  const bool vec = (D % 4 == 0) && D <= NV * 4 * 256 && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(g)) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(y) & 15) == 0;
  float4 v[NV];
  float ss = 0.f;
  if (vec) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int i = (threadIdx.x + k * 256) * 4;
      v[k] = i < D ? __ldcs(reinterpret_cast<const float4*>(xr + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
      ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
    }
  } else {
    for (int i = threadIdx.x; i < D; i += 256) ss += xr[i] * xr[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += red[w];
  const float inv = rsqrtf(tot / (float)D + eps);
  bool bad = false;
  if (vec) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int i = (threadIdx.x + k * 256) * 4;
      if (i < D) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(g + i));
        const float4 o = make_float4(v[k].x * inv * w.x, v[k].y * inv * w.y, v[k].z * inv * w.z, v[k].w * inv * w.w);
        bad |= nonfinite16<T>(o.x) | nonfinite16<T>(o.y) | nonfinite16<T>(o.z) | nonfinite16<T>(o.w);
        store4<T>(yr + i, o.x, o.y, o.z, o.w);
      }
    }
  } else {
    for (int i = threadIdx.x; i < D; i += 256) {
      const float o = xr[i] * inv * g[i];
      bad |= nonfinite16<T>(o);
      yr[i] = from_f<T>(o);
    }
  }
  if (bad) set_status(status, LLAMA_ERR_RANGE);
}

// Inputs of a GEMM with the RMSNorm folded in: y = x * g (16-bit, not yet
// scaled by rsqrt(mean(x^2)+eps)) and the row's sum of squares in slot 0 of
// its ss_n partial sums (the other slots 0).
template <typename T>
__global__ void __launch_bounds__(256) norm_prep_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                                        T* __restrict__ y, float* __restrict__ ss, int D, int ss_n,
                                                        int* status) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x;
  const float* xr = x + (size_t)r * D;
  T* yr = y + (size_t)r * D;
  __shared__ float red[8];
  float acc = 0.f;
  bool bad = false;
  for (int i = threadIdx.x; i < D; i += 256) {
    const float v = xr[i];
    acc += v * v;
    bad |= nonfinite16<T>(v * g[i]);
    yr[i] = from_f<T>(v * g[i]);
  }
  if (bad) set_status(status, LLAMA_ERR_RANGE);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < ss_n) {
    float tot = 0.f;
    if (threadIdx.x == 0)
      for (int w = 0; w < 8; ++w) tot += red[w];
    ss[(size_t)r * ss_n + threadIdx.x] = tot;
  }
}

// ----------------------------------------------------------------- argmax
// Greedy next token: largest logit, lowest index among equal maxima.
__device__ __forceinline__ void better(float& bv, int& bi, float v, int i) {
  if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
}

__global__ void __launch_bounds__(1024) argmax_kernel(const float* __restrict__ logits, int32_t* out, int V) {
  pdl_trigger();
  pdl_wait();
  const float* row = logits + (size_t)blockIdx.x * V;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int i = threadIdx.x; i < V; i += 1024) better(bv, bi, row[i], i);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    better(bv, bi, ov, oi);
  }
  __shared__ float sv[32];
  __shared__ int si[32];
  if ((threadIdx.x & 31) == 0) { sv[threadIdx.x >> 5] = bv; si[threadIdx.x >> 5] = bi; }
  __syncthreads();
  if (threadIdx.x < 32) {
    bv = sv[threadIdx.x];
    bi = si[threadIdx.x];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      better(bv, bi, ov, oi);
    }
    if (threadIdx.x == 0) out[blockIdx.x] = bi == 0x7fffffff ? 0 : bi;
  }
}

__global__ void add_lengths_kernel(int32_t* len, int B, int add) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) len[b] += add;
}

// -------------------------------------------------------- seeded generator
// SplitMix64 counter streams and Box-Muller, with ln and cos(2*pi*t) built
// from correctly rounded IEEE operations only (explicit _rn intrinsics, so
// nothing is fused): bit-identical to the host generator.
#define SG 0x9E3779B97F4A7C15ULL
#define SM1 0xBF58476D1CE4E5B9ULL
#define SM2 0x94D049BB133111EBULL

__constant__ double kCos[10] = {0x1.0000000000000p+0, -0x1.0000000000000p-1, 0x1.5555555555555p-5,
                                -0x1.6c16c16c16c17p-10, 0x1.a01a01a01a01ap-16, -0x1.27e4fb7789f5cp-22,
                                0x1.1eed8eff8d898p-29, -0x1.93974a8c07c9dp-37, 0x1.ae7f3e733b81fp-45,
                                -0x1.6827863b97d97p-53};
__constant__ double kSin[10] = {0x1.0000000000000p+0, -0x1.5555555555555p-3, 0x1.1111111111111p-7,
                                -0x1.a01a01a01a01ap-13, 0x1.71de3a556c734p-19, -0x1.ae64567f544e4p-26,
                                0x1.6124613a86d09p-33, -0x1.ae7f3e733b81fp-41, 0x1.952c77030ad4ap-49,
                                -0x1.2f49b46814157p-57};
__constant__ double kAtanh[11] = {0x1.0000000000000p+0, 0x1.5555555555555p-2, 0x1.999999999999ap-3,
                                  0x1.2492492492492p-3, 0x1.c71c71c71c71cp-4, 0x1.745d1745d1746p-4,
                                  0x1.3b13b13b13b14p-4, 0x1.1111111111111p-4, 0x1.e1e1e1e1e1e1ep-5,
                                  0x1.af286bca1af28p-5, 0x1.8618618618618p-5};

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * SM1;
  z = (z ^ (z >> 27)) * SM2;
  return z ^ (z >> 31);
}

__device__ __forceinline__ double det_log(double u) {
  int e;
  double m = frexp(u, &e);
  if (m < 0x1.6a09e667f3bcdp-1) { m = __dmul_rn(m, 2.0); e -= 1; }
  const double s = __ddiv_rn(__dsub_rn(m, 1.0), __dadd_rn(m, 1.0));
  const double s2 = __dmul_rn(s, s);
  double p = kAtanh[10];
#pragma unroll
  for (int k = 9; k >= 0; --k) p = __dadd_rn(__dmul_rn(p, s2), kAtanh[k]);
  return __dadd_rn(__dmul_rn((double)e, 0x1.62e42fefa39efp-1), __dmul_rn(__dmul_rn(2.0, s), p));
}

__device__ __forceinline__ double det_cos2pi(double t) {
  if (t > 0.5) t = __dsub_rn(1.0, t);
  const bool neg = t > 0.25;
  if (neg) t = __dsub_rn(0.5, t);
  const bool use_sin = t > 0.125;
  const double x = __dmul_rn(use_sin ? __dsub_rn(0.25, t) : t, 0x1.921fb54442d18p+2);
  const double x2 = __dmul_rn(x, x);
  double r;
  if (use_sin) {
    double p = kSin[9];
#pragma unroll
    for (int k = 8; k >= 0; --k) p = __dadd_rn(__dmul_rn(p, x2), kSin[k]);
    r = __dmul_rn(x, p);
  } else {
    double p = kCos[9];
#pragma unroll
    for (int k = 8; k >= 0; --k) p = __dadd_rn(__dmul_rn(p, x2), kCos[k]);
    r = p;
  }
  return neg ? -r : r;
}

__device__ __forceinline__ float seeded_normal(uint64_t key, uint64_t i, double sd) {
  const uint64_t d0 = mix64(key + (2 * i + 1) * SG);
  const uint64_t d1 = mix64(key + (2 * i + 2) * SG);
  const double u1 = (double)((d0 >> 11) + 1) * 0x1p-53;
  const double u2 = (double)(d1 >> 11) * 0x1p-53;
  const double z = __dmul_rn(__dsqrt_rn(__dmul_rn(-2.0, det_log(u1))), det_cos2pi(u2));
  return __double2float_rn(__dmul_rn(z, sd));
}

template <typename T, bool ROUND_BF16>
__global__ void fill_normal_kernel(T* __restrict__ dst, FillLayout L, uint64_t key, double sd) {
  const int64_t n = L.outer * L.rows * L.cols;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i % L.cols;
    const int64_t t = i / L.cols;
    const int64_t r = t % L.rows;
    const int64_t o = t / L.rows;
    const int64_t phys = o * L.outer_stride + (r * L.row_mult + L.row_off) * L.row_stride + c;
    float v = seeded_normal(key, (uint64_t)i, sd);
    if (ROUND_BF16) v = __bfloat162float(__float2bfloat16_rn(v));
    dst[phys] = from_f<T>(v);
  }
}

__global__ void fill_const_kernel(float* dst, int64_t n, float v) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = v;
}

int grid_for(int64_t n) {
  int64_t g = (n + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 16;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

uint64_t stream_key(uint64_t seed, uint64_t stream) { return mix64(seed * SG + stream * SM1 + SG); }

int launch_embed(const int32_t* tokens, int M, const void* table, int V, int D, int dtype, float* x, int* status,
                 cudaStream_t st) {
  if (M <= 0) return LLAMA_OK;
  cudaError_t err;
  if (dtype == LLAMA_F16)
    err = launch_k(embed_kernel<f16>, dim3(M), dim3(256), 0, st, tokens, static_cast<const f16*>(table), V, D, x,
                   status);
  else if (dtype == LLAMA_BF16)
    err = launch_k(embed_kernel<bf16>, dim3(M), dim3(256), 0, st, tokens, static_cast<const bf16*>(table), V, D, x,
                   status);
  else
    err = launch_k(embed_kernel<float>, dim3(M), dim3(256), 0, st, tokens, static_cast<const float*>(table), V, D, x,
                   status);
  return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int launch_rmsnorm(const float* x, const float* g, void* y, int rows, int D, float eps, int last_of_S, int dtype,
                   cudaStream_t st, int* status) {
  if (rows <= 0) return LLAMA_OK;
  cudaError_t err;
  if (dtype == LLAMA_F16)
    err = launch_k(rmsnorm_kernel<f16>, dim3(rows), dim3(256), 0, st, x, g, static_cast<f16*>(y), D, eps, last_of_S,
                   status);
  else if (dtype == LLAMA_BF16)
    err = launch_k(rmsnorm_kernel<bf16>, dim3(rows), dim3(256), 0, st, x, g, static_cast<bf16*>(y), D, eps,
                   last_of_S, status);
  else
    err = launch_k(rmsnorm_kernel<float>, dim3(rows), dim3(256), 0, st, x, g, static_cast<float*>(y), D, eps,
                   last_of_S, status);
  return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int launch_norm_prep(const float* x, const float* g, void* y, float* ss, int rows, int D, int ss_n, int dtype,
                     cudaStream_t st, int* status) {
  if (rows <= 0) return LLAMA_OK;
  if (ss_n > 256) return LLAMA_ERR_INVALID_ARG;
  cudaError_t err;
  if (dtype == LLAMA_F16)
    err = launch_k(norm_prep_kernel<f16>, dim3(rows), dim3(256), 0, st, x, g, static_cast<f16*>(y), ss, D, ss_n,
                   status);
  else if (dtype == LLAMA_BF16)
    err = launch_k(norm_prep_kernel<bf16>, dim3(rows), dim3(256), 0, st, x, g, static_cast<bf16*>(y), ss, D, ss_n,
                   status);
  else
    return LLAMA_ERR_INVALID_ARG;
  return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int launch_argmax(const float* logits, int32_t* out, int B, int V, cudaStream_t st) {
  if (B <= 0) return LLAMA_OK;
  return launch_k(argmax_kernel, dim3(B), dim3(1024), 0, st, logits, out, V) == cudaSuccess ? LLAMA_OK
                                                                                           : LLAMA_ERR_CUDA;
}

int launch_add_lengths(int32_t* len, int B, int add, cudaStream_t st) {
  if (B <= 0) return LLAMA_OK;
  return launch_k(add_lengths_kernel, dim3((B + 255) / 256), dim3(256), 0, st, len, B, add) == cudaSuccess
             ? LLAMA_OK
             : LLAMA_ERR_CUDA;
}

int launch_fill_normal(void* dst, const FillLayout& L, uint64_t seed, uint64_t stream_id, float std, int dtype,
                       cudaStream_t st, bool round_bf16) {
  const int64_t n = L.outer * L.rows * L.cols;
  if (n <= 0) return LLAMA_OK;
  const uint64_t key = stream_key(seed, stream_id);
  const double sd = (double)std;
  count_launches(1);
  if (dtype == LLAMA_BF16)
    fill_normal_kernel<bf16, false><<<grid_for(n), 256, 0, st>>>(static_cast<bf16*>(dst), L, key, sd);
  else if (dtype == LLAMA_F16 && round_bf16)
    fill_normal_kernel<f16, true><<<grid_for(n), 256, 0, st>>>(static_cast<f16*>(dst), L, key, sd);
  else if (dtype == LLAMA_F16)
    fill_normal_kernel<f16, false><<<grid_for(n), 256, 0, st>>>(static_cast<f16*>(dst), L, key, sd);
  else
    fill_normal_kernel<float, false><<<grid_for(n), 256, 0, st>>>(static_cast<float*>(dst), L, key, sd);
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

namespace {
// dst[r][c] = src[r][c] converted between 16-bit types (elt codes LLAMA_BF16 / LLAMA_F16).
template <typename D, typename S>
__global__ void convert_2d_kernel(D* __restrict__ dst, int64_t dpitch, const S* __restrict__ src, int64_t spitch,
                                  int64_t rows, int64_t cols) {
  const int64_t n = rows * cols;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / cols, c = i - r * cols;
    dst[r * dpitch + c] = from_f<D>(to_f<S>(src[r * spitch + c]));
  }
}
}  // namespace

int launch_convert_2d(void* dst, int64_t dpitch, int dst_elt, const void* src, int64_t spitch, int src_elt,
                      int64_t rows, int64_t cols, cudaStream_t st) {
  const int64_t n = rows * cols;
  if (n <= 0) return LLAMA_OK;
  count_launches(1);
  if (dst_elt == LLAMA_F16 && src_elt == LLAMA_BF16)
    convert_2d_kernel<f16, bf16><<<grid_for(n), 256, 0, st>>>(static_cast<f16*>(dst), dpitch,
                                                              static_cast<const bf16*>(src), spitch, rows, cols);
  else if (dst_elt == LLAMA_BF16 && src_elt == LLAMA_F16)
    convert_2d_kernel<bf16, f16><<<grid_for(n), 256, 0, st>>>(static_cast<bf16*>(dst), dpitch,
                                                              static_cast<const f16*>(src), spitch, rows, cols);
  else
    return LLAMA_ERR_INVALID_ARG;
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

namespace {
// Element i of the logical cache [B][Hk][c][d] (the generator's order) is
// written through the cache layout L.
template <typename T, bool ROUND_BF16>
__global__ void fill_kv_kernel(T* __restrict__ dst, KvLayout L, int Hk, int c, int d, int64_t n, uint64_t key,
                               double sd) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int dd = (int)(i % d);
    const int64_t r = i / d;
    const int t = (int)(r % c);
    const int64_t bg = r / c;
    const int g = (int)(bg % Hk), b = (int)(bg / Hk);
    float v = seeded_normal(key, (uint64_t)i, sd);
    if (ROUND_BF16) v = __bfloat162float(__float2bfloat16_rn(v));
    dst[kv_row(L, Hk, b, g, t) * d + dd] = from_f<T>(v);
  }
}

// dst (through L) <- src [B][Hk][c][d], converting S -> D.
template <typename D, typename S>
__global__ void kv_scatter_kernel(D* __restrict__ dst, KvLayout L, int Hk, int c, int d, const S* __restrict__ src,
                                  int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int dd = (int)(i % d);
    const int64_t r = i / d;
    const int t = (int)(r % c);
    const int64_t bg = r / c;
    const int g = (int)(bg % Hk), b = (int)(bg / Hk);
    dst[kv_row(L, Hk, b, g, t) * d + dd] = from_f<D>(to_f<S>(src[i]));
  }
}
}  // namespace

int launch_fill_kv(void* dst, const KvLayout& L, int B, int Hk, int c, int d, uint64_t seed, uint64_t stream_id,
                   float std, int dtype, bool round_bf16, cudaStream_t st) {
  const int64_t n = (int64_t)B * Hk * c * d;
  if (n <= 0) return LLAMA_OK;
  const uint64_t key = stream_key(seed, stream_id);
  count_launches(1);
  if (dtype == LLAMA_F16 && round_bf16)
    fill_kv_kernel<f16, true><<<grid_for(n), 256, 0, st>>>(static_cast<f16*>(dst), L, Hk, c, d, n, key, std);
  else if (dtype == LLAMA_F16)
    fill_kv_kernel<f16, false><<<grid_for(n), 256, 0, st>>>(static_cast<f16*>(dst), L, Hk, c, d, n, key, std);
  else if (dtype == LLAMA_BF16)
    fill_kv_kernel<bf16, false><<<grid_for(n), 256, 0, st>>>(static_cast<bf16*>(dst), L, Hk, c, d, n, key, std);
  else
    fill_kv_kernel<float, false><<<grid_for(n), 256, 0, st>>>(static_cast<float*>(dst), L, Hk, c, d, n, key, std);
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int launch_kv_scatter(void* dst, int dst_elt, const KvLayout& L, int B, int Hk, int c, int d, const void* src,
                      int src_elt, cudaStream_t st) {
  const int64_t n = (int64_t)B * Hk * c * d;
  if (n <= 0) return LLAMA_OK;
  count_launches(1);
#define LLAMA_SCATTER(DT, ST) \
  kv_scatter_kernel<DT, ST><<<grid_for(n), 256, 0, st>>>(static_cast<DT*>(dst), L, Hk, c, d, static_cast<const ST*>(src), n)
  if (dst_elt == LLAMA_F16 && src_elt == LLAMA_BF16) LLAMA_SCATTER(f16, bf16);
  else if (dst_elt == LLAMA_F16 && src_elt == LLAMA_F16) LLAMA_SCATTER(f16, f16);
  else if (dst_elt == LLAMA_BF16 && src_elt == LLAMA_BF16) LLAMA_SCATTER(bf16, bf16);
  else if (dst_elt == LLAMA_F32 && src_elt == LLAMA_F32) LLAMA_SCATTER(float, float);
  else return LLAMA_ERR_INVALID_ARG;
#undef LLAMA_SCATTER
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

namespace {
// A counter nothing ever increments (the target of the counter self test).
__device__ int g_never_set = 0;

// Failure-detection self test: one thread waits for something that never
// happens (kind 0: the first phase of an mbarrier nobody arrives on; kind 1:
// a device counter nobody increments), through the same bounded waits as the
// kernels use, with the given limit. The wait gives up, latches
// LLAMA_ERR_DEVICE_TIMEOUT and the kernel returns.
__global__ void wait_selftest_kernel(int kind, uint64_t limit_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  if (kind == 0) mbar_wait(&bar, 0, status, limit_ns);
  else counter_wait_geq(&g_never_set, 1, status, limit_ns);
}
}  // namespace

int launch_wait_selftest(int kind, uint64_t limit_ns, int* status, cudaStream_t st) {
  count_launches(1);
  wait_selftest_kernel<<<1, 32, 0, st>>>(kind, limit_ns, status);
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int launch_fill_const(float* dst, int64_t n, float v, cudaStream_t st) {
  if (n <= 0) return LLAMA_OK;
  count_launches(1);
  fill_const_kernel<<<grid_for(n), 256, 0, st>>>(dst, n, v);
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

}  // namespace llama
