// fp32 GEMM on the CUDA cores for the single-precision model (the fp32
// configuration must stay within 1e-3 of the oracle, which TF32 tensor cores
// would not). 64x64 output tiles, 256 threads with 4x4 register micro-tiles,
// K staged through shared memory 16 at a time. Same epilogues as the bf16 path.
#include "epilogue.cuh"
#include "kernels.h"

namespace llama {

namespace {
constexpr int TM = 64, TN = 64, TK = 16;

template <int KIND>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, int M, int K, int lda,
                                                       const float* __restrict__ W, int N, int ldw, EpiArgs e) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Ws[TK][TN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int i = threadIdx.x; i < TM * TK; i += 256) {
      const int r = i / TK, c = i % TK;
      const int gm = m0 + r, gn = n0 + r, gk = k0 + c;
      As[c][r] = (gm < M && gk < K) ? A[(size_t)gm * lda + gk] : 0.f;
      Ws[c][r] = (gn < N && gk < K) ? W[(size_t)gn * ldw + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Ws[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      epi_elem<KIND, float>(e, m0 + ty * 4 + i, n0 + tx * 4 + j, acc[i][j], acc[i][j ^ 1]);
}
}  // namespace

int gemm_f32(const float* A, int M, int K, int lda, const float* W, int N, int ldw, int kind, const EpiArgs& e,
             int* status, cudaStream_t st) {
  (void)status;
  if (M <= 0 || N <= 0 || K <= 0) return LLAMA_ERR_SHAPE;
  dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
  count_launches(1);
  switch (kind) {
    case EPI_STORE_F32: gemm_f32_kernel<EPI_STORE_F32><<<grid, 256, 0, st>>>(A, M, K, lda, W, N, ldw, e); break;
    case EPI_RESIDUAL: gemm_f32_kernel<EPI_RESIDUAL><<<grid, 256, 0, st>>>(A, M, K, lda, W, N, ldw, e); break;
    case EPI_SWIGLU: gemm_f32_kernel<EPI_SWIGLU><<<grid, 256, 0, st>>>(A, M, K, lda, W, N, ldw, e); break;
    case EPI_QKV_ROPE: gemm_f32_kernel<EPI_QKV_ROPE><<<grid, 256, 0, st>>>(A, M, K, lda, W, N, ldw, e); break;
    default: return LLAMA_ERR_INVALID_ARG;
  }
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

}  // namespace llama
