// Causal GQA prefill attention on the 5th-generation tensor cores (16-bit
// q/k/v, bf16 or fp16, head_dim 128).
//
// One CTA computes 128 queries of one head. Warp roles: warp 0 issues TMA
// loads (Q once, then K and V tiles of 128 keys into a 2-stage ring), warp 1
// allocates TMEM and issues tcgen05.mma, warps 2-5 own one query row per
// thread for the softmax and the final normalisation.
//
//   S_j = Q K_j^T      -> TMEM (two 128-column buffers, so S_{j+1} is computed
//                         while the softmax works on S_j)
//   P_j = exp2(S_j*c - m) rounded to the 16-bit type (the walkthrough rounds
//                         softmax(...) to 16 bits before the value product)
//                      -> shared memory, 128-byte swizzled K-major rows
//   O  += P_j V_j      -> TMEM (128 columns); V is read MN-major straight from
//                         the cache layout [key][d].
//
// The running maximum m is only raised when a row's new maximum exceeds it by
// more than 8 (a factor 256 in exp2 space), so O in TMEM is rescaled rarely;
// O / l is exact for any m used consistently. Query i of the tile sits at
// absolute position pos0 + q0 + i and sees keys 0 .. pos0 + q0 + i.
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace llama {

namespace {

constexpr int FA_BM = 128, FA_BN = 128, FA_D = 128;
constexpr int FA_HALF = FA_BM * 64 * 2;              // one 64-column swizzled block: 16 KB
constexpr int FA_Q_BYTES = 2 * FA_HALF;               // 32 KB
constexpr int FA_KV_BYTES = 2 * FA_HALF;              // K (or V) tile: 32 KB
constexpr int FA_STAGES = 2;
constexpr int FA_OFF_Q = 0;
constexpr int FA_OFF_K = FA_OFF_Q + FA_Q_BYTES;
constexpr int FA_OFF_V = FA_OFF_K + FA_STAGES * FA_KV_BYTES;
constexpr int FA_OFF_P = FA_OFF_V + FA_STAGES * FA_KV_BYTES;
constexpr int FA_OFF_BAR = FA_OFF_P + FA_Q_BYTES;
constexpr int FA_SMEM = FA_OFF_BAR + 256 + 1024;
constexpr uint32_t FA_TMEM_O = 0, FA_TMEM_S = 128;   // S buffers at columns 128 and 256
constexpr float FA_RESCALE = 8.0f;                    // raise the running max only past +8 (log2)

// 2^x with the hardware approximation (flushes results below 2^-126 to zero,
// which only affects probabilities too small to matter in a bf16 P).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint8_t* fa_align(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <typename T>
__global__ void __launch_bounds__(192, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, T* __restrict__ o,
                           const int32_t* __restrict__ pos0, int S, int H, int Hk, float scale_log2, int* status) {
  extern __shared__ uint8_t fa_smem_raw[];
  uint8_t* smem = fa_align(fa_smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + FA_OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;    // [2]
  uint64_t* kv_empty = bars + 3;   // [2]
  uint64_t* s_full = bars + 5;     // [2]
  uint64_t* p_full = bars + 7;
  uint64_t* o_done = bars + 8;
  uint64_t* drain = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Linear block order is longest-first across all heads and sequences
  // (CTAs start roughly in block order), so the causal work packs evenly.
  const int nqt = (S + FA_BM - 1) / FA_BM;
  const int HB = gridDim.x / nqt;                       // heads x sequences
  const int hb = blockIdx.x % HB;
  const int qt = nqt - 1 - (int)(blockIdx.x / HB);
  const int h = hb % H, b = hb / H;
  const int g = h / (H / Hk);
  const int q0 = qt * FA_BM;

  pdl_trigger();
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); mbar_init(&s_full[i], 1); }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();

  const int p0 = pos0 ? pos0[b] : 0;
  const int n_keys = p0 + S;                              // keys of this sequence
  const int k_end = min(n_keys, p0 + q0 + FA_BM);         // keys this tile needs
  const int n_kt = (k_end + FA_BN - 1) / FA_BN;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    mbar_arrive_expect_tx(q_full, FA_Q_BYTES);
    tma_load_3d(smem + FA_OFF_Q, &tmQ, q_full, 0, q0, b * H + h);
    tma_load_3d(smem + FA_OFF_Q + FA_HALF, &tmQ, q_full, 64, q0, b * H + h);
    int issued = 0;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      const int st = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      if (!mbar_wait(&kv_empty[st], ph ^ 1, status)) { ok = false; break; }
      mbar_arrive_expect_tx(&kv_full[st], 2 * FA_KV_BYTES);
      uint8_t* kd = smem + FA_OFF_K + st * FA_KV_BYTES;
      uint8_t* vd = smem + FA_OFF_V + st * FA_KV_BYTES;
      tma_load_3d(kd, &tmK, &kv_full[st], 0, j * FA_BN, b * Hk + g);
      tma_load_3d(kd + FA_HALF, &tmK, &kv_full[st], 64, j * FA_BN, b * Hk + g);
      tma_load_3d(vd, &tmV, &kv_full[st], 0, j * FA_BN, b * Hk + g);
      tma_load_3d(vd + FA_HALF, &tmV, &kv_full[st], 64, j * FA_BN, b * Hk + g);
      ++issued;
    }
    if (!ok) {  // let issued copies land before the CTA can exit
      mbar_wait(q_full, 0, status);
      for (int j = issued - 1; j >= 0 && j >= issued - 2; --j) mbar_wait(&kv_full[j & 1], (j >> 1) & 1, status);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc_s = umma_idesc_16(UmmaFmt<T>::value, FA_BM, FA_BN, false);
    constexpr uint32_t idesc_o = umma_idesc_16(UmmaFmt<T>::value, FA_BM, FA_D, true);
    const uint32_t q_addr = smem_u32(smem + FA_OFF_Q), p_addr = smem_u32(smem + FA_OFF_P);
    bool ok = mbar_wait(q_full, 0, status), any = false;
    auto issue_s = [&](int j) -> bool {
      const int st = j & 1;
      if (!mbar_wait(&kv_full[st], (j >> 1) & 1, status)) return false;
      tc_fence_after();
      const uint32_t k_addr = smem_u32(smem + FA_OFF_K + st * FA_KV_BYTES);
      const uint32_t d_tmem = tmem + FA_TMEM_S + (uint32_t)st * 128;
#pragma unroll
      for (int ks = 0; ks < FA_D / 16; ++ks) {
        const uint32_t off = (uint32_t)(ks >> 2) * FA_HALF + (uint32_t)(ks & 3) * 32;
        umma_bf16(d_tmem, umma_desc_sw128(q_addr + off), umma_desc_sw128(k_addr + off), idesc_s, ks != 0);
      }
      umma_commit(&s_full[st]);
      any = true;
      return true;
    };
    if (ok && n_kt > 0) ok = issue_s(0);
    for (int j = 0; j < n_kt && ok; ++j) {
      if (j + 1 < n_kt && !(ok = issue_s(j + 1))) break;
      if (!(ok = mbar_wait(p_full, j & 1, status))) break;
      tc_fence_after();
      const int st = j & 1;
      const uint32_t v_addr = smem_u32(smem + FA_OFF_V + st * FA_KV_BYTES);
#pragma unroll
      for (int ks = 0; ks < FA_BN / 16; ++ks) {
        const uint32_t p_off = (uint32_t)(ks >> 2) * FA_HALF + (uint32_t)(ks & 3) * 32;
        umma_bf16(tmem + FA_TMEM_O, umma_desc_sw128(p_addr + p_off), umma_desc_sw128_mn(v_addr + ks * 2048, FA_HALF),
                  idesc_o, (j | ks) != 0);
      }
      umma_commit(&kv_empty[st]);
      umma_commit(o_done);
    }
    if (!ok && any) {
      umma_commit(drain);
      mbar_wait(drain, 0, status);
    }
  } else if (warp >= 2) {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                  // query row in the tile
    const int qpos = p0 + q0 + r;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint8_t* p_row = smem + FA_OFF_P + r * 128;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      const int st = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[st], (j >> 1) & 1, status)) && ok;
      tc_fence_after();
      float sv[128];
      if (ok) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float t[32];
          tmem_ld32(tmem + lane_off + FA_TMEM_S + (uint32_t)st * 128 + c * 32, t);
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[c * 32 + i] = t[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 128; ++i) sv[i] = 0.f;
      }
      const int kbase = j * FA_BN;
      // masked tiles: the last one or two of a causal row block
      if (kbase + FA_BN - 1 > p0 + q0) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (kbase + i > qpos) sv[i] = -INFINITY;
      }
      float mx = sv[0];
#pragma unroll
      for (int i = 1; i < 128; ++i) mx = fmaxf(mx, sv[i]);
      mx *= scale_log2;                       // scale > 0: max of the scaled scores
      float corr = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_used = mx;
      } else if (mx > m_used + FA_RESCALE) {
        corr = fast_exp2(m_used - mx);
        m_used = mx;
        rescale = true;
      }
      float rowsum = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float a = fast_exp2(fmaf(sv[2 * i], scale_log2, -m_used));
        const float c2 = fast_exp2(fmaf(sv[2 * i + 1], scale_log2, -m_used));
        rowsum += a + c2;
        pk[i] = pack2<T>(a, c2);
      }
      l = l * corr + rowsum;
      // P and O may be touched only once the previous P V product has finished
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, status)) && ok;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale) && ok) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float t[32];
          tmem_ld32(tmem + lane_off + FA_TMEM_O + c * 32, t);
#pragma unroll
          for (int i = 0; i < 32; ++i) t[i] *= corr;
          tmem_st32(tmem + lane_off + FA_TMEM_O + c * 32, t);
        }
        tmem_st_wait();
      }
      // P row: 16-byte chunk cc of 16 goes to block cc/8, swizzled position (cc%8) ^ (r%8)
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        uint4* dst = reinterpret_cast<uint4*>(p_row + (cc >> 3) * FA_HALF + (((cc & 7) ^ (r & 7)) << 4));
        *dst = make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // final: O / l to global memory
    if (n_kt > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(o_done, (n_kt - 1) & 1, status)) && ok;
      tc_fence_after();
    }
    const int qi = q0 + r;
    const float inv = 1.f / l;
    T* dst = o + ((size_t)b * S + (qi < S ? qi : 0)) * H * FA_D + (size_t)h * FA_D;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float t[32];
      if (ok) tmem_ld32(tmem + lane_off + FA_TMEM_O + c * 32, t);
      else {
#pragma unroll
        for (int i = 0; i < 32; ++i) t[i] = 0.f;
      }
      if (qi < S) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = pack2<T>(t[2 * i] * inv, t[2 * i + 1] * inv);
        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// [outer][rows][128] 16-bit -> 3-D map with boxes of 64 x 128 x 1, 128-byte swizzle.
int make_tmap_3d(CUtensorMap* map, const void* base, int64_t outer, int64_t rows, bool is_f16) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return LLAMA_ERR_CUDA;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  if (reinterpret_cast<uintptr_t>(base) & 15) return LLAMA_ERR_INVALID_ARG;
  cuuint64_t gdim[3] = {(cuuint64_t)FA_D, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t gstride[2] = {(cuuint64_t)FA_D * 2, (cuuint64_t)rows * FA_D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, is_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void*>(base), gdim, gstride, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LLAMA_OK : LLAMA_ERR_CUDA;
}

}  // namespace

template <typename T>
static int attention_prefill_tc_t(const void* q, const void* kc, const void* vc, void* o, const int32_t* pos0, int B,
                                  int S, int H, int Hk, int Smax, int* status, cudaStream_t st) {
  constexpr bool F16 = std::is_same<T, f16>::value;
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = make_tmap_3d(&tq, q, (int64_t)B * H, S, F16)) != LLAMA_OK) return rc;
  if ((rc = make_tmap_3d(&tk, kc, (int64_t)B * Hk, Smax, F16)) != LLAMA_OK) return rc;
  if ((rc = make_tmap_3d(&tv, vc, (int64_t)B * Hk, Smax, F16)) != LLAMA_OK) return rc;
  auto kern = attn_prefill_tc_kernel<T>;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, FA_SMEM) != cudaSuccess)
      return LLAMA_ERR_CUDA;
    attr = true;
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)FA_D);
  const cudaError_t err = launch_k(kern, dim3(((S + FA_BM - 1) / FA_BM) * H * B), dim3(192), FA_SMEM, st, tq, tk, tv,
                                   static_cast<T*>(o), pos0, S, H, Hk, scale_log2, status);
  return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int attention_prefill_tc(const void* q, const void* kc, const void* vc, void* o, const int32_t* pos0, int B, int S,
                         int H, int Hk, int Smax, int elt, int* status, cudaStream_t st) {
  if (elt == LLAMA_F16) return attention_prefill_tc_t<f16>(q, kc, vc, o, pos0, B, S, H, Hk, Smax, status, st);
  return attention_prefill_tc_t<bf16>(q, kc, vc, o, pos0, B, S, H, Hk, Smax, status, st);
}

}  // namespace llama
