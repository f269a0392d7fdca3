// Causal GQA prefill attention on the 5th-generation tensor cores (16-bit
// q/k/v, bf16 or fp16, head_dim 128).
//
// Three kernels share the arithmetic below: a per-tile one (one CTA per 128
// queries of one head), a persistent one (one CTA per SM looping over such
// items) and a persistent one whose items are the same 128 queries of two
// heads of one GQA group (each described above its definition).
//
// One CTA computes 128 queries of one head. Warp roles: warp 0 issues TMA
// loads (Q once, then K and V tiles of 128 keys into 2-stage rings), warp 1
// allocates TMEM and issues tcgen05.mma, warps 2-5 run the softmax: query row
// r (TMEM lane r) belongs to one thread of the warp that may read that lane
// quarter, which keeps the row's running maximum and sum in registers, so no
// value is exchanged between threads inside the key loop.
//
//   S_j = Q K_j^T      -> TMEM (two 128-column buffers, so S_{j+1} is computed
//                         while the softmax works on S_j)
//   P_j = exp2(S_j*c - m) rounded to the 16-bit type (the walkthrough rounds
//                         softmax(...) to 16 bits before the value product)
//                      -> TMEM (64 columns, two keys per column), the A
//                         operand of the next product
//   O  += P_j V_j      -> TMEM (128 columns); V is read MN-major straight from
//                         the cache layout [key][d].
//
// The running maximum m is only raised when a row's new maximum exceeds it by
// more than 8 (a factor 256 in exp2 space), so O in TMEM is rescaled rarely;
// O / l is exact for any m used consistently. Query i of the tile sits at
// absolute position pos0 + q0 + i and sees keys 0 .. pos0 + q0 + i.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>
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
constexpr int FA_OFF_BAR = FA_OFF_V + FA_STAGES * FA_KV_BYTES;
constexpr int FA_SMEM = FA_OFF_BAR + 256 + 1024;
constexpr uint32_t FA_TMEM_O = 0, FA_TMEM_S = 128;   // S buffers at columns 128 and 256
constexpr uint32_t FA_TMEM_P = 384;                   // P: 64 columns, keys 2c and 2c+1 in column c
constexpr float FA_RESCALE = 8.0f;                    // raise the running max only past +8 (log2)

// 2^x with the hardware approximation (flushes results below 2^-126 to zero,
// which only affects probabilities too small to matter in a 16-bit P).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Largest of three (one instruction on sm_100a).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Page j of sequence b (page 0 for an index outside the pool).
__device__ __forceinline__ int kv_page(const int32_t* table, int max_pages, int n_pages, int b, int j) {
  const int p = table[(size_t)b * max_pages + j];
  return (unsigned)p < (unsigned)n_pages ? p : 0;
}

__device__ __forceinline__ uint8_t* fa_align(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

constexpr int FA_THREADS = 192;

// The softmax of one 128-key tile for the query row this thread owns: the
// row's 128 scores of S buffer `s_tmem` (TMEM lane base in lane_off), keys
// past qpos masked on diagonal tiles (kbase = the tile's first key), the
// running maximum m_used raised only past +FA_RESCALE (first tile: set), the
// 64 packed probabilities in pk and the tile's row sum returned. corr is the
// factor O and l must be multiplied by (1 unless the maximum was raised).
template <typename T>
__device__ __forceinline__ float fa_tile_softmax(uint32_t s_tmem, bool ok, bool masked, int kbase, int qpos,
                                                 float scale_log2, bool first, float& m_used, float& corr,
                                                 uint32_t (&pk)[64]) {
  float sv[128];
  if (ok) {
    uint32_t u0[32], u1[32], u2[32], u3[32];
    tmem_ld32_nowait(s_tmem, u0);
    tmem_ld32_nowait(s_tmem + 32, u1);
    tmem_ld32_nowait(s_tmem + 64, u2);
    tmem_ld32_nowait(s_tmem + 96, u3);
    tmem_ld_wait();
#pragma unroll
    for (int x = 0; x < 32; ++x) {
      sv[x] = __uint_as_float(u0[x]);
      sv[32 + x] = __uint_as_float(u1[x]);
      sv[64 + x] = __uint_as_float(u2[x]);
      sv[96 + x] = __uint_as_float(u3[x]);
    }
  } else {
#pragma unroll
    for (int x = 0; x < 128; ++x) sv[x] = 0.f;
  }
  if (masked) {
#pragma unroll
    for (int x = 0; x < 128; ++x)
      if (kbase + x > qpos) sv[x] = -INFINITY;
  }
  float mx8[8];
#pragma unroll
  for (int x = 0; x < 8; ++x) mx8[x] = sv[x];
#pragma unroll
  for (int x = 8; x < 120; x += 16) {
#pragma unroll
    for (int c = 0; c < 8; ++c) mx8[c] = fmax3(mx8[c], sv[x + c], sv[x + 8 + c]);
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) mx8[c] = fmaxf(mx8[c], sv[120 + c]);
  const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])) *
                   scale_log2;
  corr = 1.f;
  if (first) {
    m_used = mx;
  } else if (mx > m_used + FA_RESCALE) {
    corr = fast_exp2(m_used - mx);
    m_used = mx;
  }
  float sum8[8];
#pragma unroll
  for (int x = 0; x < 8; ++x) sum8[x] = 0.f;
#pragma unroll
  for (int x = 0; x < 64; ++x) {
    const float a = fast_exp2(fmaf(sv[2 * x], scale_log2, -m_used));
    const float b = fast_exp2(fmaf(sv[2 * x + 1], scale_log2, -m_used));
    sum8[x & 7] += a + b;
    pk[x] = pack2<T>(a, b);
  }
  return ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
}

// O *= corr for this thread's row (all 128 columns).
__device__ __forceinline__ void fa_rescale_o(uint32_t o_tmem, float corr) {
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    float t[32];
    tmem_ld32(o_tmem + c * 32, t);
#pragma unroll
    for (int i = 0; i < 32; ++i) t[i] *= corr;
    tmem_st32(o_tmem + c * 32, t);
  }
  tmem_st_wait();
}

// P of this thread's row into the 64 P columns.
__device__ __forceinline__ void fa_store_p(uint32_t p_tmem, const uint32_t (&pk)[64]) {
  tmem_st32_u(p_tmem, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
  tmem_st32_u(p_tmem + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
  tmem_st_wait();
}

// O / l of this thread's row (128 columns) to dst, 16-byte stores.
template <typename T>
__device__ __forceinline__ void fa_store_o(uint32_t o_tmem, bool ok, float inv, T* dst, bool valid) {
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    float t[32];
    if (ok) tmem_ld32(o_tmem + c * 32, t);
    else {
#pragma unroll
      for (int i = 0; i < 32; ++i) t[i] = 0.f;
    }
    if (valid) {
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i] = pack2<T>(t[2 * i] * inv, t[2 * i + 1] * inv);
      uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(FA_THREADS, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, T* __restrict__ o,
                           const int32_t* __restrict__ pos0, int S, int H, int Hk, float scale_log2,
                           const int32_t* __restrict__ kv_table, int kv_max_pages, int kv_pages, int* status) {
  extern __shared__ uint8_t fa_smem_raw[];
  uint8_t* smem = fa_align(fa_smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + FA_OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;     // [2]
  uint64_t* k_empty = bars + 3;    // [2] released once S = Q K^T has read the tile
  uint64_t* v_full = bars + 5;     // [2]
  uint64_t* v_empty = bars + 7;    // [2] released once O += P V has read the tile
  uint64_t* s_full = bars + 9;     // [2]
  uint64_t* p_full = bars + 11;
  uint64_t* o_done = bars + 12;
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
    }
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
    // K and V have rings of their own: K tile j+2 can arrive as soon as
    // S_j has been computed, while V tile j+2 waits for P_j V_j.
    int k_issued = 0, v_issued = 0;
    bool ok = true;
    for (int j = 0; j < n_kt && ok; ++j) {
      const int st = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      if (!mbar_wait(&k_empty[st], ph ^ 1, status)) { ok = false; break; }
      // tile j: 128 keys of (b, g) at row j*128 of the contiguous cache, or
      // all 128 rows of page kv_table[b][j] of the paged one
      const int kv_y = kv_table ? 0 : j * FA_BN;
      const int kv_z = kv_table ? kv_page(kv_table, kv_max_pages, kv_pages, b, j) * Hk + g : b * Hk + g;
      mbar_arrive_expect_tx(&k_full[st], FA_KV_BYTES);
      uint8_t* kd = smem + FA_OFF_K + st * FA_KV_BYTES;
      tma_load_3d(kd, &tmK, &k_full[st], 0, kv_y, kv_z);
      tma_load_3d(kd + FA_HALF, &tmK, &k_full[st], 64, kv_y, kv_z);
      ++k_issued;
      if (!mbar_wait(&v_empty[st], ph ^ 1, status)) { ok = false; break; }
      mbar_arrive_expect_tx(&v_full[st], FA_KV_BYTES);
      uint8_t* vd = smem + FA_OFF_V + st * FA_KV_BYTES;
      tma_load_3d(vd, &tmV, &v_full[st], 0, kv_y, kv_z);
      tma_load_3d(vd + FA_HALF, &tmV, &v_full[st], 64, kv_y, kv_z);
      ++v_issued;
    }
    if (!ok) {  // let issued copies land before the CTA can exit
      mbar_wait(q_full, 0, status);
      for (int j = k_issued - 1; j >= 0 && j >= k_issued - 2; --j) mbar_wait(&k_full[j & 1], (j >> 1) & 1, status);
      for (int j = v_issued - 1; j >= 0 && j >= v_issued - 2; --j) mbar_wait(&v_full[j & 1], (j >> 1) & 1, status);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc_s = umma_idesc_16(UmmaFmt<T>::value, FA_BM, FA_BN, false);
    constexpr uint32_t idesc_o = umma_idesc_16(UmmaFmt<T>::value, FA_BM, FA_D, true);
    const uint32_t q_addr = smem_u32(smem + FA_OFF_Q);
    bool ok = mbar_wait(q_full, 0, status), any = false;
    auto issue_s = [&](int j) -> bool {
      const int st = j & 1;
      if (!mbar_wait(&k_full[st], (j >> 1) & 1, status)) return false;
      tc_fence_after();
      const uint32_t k_addr = smem_u32(smem + FA_OFF_K + st * FA_KV_BYTES);
      const uint32_t d_tmem = tmem + FA_TMEM_S + (uint32_t)st * 128;
#pragma unroll
      for (int ks = 0; ks < FA_D / 16; ++ks) {
        const uint32_t off = (uint32_t)(ks >> 2) * FA_HALF + (uint32_t)(ks & 3) * 32;
        umma_bf16(d_tmem, umma_desc_sw128(q_addr + off), umma_desc_sw128(k_addr + off), idesc_s, ks != 0);
      }
      umma_commit(&s_full[st]);
      umma_commit(&k_empty[st]);
      any = true;
      return true;
    };
    if (ok && n_kt > 0) ok = issue_s(0);
    for (int j = 0; j < n_kt && ok; ++j) {
      if (j + 1 < n_kt && !(ok = issue_s(j + 1))) break;
      if (!(ok = mbar_wait(p_full, j & 1, status))) break;
      const int st = j & 1;
      if (!(ok = mbar_wait(&v_full[st], (j >> 1) & 1, status))) break;
      tc_fence_after();
      const uint32_t v_addr = smem_u32(smem + FA_OFF_V + st * FA_KV_BYTES);
#pragma unroll
      for (int ks = 0; ks < FA_BN / 16; ++ks)   // 16 keys = 8 P columns per step
        umma_ts(tmem + FA_TMEM_O, tmem + FA_TMEM_P + ks * 8, umma_desc_sw128_mn(v_addr + ks * 2048, FA_HALF), idesc_o,
                (j | ks) != 0);
      umma_commit(&v_empty[st]);
      umma_commit(o_done);
    }
    if (!ok && any) {
      umma_commit(drain);
      mbar_wait(drain, 0, status);
    }
  } else if (warp >= 2) {
    const int quarter = warp & 3;                       // TMEM lanes this warp may read
    const int r = quarter * 32 + lane;                  // query row in the tile
    const int qpos = p0 + q0 + r;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      const int st = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[st], (j >> 1) & 1, status)) && ok;
      tc_fence_after();
      uint32_t pk[64];
      float corr;
      const float rowsum = fa_tile_softmax<T>(tmem + lane_off + FA_TMEM_S + (uint32_t)st * 128, ok,
                                              j * FA_BN + FA_BN - 1 > p0 + q0, j * FA_BN, qpos, scale_log2, j == 0,
                                              m_used, corr, pk);
      l = l * corr + rowsum;
      // P and O may be touched only once the previous P V product has finished
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, status)) && ok;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, corr != 1.f) && ok) fa_rescale_o(tmem + lane_off + FA_TMEM_O, corr);
      if (ok) fa_store_p(tmem + lane_off + FA_TMEM_P, pk);
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // final: O / l to global memory
    if (n_kt > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(o_done, (n_kt - 1) & 1, status)) && ok;
      tc_fence_after();
    }
    const int qi = q0 + r;
    T* dst = o + ((size_t)b * S + (qi < S ? qi : 0)) * H * FA_D + (size_t)h * FA_D;
    fa_store_o<T>(tmem + lane_off + FA_TMEM_O, ok, 1.f / l, dst, qi < S);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------ persistent
// The same computation with one CTA per SM looping over (query tile, head,
// sequence) items, so that the start of one item overlaps the end of the
// previous one: Q is double-buffered and loaded while the previous item runs,
// and the K/V rings, the S buffers and the P/O barriers run on across items.
// At the end of an item the softmax warps read O out of TMEM and store O / l;
// meanwhile the tensor cores already compute the next item's first S. The
// next item's first P V product needs that item's first P, which the same
// threads store only after reading O, so O is never overwritten early.
//
// Items are taken in the longest-first order of the per-tile kernel, dealt
// to the CTAs in a snake (round r goes to CTAs 0..G-1 for even r and G-1..0
// for odd r), which balances the decreasing causal lengths.
//
// Barrier phases are counted per CTA over all items: global tile t uses K/V
// and S stage t&1; item i uses Q buffer i&1. Every wait is bounded; after a
// failed wait a role stops waiting (and issuing) but walks its loops to the
// end.
constexpr int FP_THREADS = 192;
constexpr int kPersistentMaxS = 4096;
constexpr int FP_OFF_Q = 0;                                      // two Q buffers
constexpr int FP_OFF_K = FP_OFF_Q + 2 * FA_Q_BYTES;
constexpr int FP_OFF_V = FP_OFF_K + FA_STAGES * FA_KV_BYTES;
constexpr int FP_OFF_BAR = FP_OFF_V + FA_STAGES * FA_KV_BYTES;
constexpr int FP_SMEM = FP_OFF_BAR + 256 + 1024;

__device__ __forceinline__ int fp_item(int c, int G, int i) { return i * G + ((i & 1) ? G - 1 - c : c); }

struct FpItem {
  int b, h, g, q0, p0, n_kt;
};

__device__ __forceinline__ FpItem fp_decode(int w, int S, int H, int Hk, int B, const int32_t* pos0) {
  const int nqt = (S + FA_BM - 1) / FA_BM;
  const int HB = H * B;
  FpItem it;
  const int hb = w % HB;
  it.q0 = (nqt - 1 - w / HB) * FA_BM;
  it.h = hb % H;
  it.b = hb / H;
  it.g = it.h / (H / Hk);
  it.p0 = pos0 ? pos0[it.b] : 0;
  const int k_end = min(it.p0 + S, it.p0 + it.q0 + FA_BM);
  it.n_kt = (k_end + FA_BN - 1) / FA_BN;
  return it;
}

template <typename T>
__global__ void __launch_bounds__(FP_THREADS, 1)
    attn_prefill_tc_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                                      const __grid_constant__ CUtensorMap tmV, T* __restrict__ o,
                                      const int32_t* __restrict__ pos0, int B, int S, int H, int Hk, float scale_log2,
                                      const int32_t* __restrict__ kv_table, int kv_max_pages, int kv_pages,
                                      int* status) {
  extern __shared__ uint8_t fa_smem_raw[];
  uint8_t* smem = fa_align(fa_smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + FP_OFF_BAR);
  uint64_t* q_full = bars + 0;     // [2]
  uint64_t* q_empty = bars + 2;    // [2] released once the item's last S = Q K^T has read Q
  uint64_t* k_full = bars + 4;     // [2]
  uint64_t* k_empty = bars + 6;    // [2]
  uint64_t* v_full = bars + 8;     // [2]
  uint64_t* v_empty = bars + 10;   // [2]
  uint64_t* s_full = bars + 12;    // [2]
  uint64_t* p_full = bars + 14;    // softmax threads stored P (128 arrivals)
  uint64_t* o_done = bars + 15;    // O += P V finished
  uint64_t* drain = bars + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = ((S + FA_BM - 1) / FA_BM) * H * B;
  const int c = blockIdx.x, G = gridDim.x;

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1);
      mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
    }
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

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    int t = 0, q_issued = 0, k_issued = 0, v_issued = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int w = fp_item(c, G, i);
      if (w >= total) break;
      const FpItem it = fp_decode(w, S, H, Hk, B, pos0);
      const int qs = i & 1;
      if (!(ok = mbar_wait(&q_empty[qs], ((i >> 1) & 1) ^ 1, status))) break;
      mbar_arrive_expect_tx(&q_full[qs], FA_Q_BYTES);
      uint8_t* qd = smem + FP_OFF_Q + qs * FA_Q_BYTES;
      tma_load_3d(qd, &tmQ, &q_full[qs], 0, it.q0, it.b * H + it.h);
      tma_load_3d(qd + FA_HALF, &tmQ, &q_full[qs], 64, it.q0, it.b * H + it.h);
      ++q_issued;
      for (int j = 0; j < it.n_kt; ++j, ++t) {
        const int st = t & 1;
        const uint32_t ph = (t >> 1) & 1;
        if (!(ok = mbar_wait(&k_empty[st], ph ^ 1, status))) break;
        const int kv_y = kv_table ? 0 : j * FA_BN;
        const int kv_z = kv_table ? kv_page(kv_table, kv_max_pages, kv_pages, it.b, j) * Hk + it.g : it.b * Hk + it.g;
        mbar_arrive_expect_tx(&k_full[st], FA_KV_BYTES);
        uint8_t* kd = smem + FP_OFF_K + st * FA_KV_BYTES;
        tma_load_3d(kd, &tmK, &k_full[st], 0, kv_y, kv_z);
        tma_load_3d(kd + FA_HALF, &tmK, &k_full[st], 64, kv_y, kv_z);
        ++k_issued;
        if (!(ok = mbar_wait(&v_empty[st], ph ^ 1, status))) break;
        mbar_arrive_expect_tx(&v_full[st], FA_KV_BYTES);
        uint8_t* vd = smem + FP_OFF_V + st * FA_KV_BYTES;
        tma_load_3d(vd, &tmV, &v_full[st], 0, kv_y, kv_z);
        tma_load_3d(vd + FA_HALF, &tmV, &v_full[st], 64, kv_y, kv_z);
        ++v_issued;
      }
    }
    if (!ok) {  // let issued copies land before the CTA can exit
      for (int i = q_issued - 1; i >= 0 && i >= q_issued - 2; --i) mbar_wait(&q_full[i & 1], (i >> 1) & 1, status);
      for (int j = k_issued - 1; j >= 0 && j >= k_issued - 2; --j) mbar_wait(&k_full[j & 1], (j >> 1) & 1, status);
      for (int j = v_issued - 1; j >= 0 && j >= v_issued - 2; --j) mbar_wait(&v_full[j & 1], (j >> 1) & 1, status);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc_s = umma_idesc_16(UmmaFmt<T>::value, FA_BM, FA_BN, false);
    constexpr uint32_t idesc_o = umma_idesc_16(UmmaFmt<T>::value, FA_BM, FA_D, true);
    bool ok = true, any = false;
    auto issue_s = [&](int t, uint32_t q_addr) -> bool {
      const int st = t & 1;
      if (!mbar_wait(&k_full[st], (t >> 1) & 1, status)) return false;
      tc_fence_after();
      const uint32_t k_addr = smem_u32(smem + FP_OFF_K + st * FA_KV_BYTES);
      const uint32_t d_tmem = tmem + FA_TMEM_S + (uint32_t)st * 128;
#pragma unroll
      for (int ks = 0; ks < FA_D / 16; ++ks) {
        const uint32_t off = (uint32_t)(ks >> 2) * FA_HALF + (uint32_t)(ks & 3) * 32;
        umma_bf16(d_tmem, umma_desc_sw128(q_addr + off), umma_desc_sw128(k_addr + off), idesc_s, ks != 0);
      }
      umma_commit(&s_full[st]);
      umma_commit(&k_empty[st]);
      any = true;
      return true;
    };
    int t = 0;
    for (int i = 0; ok; ++i) {
      const int w = fp_item(c, G, i);
      if (w >= total) break;
      const int n_kt = fp_decode(w, S, H, Hk, B, pos0).n_kt;
      const int qs = i & 1;
      if (!(ok = mbar_wait(&q_full[qs], (i >> 1) & 1, status))) break;
      tc_fence_after();
      const uint32_t q_addr = smem_u32(smem + FP_OFF_Q + qs * FA_Q_BYTES);
      if (!(ok = issue_s(t, q_addr))) break;
      for (int j = 0; j < n_kt; ++j) {
        const int tj = t + j;
        if (j + 1 < n_kt) {
          if (!(ok = issue_s(tj + 1, q_addr))) break;
        } else {
          umma_commit(&q_empty[qs]);  // every S of this item is issued: Q is free once they finish
        }
        if (!(ok = mbar_wait(p_full, tj & 1, status))) break;
        const int st = tj & 1;
        if (!(ok = mbar_wait(&v_full[st], (tj >> 1) & 1, status))) break;
        // (the first product of an item overwrites O: the softmax threads read
        // the previous item's O out before they stored this item's first P)
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + FP_OFF_V + st * FA_KV_BYTES);
#pragma unroll
        for (int ks = 0; ks < FA_BN / 16; ++ks)
          umma_ts(tmem + FA_TMEM_O, tmem + FA_TMEM_P + ks * 8, umma_desc_sw128_mn(v_addr + ks * 2048, FA_HALF),
                  idesc_o, (j | ks) != 0);
        umma_commit(&v_empty[st]);
        umma_commit(o_done);
      }
      t += n_kt;
    }
    if (!ok && any) {
      umma_commit(drain);
      mbar_wait(drain, 0, status);
    }
  } else if (warp >= 2) {
    const int quarter = warp & 3;                       // TMEM lanes this warp may read
    const int r = quarter * 32 + lane;                  // query row in the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    int t = 0;
    for (int i = 0;; ++i) {
      const int w = fp_item(c, G, i);
      if (w >= total) break;
      const FpItem it = fp_decode(w, S, H, Hk, B, pos0);
      const int qpos = it.p0 + it.q0 + r;
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < it.n_kt; ++j, ++t) {
        const int st = t & 1;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&s_full[st], (t >> 1) & 1, status));
        tc_fence_after();
        uint32_t pk[64];
        float corr;
        const float rowsum = fa_tile_softmax<T>(tmem + lane_off + FA_TMEM_S + (uint32_t)st * 128, ok,
                                                j * FA_BN + FA_BN - 1 > it.p0 + it.q0, j * FA_BN, qpos, scale_log2,
                                                j == 0, m_used, corr, pk);
        l = l * corr + rowsum;
        // P (and O) may be touched only once the previous P V product has finished
        if (t > 0 && ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (t - 1) & 1, status));
        tc_fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f) && ok) fa_rescale_o(tmem + lane_off + FA_TMEM_O, corr);
        if (ok) fa_store_p(tmem + lane_off + FA_TMEM_P, pk);
        tc_fence_before();
        mbar_arrive(p_full);
      }
      // the item's last P V product, then O / l out of TMEM (the next item's
      // first P V product, which overwrites O, waits for this thread's next P)
      if (it.n_kt > 0 && ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (t - 1) & 1, status));
      tc_fence_after();
      const int qi = it.q0 + r;
      T* dst = o + ((size_t)it.b * S + (qi < S ? qi : 0)) * H * FA_D + (size_t)it.h * FA_D;
      fa_store_o<T>(tmem + lane_off + FA_TMEM_O, ok, 1.f / l, dst, qi < S);
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------- two heads per item
// The persistent computation on items of two query tiles: the same 128
// queries of two heads of one GQA group (h0 = 2p and h0 + 1, which read the
// same K and V). Every K and V tile loaded serves both tiles, and two softmax
// warpgroups work on different tiles (A: head h0, B: head h0 + 1), so one
// group's exponentials overlap the other's TMEM
// loads, maxima, stores and waits while the tensor pipe alternates between
// the two. Per key tile t the MMA issuer runs P_A(t) V(t), S_A(t+1),
// P_B(t) V(t), S_B(t+1) (S_A(t0), S_B(t0) at the start of an item).
//
// 384 threads in three warpgroups: warp 0 issues TMA loads, warp 1 the
// products (warps 2-3 idle); warps 4-7 run the softmax of tile A and warps
// 8-11 that of tile B (thread = query row = TMEM lane). The first warpgroup
// hands registers to the other two (setmaxnreg): it drops to FD_REGS_LOW and
// the softmax groups rise to FD_REGS_HIGH, 128 x 96 + 256 x 192 = 61440
// registers, what the launch holds at 160 per thread. The host launches the
// kernel only when its compiled register count is at least that (else the
// raise would wait for registers that never come) and runs the one-tile
// kernel otherwise.
//
// TMEM: O_A [0,128), O_B [128,256), S_A [256,384), S_B [384,512). A tile's P
// (64 columns, keys 2c and 2c+1 in column c) is written over the first half
// of its own S, which the softmax thread has read by then. S_X(t+1) overwrites
// P_X(t), so it is issued only once P_X(t) V(t) has completed (o_done[X]);
// this also makes O_X final up to tile t whenever the softmax sees S_X(t+1),
// so a rescale of O needs no wait. Q: one buffer per tile, reloaded once the
// item's last S of that tile has completed (q_empty[X]); K and V: 2-stage
// rings, released by commits after S_B(t) and P_B(t) V(t) (a commit covers
// every product issued before it, the A products included).
//
// Needs an even number of query heads per KV head; otherwise the one-tile
// persistent kernel runs.
constexpr int FD_THREADS = 384;
constexpr int FD_REGS_LOW = 96, FD_REGS_HIGH = 192;
static_assert(128 * FD_REGS_LOW + 256 * FD_REGS_HIGH <= FD_THREADS * 160, "register split exceeds the launch");
constexpr int FD_OFF_Q = 0;                                      // Q_A, Q_B
constexpr int FD_OFF_K = FD_OFF_Q + 2 * FA_Q_BYTES;
constexpr int FD_OFF_V = FD_OFF_K + FA_STAGES * FA_KV_BYTES;
constexpr int FD_OFF_BAR = FD_OFF_V + FA_STAGES * FA_KV_BYTES;
constexpr int FD_SMEM = FD_OFF_BAR + 256 + 1024;
constexpr uint32_t FD_TMEM_O = 0, FD_TMEM_S = 256;   // O_X at 128 X, S_X at 256 + 128 X

struct FdItem {
  int b, h0, g, q0, p0, n_kt;
};

// Item w in longest-first order: query tile (from the last), then head pair
// and sequence.
__device__ __forceinline__ FdItem fd_decode(int w, int S, int H, int Hk, int B, const int32_t* pos0) {
  const int nqt = (S + FA_BM - 1) / FA_BM;
  const int HP = (H / 2) * B;
  FdItem it;
  const int hb = w % HP;
  it.q0 = (nqt - 1 - w / HP) * FA_BM;
  it.h0 = 2 * (hb % (H / 2));
  it.b = hb / (H / 2);
  it.g = it.h0 / (H / Hk);
  it.p0 = pos0 ? pos0[it.b] : 0;
  const int k_end = min(it.p0 + S, it.p0 + it.q0 + FA_BM);
  it.n_kt = (k_end + FA_BN - 1) / FA_BN;
  return it;
}

// The dual kernel's barriers, in shared memory after the K and V rings.
struct FdBars {
  uint64_t *q_full, *q_empty, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_full, *o_done, *drain;
  __device__ explicit FdBars(uint8_t* smem) {
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + FD_OFF_BAR);
    q_full = bars + 0;     // [tile]
    q_empty = bars + 2;    // [tile] the item's last S of that tile has read Q
    k_full = bars + 4;     // [stage]
    k_empty = bars + 6;    // [stage] S_B (and the S_A before it) has read K
    v_full = bars + 8;     // [stage]
    v_empty = bars + 10;   // [stage] P_B V (and P_A V) has read V
    s_full = bars + 12;    // [tile]
    p_full = bars + 14;    // [tile] the tile's 128 softmax threads stored P
    o_done = bars + 16;    // [tile] P V of the tile finished
    drain = bars + 18;
  }
};

// Warps 0-3 of the dual kernel: warp 0 lane 0 issues the TMA loads, warp 1
// lane 0 the products.
template <typename T>
__device__ __forceinline__ void fd_loads_and_products(uint8_t* smem, uint32_t tmem, int warp, int lane,
                                                      const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                                      const CUtensorMap& tmV, const int32_t* __restrict__ pos0,
                                                      int B, int S, int H, int Hk,
                                                      const int32_t* __restrict__ kv_table, int kv_max_pages,
                                                      int kv_pages, int* status) {
  FdBars fb(smem);
  uint64_t *q_full = fb.q_full, *q_empty = fb.q_empty, *k_full = fb.k_full, *k_empty = fb.k_empty;
  uint64_t *v_full = fb.v_full, *v_empty = fb.v_empty, *s_full = fb.s_full, *p_full = fb.p_full;
  uint64_t *o_done = fb.o_done, *drain = fb.drain;
  const int total = ((S + FA_BM - 1) / FA_BM) * (H / 2) * B;
  const int c = blockIdx.x, G = gridDim.x;
  if (warp == 0 && lane == 0) {

    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    int t = 0, qa_issued = 0, qb_issued = 0, k_issued = 0, v_issued = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int w = fp_item(c, G, i);
      if (w >= total) break;
      const FdItem it = fd_decode(w, S, H, Hk, B, pos0);
      for (int j = 0; j < it.n_kt; ++j, ++t) {
        const int st = t & 1;
        const uint32_t ph = (t >> 1) & 1;
        if (!(ok = mbar_wait(&k_empty[st], ph ^ 1, status))) break;
        const int kv_y = kv_table ? 0 : j * FA_BN;
        const int kv_z = kv_table ? kv_page(kv_table, kv_max_pages, kv_pages, it.b, j) * Hk + it.g : it.b * Hk + it.g;
        mbar_arrive_expect_tx(&k_full[st], FA_KV_BYTES);
        uint8_t* kd = smem + FD_OFF_K + st * FA_KV_BYTES;
        tma_load_3d(kd, &tmK, &k_full[st], 0, kv_y, kv_z);
        tma_load_3d(kd + FA_HALF, &tmK, &k_full[st], 64, kv_y, kv_z);
        ++k_issued;
        if (j == 0) {   // the item's Q tiles, after its first K (which does not wait for the last item's S)
          for (int x = 0; x < 2 && ok; ++x) {
            if (!(ok = mbar_wait(&q_empty[x], (i & 1) ^ 1, status))) break;
            mbar_arrive_expect_tx(&q_full[x], FA_Q_BYTES);
            uint8_t* qd = smem + FD_OFF_Q + x * FA_Q_BYTES;
            tma_load_3d(qd, &tmQ, &q_full[x], 0, it.q0, it.b * H + it.h0 + x);
            tma_load_3d(qd + FA_HALF, &tmQ, &q_full[x], 64, it.q0, it.b * H + it.h0 + x);
            ++(x ? qb_issued : qa_issued);
          }
          if (!ok) break;
        }
        if (!(ok = mbar_wait(&v_empty[st], ph ^ 1, status))) break;
        mbar_arrive_expect_tx(&v_full[st], FA_KV_BYTES);
        uint8_t* vd = smem + FD_OFF_V + st * FA_KV_BYTES;
        tma_load_3d(vd, &tmV, &v_full[st], 0, kv_y, kv_z);
        tma_load_3d(vd + FA_HALF, &tmV, &v_full[st], 64, kv_y, kv_z);
        ++v_issued;
      }
    }
    if (!ok) {  // let issued copies land before the CTA can exit
      if (qa_issued > 0) mbar_wait(&q_full[0], (qa_issued - 1) & 1, status);
      if (qb_issued > 0) mbar_wait(&q_full[1], (qb_issued - 1) & 1, status);
      for (int j = k_issued - 1; j >= 0 && j >= k_issued - 2; --j) mbar_wait(&k_full[j & 1], (j >> 1) & 1, status);
      for (int j = v_issued - 1; j >= 0 && j >= v_issued - 2; --j) mbar_wait(&v_full[j & 1], (j >> 1) & 1, status);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc_s = umma_idesc_16(UmmaFmt<T>::value, FA_BM, FA_BN, false);
    constexpr uint32_t idesc_o = umma_idesc_16(UmmaFmt<T>::value, FA_BM, FA_D, true);
    bool any = false;
    // S_x(t) = Q_x K(t)^T over P_x(t-1), once P_x(t-1) V(t-1) has completed;
    // `last`: the item's last S of tile x, after which Q_x may be reloaded
    auto issue_s = [&](int x, int t, bool last) -> bool {
      const int st = t & 1;
      if (t > 0 && !mbar_wait(&o_done[x], (t - 1) & 1, status)) return false;
      if (x == 0 && !mbar_wait(&k_full[st], (t >> 1) & 1, status)) return false;
      tc_fence_after();
      const uint32_t q_addr = smem_u32(smem + FD_OFF_Q + x * FA_Q_BYTES);
      const uint32_t k_addr = smem_u32(smem + FD_OFF_K + st * FA_KV_BYTES);
      const uint32_t d_tmem = tmem + FD_TMEM_S + (uint32_t)x * 128;
#pragma unroll
      for (int ks = 0; ks < FA_D / 16; ++ks) {
        const uint32_t off = (uint32_t)(ks >> 2) * FA_HALF + (uint32_t)(ks & 3) * 32;
        umma_bf16(d_tmem, umma_desc_sw128(q_addr + off), umma_desc_sw128(k_addr + off), idesc_s, ks != 0);
      }
      umma_commit(&s_full[x]);
      if (x == 1) umma_commit(&k_empty[st]);
      if (last) umma_commit(&q_empty[x]);
      any = true;
      return true;
    };
    // O_x (+)= P_x(t) V(t); j == 0 starts the item's O
    auto issue_pv = [&](int x, int t, int j) -> bool {
      const int st = t & 1;
      if (!mbar_wait(&p_full[x], t & 1, status)) return false;
      if (x == 0 && !mbar_wait(&v_full[st], (t >> 1) & 1, status)) return false;
      tc_fence_after();
      const uint32_t v_addr = smem_u32(smem + FD_OFF_V + st * FA_KV_BYTES);
      const uint32_t p_tmem = tmem + FD_TMEM_S + (uint32_t)x * 128;
#pragma unroll
      for (int ks = 0; ks < FA_BN / 16; ++ks)
        umma_ts(tmem + FD_TMEM_O + (uint32_t)x * 128, p_tmem + ks * 8,
                umma_desc_sw128_mn(v_addr + ks * 2048, FA_HALF), idesc_o, (j | ks) != 0);
      if (x == 1) umma_commit(&v_empty[st]);
      umma_commit(&o_done[x]);
      return true;
    };
    bool ok = true;
    int t = 0;
    for (int i = 0; ok; ++i) {
      const int w = fp_item(c, G, i);
      if (w >= total) break;
      const int n_kt = fd_decode(w, S, H, Hk, B, pos0).n_kt;
      for (int x = 0; x < 2 && ok; ++x) ok = mbar_wait(&q_full[x], i & 1, status);
      if (!ok || !(ok = issue_s(0, t, n_kt == 1)) || !(ok = issue_s(1, t, n_kt == 1))) break;
      for (int j = 0; j < n_kt && ok; ++j) {
        const int tj = t + j;
        const bool more = j + 1 < n_kt, last_next = j + 2 == n_kt;
        ok = issue_pv(0, tj, j) && (!more || issue_s(0, tj + 1, last_next)) && issue_pv(1, tj, j) &&
             (!more || issue_s(1, tj + 1, last_next));
      }
      t += n_kt;
    }
    if (!ok && any) {
      umma_commit(drain);
      mbar_wait(drain, 0, status);
    }
  }
}

// Warps 4-11 of the dual kernel: the softmax of tile A (warps 4-7) or B (8-11).
template <typename T>
__device__ __forceinline__ void fd_softmax(uint8_t* smem, uint32_t tmem, int warp, int lane, T* __restrict__ o,
                                           const int32_t* __restrict__ pos0, int B, int S, int H, int Hk,
                                           float scale_log2, int* status) {
  const FdBars fb(smem);
  uint64_t *s_full = fb.s_full, *p_full = fb.p_full, *o_done = fb.o_done;
  const int total = ((S + FA_BM - 1) / FA_BM) * (H / 2) * B;
  const int c = blockIdx.x, G = gridDim.x;
  {
    const int x = (warp - 4) >> 2;                      // 0: tile A (head h0), 1: tile B (head h0 + 1)
    const int quarter = warp & 3;                       // TMEM lanes this warp may read
    const int r = quarter * 32 + lane;                  // query row in the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_tm = tmem + lane_off + FD_TMEM_S + (uint32_t)x * 128;
    const uint32_t o_tm = tmem + lane_off + FD_TMEM_O + (uint32_t)x * 128;
    bool ok = true;
    int t = 0;
    for (int i = 0;; ++i) {
      const int w = fp_item(c, G, i);
      if (w >= total) break;
      const FdItem it = fd_decode(w, S, H, Hk, B, pos0);
      const int qpos = it.p0 + it.q0 + r;
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < it.n_kt; ++j, ++t) {
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&s_full[x], t & 1, status));
        tc_fence_after();
        uint32_t pk[64];
        float corr;
        const float rowsum = fa_tile_softmax<T>(s_tm, ok, j * FA_BN + FA_BN - 1 > it.p0 + it.q0, j * FA_BN, qpos,
                                                scale_log2, j == 0, m_used, corr, pk);
        l = l * corr + rowsum;
        // O_x is final up to tile t-1: S_x(t) was issued after P_x(t-1) V(t-1) completed
        if (__any_sync(0xffffffffu, corr != 1.f) && ok) fa_rescale_o(o_tm, corr);
        if (ok) fa_store_p(s_tm, pk);
        tc_fence_before();
        mbar_arrive(&p_full[x]);
      }
      // the item's last product, then O / l out of TMEM (the next item's first
      // product, which overwrites O, waits for this thread's next P)
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_done[x], (t - 1) & 1, status));
      tc_fence_after();
      const int qi = it.q0 + r;
      T* dst = o + ((size_t)it.b * S + (qi < S ? qi : 0)) * H * FA_D + (size_t)(it.h0 + x) * FA_D;
      fa_store_o<T>(o_tm, ok, 1.f / l, dst, qi < S);
      tc_fence_before();
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(FD_THREADS, 1)
    attn_prefill_tc_dual_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                                const __grid_constant__ CUtensorMap tmV, T* __restrict__ o,
                                const int32_t* __restrict__ pos0, int B, int S, int H, int Hk, float scale_log2,
                                const int32_t* __restrict__ kv_table, int kv_max_pages, int kv_pages, int* status) {
  extern __shared__ uint8_t fa_smem_raw[];
  uint8_t* smem = fa_align(fa_smem_raw);
  const FdBars fb(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fb.drain + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&fb.q_full[i], 1); mbar_init(&fb.q_empty[i], 1);
      mbar_init(&fb.k_full[i], 1); mbar_init(&fb.k_empty[i], 1);
      mbar_init(&fb.v_full[i], 1); mbar_init(&fb.v_empty[i], 1);
      mbar_init(&fb.s_full[i], 1);
      mbar_init(&fb.p_full[i], 128);
      mbar_init(&fb.o_done[i], 1);
    }
    mbar_init(fb.drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(FD_REGS_LOW) : "memory");
    fd_loads_and_products<T>(smem, tmem, warp, lane, tmQ, tmK, tmV, pos0, B, S, H, Hk, kv_table, kv_max_pages,
                             kv_pages, status);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(FD_REGS_HIGH) : "memory");
    fd_softmax<T>(smem, tmem, warp, lane, o, pos0, B, S, H, Hk, scale_log2, status);
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
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  if (!fn) return LLAMA_ERR_CUDA;
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

// The dual kernel's register hand-off fits the registers its launch holds
// (compiled count x threads); checked once per instantiation.
template <typename T>
bool dual_regs_ok() {
  static std::once_flag once;
  static bool ok = false;
  std::call_once(once, [] {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(attn_prefill_tc_dual_kernel<T>)) == cudaSuccess)
      ok = fa.numRegs * FD_THREADS >= 128 * FD_REGS_LOW + 256 * FD_REGS_HIGH;
    else
      cudaGetLastError();
  });
  return ok;
}

template <typename T>
static int attention_prefill_tc_t(const void* q, const void* kc, const void* vc, void* o, const int32_t* pos0, int B,
                                  int S, int H, int Hk, int Smax, int* status, cudaStream_t st,
                                  const int32_t* kv_table, int kv_max_pages, int kv_pages) {
  constexpr bool F16 = std::is_same<T, f16>::value;
  CUtensorMap tq, tk, tv;
  int rc;
  // contiguous: [B*Hk][Smax][128]; paged: [kv_pages*Hk][128][128]
  const int64_t kv_outer = kv_table ? (int64_t)kv_pages * Hk : (int64_t)B * Hk;
  const int64_t kv_rows = kv_table ? KV_PAGE : Smax;
  if (kv_table && (kv_pages <= 0 || kv_max_pages <= 0)) return LLAMA_ERR_INVALID_ARG;
  if ((rc = make_tmap_3d(&tq, q, (int64_t)B * H, S, F16)) != LLAMA_OK) return rc;
  if ((rc = make_tmap_3d(&tk, kc, kv_outer, kv_rows, F16)) != LLAMA_OK) return rc;
  if ((rc = make_tmap_3d(&tv, vc, kv_outer, kv_rows, F16)) != LLAMA_OK) return rc;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)FA_D);
  // Two heads per item (the dual kernel) wherever the heads of a GQA group
  // pair up: measured 11-18% faster than the one-head persistent kernel at
  // 2048 queries (B = 1, 4, 16) and 12-14% faster than the per-tile kernel at
  // 8192 and 32768. Otherwise short chunks (few key tiles per item) run the
  // one-head persistent kernel, which hides each item's start and end behind
  // its neighbours (10% faster than the per-tile kernel at 2048 queries, 6-8%
  // slower at 32768). LLAMA_ATTN_NO_DUAL and LLAMA_ATTN_PER_TILE select the
  // other kernels, for comparisons.
  static const bool per_tile = getenv("LLAMA_ATTN_PER_TILE") != nullptr;
  static const bool no_dual = getenv("LLAMA_ATTN_NO_DUAL") != nullptr;
  if (!no_dual && !per_tile && (H / Hk) % 2 == 0 && dual_regs_ok<T>()) {
    auto kern = attn_prefill_tc_dual_kernel<T>;
    if (const int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), FD_SMEM)) return rc;
    const long long items = (long long)((S + FA_BM - 1) / FA_BM) * (H / 2) * B;
    const int grid = (int)std::min<long long>(items, num_sms());
    const cudaError_t err = launch_k(kern, dim3(grid), dim3(FD_THREADS), FD_SMEM, st, tq, tk, tv, static_cast<T*>(o),
                                     pos0, B, S, H, Hk, scale_log2, kv_table, kv_max_pages, kv_pages, status);
    return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
  }
  if (!per_tile && S <= kPersistentMaxS) {
    auto kern = attn_prefill_tc_persistent_kernel<T>;
    if (const int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), FP_SMEM)) return rc;
    const long long items = (long long)((S + FA_BM - 1) / FA_BM) * H * B;
    const int grid = (int)std::min<long long>(items, num_sms());
    const cudaError_t err = launch_k(kern, dim3(grid), dim3(FP_THREADS), FP_SMEM, st, tq, tk, tv, static_cast<T*>(o),
                                     pos0, B, S, H, Hk, scale_log2, kv_table, kv_max_pages, kv_pages, status);
    return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
  }
  auto kern = attn_prefill_tc_kernel<T>;
  if (const int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), FA_SMEM)) return rc;
  const cudaError_t err = launch_k(kern, dim3(((S + FA_BM - 1) / FA_BM) * H * B), dim3(FA_THREADS), FA_SMEM, st, tq,
                                   tk, tv,
                                   static_cast<T*>(o), pos0, S, H, Hk, scale_log2, kv_table, kv_max_pages, kv_pages,
                                   status);
  return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int attention_prefill_tc(const void* q, const void* kc, const void* vc, void* o, const int32_t* pos0, int B, int S,
                         int H, int Hk, int Smax, int elt, int* status, cudaStream_t st, const int32_t* kv_table,
                         int kv_max_pages, int kv_pages) {
  if (elt == LLAMA_F16)
    return attention_prefill_tc_t<f16>(q, kc, vc, o, pos0, B, S, H, Hk, Smax, status, st, kv_table, kv_max_pages,
                                       kv_pages);
  return attention_prefill_tc_t<bf16>(q, kc, vc, o, pos0, B, S, H, Hk, Smax, status, st, kv_table, kv_max_pages,
                                      kv_pages);
}

}  // namespace llama
