// tcgen05 GEMMs for the 16-bit projections: acc = x W^T with x [M,K], W [N,K]
// (bf16 or fp16 operands, fp32 accumulation).
//
// Three kernels share the same warp roles (warp 0: TMA producer, warp 1: MMA
// issuer and TMEM owner, warps 2-5: epilogue reading TMEM):
//
//  * gemm_pair (M large, at least one wave of tiles: prefill): clusters of two
//    SMs, 256x256 output tiles; each CTA loads its 128 rows of x and its 128
//    rows of W, the leader issues tcgen05.mma.cta_group::2 (M=256, N=256) and
//    each CTA drains its 128 rows of the accumulator.
//  * gemm_wide (M large, fewer tiles than SMs): persistent, one CTA per SM,
//    128x256 output tiles, split stream-K over all SMs with an owner fixup.
//    Both keep double-buffered fp32 accumulators in TMEM (2 x 256 columns) so
//    the epilogue of one tile overlaps the main loop of the next.
//  * gemm_skinny (M <= 256, decode and short prompts): the weight tile is the
//    MMA's A operand (128 weight rows) and the tokens are its N side, so a
//    decode step streams each weight byte exactly once at full MMA width.
//    Persistent stream-K: every CTA streams an equal share of (tile, k-block)
//    units; a split tile is finished by the CTA holding its k-block 0, which
//    waits (bounded) for the other shares and sums them in CTA order, except
//    for the residual epilogue, where each share is added into x atomically.
//
// All are launched with programmatic dependent launch: weight tiles are
// requested before waiting for the previous kernel, activations after.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <cstdlib>
#include <mutex>
#include <type_traits>

#include "device_cache.h"
#include "epilogue.cuh"
#include "kernels.h"

namespace llama {

namespace {

constexpr int BK = 64;                    // K elements per stage (128 B rows, 128B swizzle)
constexpr int W_BM = 128, W_BN = 256;     // wide tile
constexpr int W_STAGES = 4;
constexpr int W_A_BYTES = W_BM * BK * 2;  // 16 KB
constexpr int W_B_BYTES = W_BN * BK * 2;  // 32 KB
constexpr int W_STAGE_BYTES = W_A_BYTES + W_B_BYTES;
constexpr int W_SMEM = W_STAGES * W_STAGE_BYTES + 1024 + 256;
constexpr int kThreads = 192;

constexpr int S_BM = 128;                 // skinny: weight rows per CTA
constexpr int S_A_BYTES = S_BM * BK * 2;  // 16 KB

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Wait for the loads this producer issued last (ring positions before
// (stage, phase)); used only on the error path so no copy is in flight when
// the CTA exits.
__device__ void drain_loads(uint64_t* full, int stage, uint32_t phase, int issued, int nstages, int* status) {
  for (int i = 0; i < issued && i < nstages; ++i) {
    if (--stage < 0) { stage = nstages - 1; phase ^= 1; }
    mbar_wait(&full[stage], phase, status);
  }
}

// ------------------------------------------------------------------ wide
__device__ __forceinline__ long long sk_first(long long c, long long U, long long G) { return U * c / G; }
__device__ __forceinline__ long long sk_owner(long long u, long long U, long long G) { return ((u + 1) * G - 1) / U; }

// The pieces of work of one wide-GEMM CTA, in order: whole tiles c, c+G, ...
// below T_dp (data-parallel waves), then its share of the stream-K region.
// The stream-K region is the tiles [T_dp, T) cut into (tile, k-block) units,
// tile-major; CTA c < G_sk takes units [U*c/G_sk, U*(c+1)/G_sk). Every role of
// the CTA walks the same sequence.
struct WideWork {
  int c, G, kb, T_dp, i, dp_n;
  long long u, u1, u_start;
  __device__ WideWork(int c_, int G_, int kb_, int T, int T_dp_, int G_sk) : c(c_), G(G_), kb(kb_), T_dp(T_dp_), i(0) {
    dp_n = T_dp > c ? (T_dp - c + G - 1) / G : 0;
    const long long U = (long long)(T - T_dp) * kb;
    u = u1 = 0;
    if (c < G_sk) { u = sk_first(c, U, G_sk); u1 = sk_first(c + 1, U, G_sk); }
    u_start = u;
  }
  // tile index, first k-block and number of k-blocks of the next piece; slot
  // is 0 for the CTA's first stream-K piece and 1 for any later one
  __device__ bool next(int& tile, int& klo, int& n, int& slot) {
    if (i < dp_n) { tile = c + i * G; klo = 0; n = kb; slot = 0; ++i; return true; }
    if (u < u1) {
      tile = T_dp + (int)(u / kb);
      klo = (int)(u % kb);
      n = (int)((u1 - u) < (kb - klo) ? (u1 - u) : (kb - klo));
      slot = u == u_start ? 0 : 1;
      u += n;
      return true;
    }
    return false;
  }
  __device__ bool next(int& tile, int& klo, int& n) {
    int slot;
    return next(tile, klo, n, slot);
  }
};

// A piece that covers its whole tile runs the epilogue from TMEM. A split
// tile has one owner, the CTA whose piece holds k-block 0: that piece is the
// last of the owner's range, while every other piece of the tile is the first
// of its CTA's range (it starts inside the tile), so the other contributors
// finish their share early. They store it in their CTA's workspace slot and
// count themselves in the tile's counter; the owner waits (bounded) for the
// count, adds the shares in CTA order to its own accumulator from TMEM, runs
// the epilogue and re-arms the counter. The sum order is fixed, so results do
// not depend on timing. Every CTA of the grid is resident at once (one CTA per
// SM, grid <= SMs), and an owner only waits for first pieces, which wait for
// nothing, so the waits always end.
//
// Workspace slot layout: float4 (c * 8 + j) * 128 + r holds columns
// 32c + 4j .. 32c + 4j + 3 of tile row r, so a warp's 32 rows are 512
// contiguous bytes.
template <int KIND, typename T>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_wide_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                     int K, EpiArgs epi, int T_dp, int G_sk, float* __restrict__ ws, int* __restrict__ counters,
                     int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + W_STAGES * W_STAGE_BYTES);
  uint64_t* empty = full + W_STAGES;
  uint64_t* accf = empty + W_STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (M + W_BM - 1) / W_BM, n_tiles = (N + W_BN - 1) / W_BN;
  const int tiles = m_tiles * n_tiles;
  const int kb = (K + BK - 1) / BK;

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < W_STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&accf[a], 1); mbar_init(&acce[a], 128); }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WideWork work(blockIdx.x, gridDim.x, kb, tiles, T_dp, G_sk);
  int tile, klo, n;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    const uint64_t pol_a = l2_policy_evict_last(), pol_b = l2_policy_evict_last();
    // The weight tiles of the first stages do not depend on the previous
    // kernel: request them before waiting for it, their activation halves after.
    bool have = work.next(tile, klo, n);
    const int pre = have ? (n < W_STAGES ? n : W_STAGES) : 0;
    {
      const int n0 = have ? (tile / m_tiles) * W_BN : 0;
      for (int k = 0; k < pre; ++k) {
        mbar_arrive_expect_tx(&full[k], W_STAGE_BYTES);
        tma_load_2d(smem + k * W_STAGE_BYTES + W_A_BYTES, &tmB, &full[k], (klo + k) * BK, n0, pol_b);
      }
      pdl_wait();
      const int m0 = have ? (tile % m_tiles) * W_BM : 0;
      for (int k = 0; k < pre; ++k) tma_load_2d(smem + k * W_STAGE_BYTES, &tmA, &full[k], (klo + k) * BK, m0, pol_a);
    }
    int stage = pre % W_STAGES, issued = pre, k_start = pre;
    uint32_t phase = pre == W_STAGES ? 1u : 0u;
    bool ok = true;
    for (; have && ok; have = work.next(tile, klo, n), k_start = 0) {
      const int m0 = (tile % m_tiles) * W_BM, n0 = (tile / m_tiles) * W_BN;
      for (int k = k_start; k < n; ++k) {
        if (!mbar_wait(&empty[stage], phase ^ 1, status)) { ok = false; break; }
        uint8_t* sa = smem + stage * W_STAGE_BYTES;
        mbar_arrive_expect_tx(&full[stage], W_STAGE_BYTES);
        tma_load_2d(sa, &tmA, &full[stage], (klo + k) * BK, m0, pol_a);
        tma_load_2d(sa + W_A_BYTES, &tmB, &full[stage], (klo + k) * BK, n0, pol_b);
        ++issued;
        if (++stage == W_STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok) drain_loads(full, stage, phase, issued, W_STAGES, status);
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = umma_idesc_16(UmmaFmt<T>::value, W_BM, W_BN);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true, any = false;
    while (ok && work.next(tile, klo, n)) {
      if (!mbar_wait(&acce[acc], acc_phase ^ 1, status)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem + acc * W_BN;
      for (int k = 0; k < n; ++k) {
        if (!mbar_wait(&full[stage], phase, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + stage * W_STAGE_BYTES);
        const uint32_t b_addr = a_addr + W_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_bf16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32), idesc,
                    (k | kk) != 0);
        umma_commit(&empty[stage]);
        any = true;
        if (++stage == W_STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      umma_commit(&accf[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (!ok && any) {  // let issued MMAs finish before TMEM is released
      umma_commit(drain);
      mbar_wait(drain, 0, status);
    }
  } else if (warp >= 2) {
    pdl_wait();  // the epilogue reads and writes memory owned by earlier kernels
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const long long U = (long long)(tiles - T_dp) * kb;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool failed = false;  // after a timed-out wait the MMA has stopped: no further waits
    while (work.next(tile, klo, n)) {
      const int m0 = (tile % m_tiles) * W_BM, n0 = (tile / m_tiles) * W_BN;
      const bool whole = klo == 0 && n == kb;
      const int s = tile - T_dp;  // stream-K tile index (split tiles only)
      // contributors other than the owner: CTAs (c_own, c_hi], each one slot
      long long c_own = 0, c_hi = 0;
      if (!whole) {
        const long long t0 = (long long)s * kb;
        c_own = sk_owner(t0, U, G_sk);
        c_hi = sk_owner(t0 + kb - 1, U, G_sk);
      }
      if (!whole && klo == 0) {  // owner: wait for the other shares before touching TMEM
        if (threadIdx.x == 64) {
          const int need = (int)(c_hi - c_own);
          counter_wait_geq(&counters[s], need, status);  // a timeout is latched in status
          counters[s] = 0;  // every other contributor has counted itself: re-arm
        }
        named_bar_sync(1, 128);
        __threadfence();
      }
      // the whole warp decides together so the warp-wide TMEM loads stay converged
      if (!failed) failed = !__all_sync(0xffffffffu, mbar_wait(&accf[acc], acc_phase, status));
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + acc * W_BN;
      float4* mine = reinterpret_cast<float4*>(ws) + (size_t)blockIdx.x * (W_BM * W_BN / 4) + row;
      const float rs = (KIND == EPI_QKV_ROPE || KIND == EPI_SWIGLU) && epi.ss_in && klo == 0 && m0 + row < M
                           ? norm_row_scale(epi, m0 + row) : 1.f;
      float ssq = 0.f;
#pragma unroll 1
      for (int c = 0; c < W_BN / 32; ++c) {
        float v[32];
        if (failed) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        } else {
          tmem_ld32(base + c * 32, v);
        }
        if (whole) {
          if (!failed && n0 + c * 32 < N) ssq += epi_row32<KIND, T>(epi, m0 + row, n0 + c * 32, v, rs);
        } else if (klo != 0) {  // a share for the owner
#pragma unroll
          for (int j = 0; j < 8; ++j)
            __stcg(mine + (c * 8 + j) * W_BM, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        } else {  // owner: add the shares in CTA order, then the epilogue
          for (long long cc = c_own + 1; cc <= c_hi; ++cc) {
            const float4* p4 = reinterpret_cast<const float4*>(ws) + (size_t)cc * (W_BM * W_BN / 4) + row;
            float4 x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = __ldcg(p4 + (c * 8 + j) * W_BM);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              v[4 * j] += x[j].x; v[4 * j + 1] += x[j].y; v[4 * j + 2] += x[j].z; v[4 * j + 3] += x[j].w;
            }
          }
          if (!failed && n0 + c * 32 < N) ssq += epi_row32<KIND, T>(epi, m0 + row, n0 + c * 32, v, rs);
        }
      }
      if (KIND == EPI_RESIDUAL && epi.ss_out && klo == 0 && m0 + row < M)
        epi.ss_out[(size_t)(m0 + row) * epi.ss_n + n0 / W_BN] = ssq;
      tc_fence_before();
      mbar_arrive(&acce[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      if (!whole && klo != 0) {  // publish the share
        __threadfence();
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) atomicAdd(&counters[s], 1);
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

// ------------------------------------------------------------- wide, pair
// The same product on CTA pairs (clusters of 2 SMs): a pair owns a 256x256
// output tile; each CTA loads its 128 rows of A and its 128 rows of W (half
// of the tile's columns) per 64-wide k-block, and the leader CTA (rank 0)
// issues tcgen05.mma.cta_group::2 (M=256, N=256), which reads the operands
// from both CTAs' shared memory and leaves rows 0-127 of the tile in the
// leader's TMEM and rows 128-255 in the peer's. Each SM thus moves 32 KB per
// k-block instead of 48 KB for the same flops. Barriers: the TMA loads of
// both CTAs count their bytes on the leader's `full` barrier; the leader's
// commits arrive on `empty` and `accf` in both CTAs; both CTAs' epilogue
// threads arrive on the leader's `acce`.
constexpr int P_BM = 128, P_BN = 256;                 // rows per CTA, columns per pair tile
constexpr int P_A_BYTES = P_BM * BK * 2;              // 16 KB
constexpr int P_B_BYTES = (P_BN / 2) * BK * 2;        // 16 KB (this CTA's half of the columns)
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;
constexpr int P_STAGES = 6;
constexpr int P_SMEM = P_STAGES * P_STAGE_BYTES + 1024 + 256;

// Tile t of the pair grid as (256-row block m, 256-column block n): groups of
// G row blocks, each group taken column by column with its row blocks
// innermost (G = m_tiles is plain column-major order).
__device__ __forceinline__ void pair_tile(int t, int m_tiles, int G, int& m, int& n, int n_tiles) {
  const int per = G * n_tiles;
  const int g = t / per;
  const int r = t - g * per;
  const int m0 = g * G;
  const int gm = min(G, m_tiles - m0);
  n = r / gm;
  m = m0 + (r - n * gm);
}

// A chain runs up to kMaxJobs CTA-pair GEMMs in one persistent launch (one
// layer's Wo, w1/w3, w2 and the next layer's QKV projections). The tiles of all
// jobs form one list, job after job, each job's tiles in its own order
// (pair_tile with its m_group); pair p takes positions p, p + pairs, ... in
// order. A job may read rows another job of the chain writes (dep): before
// reading the 128 rows of block r of its A operand, and before its epilogue
// touches rows of r, a CTA waits (bounded) until the dep job has published
// all of its tiles of r (ready counter == the dep job's column tiles). A tile
// only waits for tiles earlier in the list, every pair handles its
// positions in order, and all pairs are resident at once, so every wait ends.
// The first job reads what earlier kernels wrote (programmatic dependent
// launch: its weight tiles are requested before griddepcontrol.wait).
constexpr int kMaxJobs = 4;
struct ChainJob {
  int M, N, K, kind, m_group;
  int m_tiles, n_tiles, kb, G, tile0;  // tile0: first list position of the job
  int dep;                             // job whose output rows it reads (-1: none)
  int* ready;                          // per-128-row counters this job publishes (nullptr: none)
  EpiArgs epi;
};
struct ChainArgs {
  CUtensorMap tmA[kMaxJobs];
  CUtensorMap tmB[kMaxJobs];
  ChainJob job[kMaxJobs];
  int n_jobs, total;
};

// List position t -> job j, 256-row block m and 256-column block n.
__device__ __forceinline__ int chain_tile(const ChainArgs& c, int t, int& m, int& n) {
  int j = 0;
  while (j + 1 < c.n_jobs && t >= c.job[j + 1].tile0) ++j;
  const ChainJob& J = c.job[j];
  pair_tile(t - J.tile0, J.m_tiles, J.G, m, n, J.n_tiles);
  return j;
}

template <int KIND, typename T>
__device__ __forceinline__ float chain_epi_row32(const EpiArgs& e, int m, int n0, const float (&v)[32], float rs) {
  return epi_row32<KIND, T>(e, m, n0, v, rs);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_chain_kernel(const __grid_constant__ ChainArgs args, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P_STAGES * P_STAGE_BYTES);
  uint64_t* empty = full + P_STAGES;
  uint64_t* accf = empty + P_STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;
  const int tiles = args.total;

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&accf[a], 1); mbar_init(&acce[a], 2 * 128); }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc2(tmem_slot, 512); tmem_relinquish2(); }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM of both allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // rows of block mb of job j's A operand (and output) are complete in its dep job
  auto rows_ready = [&](int j, int mb) -> bool {
    const int d = args.job[j].dep;
    if (d < 0) return true;
    return counter_wait_geq(args.job[d].ready + 2 * mb + (int)rank, args.job[d].n_tiles, status);
  };

  if (warp == 0 && lane == 0) {
    for (int j = 0; j < args.n_jobs; ++j) {
      tma_prefetch_desc(&args.tmA[j]);
      tma_prefetch_desc(&args.tmB[j]);
    }
    const uint64_t pol_a = l2_policy_evict_last(), pol_b = l2_policy_evict_last();
    int stage = 0, issued = 0;
    uint32_t phase = 0;
    bool ok = true;
    bool waited = false;   // griddepcontrol.wait done (before the first A operand)
    for (int t = pair; t < tiles && ok; t += pairs) {
      int tm, tn;
      const int j = chain_tile(args, t, tm, tn);
      const ChainJob& J = args.job[j];
      const CUtensorMap* ta = &args.tmA[j];
      const CUtensorMap* tb = &args.tmB[j];
      const int m0 = tm * 2 * P_BM + (int)rank * P_BM;
      const int n0 = tn * P_BN + (int)rank * (P_BN / 2);
      int k = 0;
      if (!waited) {  // weight halves of the first stages before waiting for the previous kernel
        const int pre = J.kb < P_STAGES ? J.kb : P_STAGES;
        for (; k < pre; ++k) {
          if (leader) mbar_arrive_expect_tx(&full[k], 2 * P_STAGE_BYTES);
          tma_load_2d_pair(smem + k * P_STAGE_BYTES + P_A_BYTES, tb, mapa_shared(smem_u32(&full[k]), 0), k * BK, n0,
                           pol_b);
        }
        pdl_wait();
        waited = true;
        ok = rows_ready(j, tm);
        fence_proxy_async_global();
        for (int kk = 0; kk < pre; ++kk)   // issued even after a failed wait: the barriers expect these bytes
          tma_load_2d_pair(smem + kk * P_STAGE_BYTES, ta, mapa_shared(smem_u32(&full[kk]), 0), kk * BK, m0, pol_a);
        issued = pre;
        stage = pre % P_STAGES;
        phase = pre == P_STAGES ? 1u : 0u;
        if (!ok) break;
      } else {
        if (!(ok = rows_ready(j, tm))) break;
        fence_proxy_async_global();
      }
      for (; k < J.kb; ++k) {
        if (!mbar_wait(&empty[stage], phase ^ 1, status)) { ok = false; break; }
        uint8_t* sa = smem + stage * P_STAGE_BYTES;
        const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
        if (leader) mbar_arrive_expect_tx(&full[stage], 2 * P_STAGE_BYTES);
        tma_load_2d_pair(sa, ta, fb, k * BK, m0, pol_a);
        tma_load_2d_pair(sa + P_A_BYTES, tb, fb, k * BK, n0, pol_b);
        ++issued;
        if (++stage == P_STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (!waited) pdl_wait();
    if (!ok && leader) drain_loads(full, stage, phase, issued, P_STAGES, status);
  } else if (warp == 1 && lane == 0 && leader) {
    constexpr uint32_t idesc = umma_idesc_16(UmmaFmt<T>::value, 2 * P_BM, P_BN);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true, any = false;
    for (int t = pair; t < tiles && ok; t += pairs) {
      int tm, tn;
      const int kb = args.job[chain_tile(args, t, tm, tn)].kb;
      if (!mbar_wait_cluster(&acce[acc], acc_phase ^ 1, status)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem + acc * P_BN;
      for (int k = 0; k < kb; ++k) {
        if (!mbar_wait(&full[stage], phase, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + stage * P_STAGE_BYTES);
        const uint32_t b_addr = a_addr + P_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma2_f16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32), idesc,
                    (k | kk) != 0);
        umma2_commit_pair(&empty[stage], 0x3);
        any = true;
        if (++stage == P_STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      umma2_commit_pair(&accf[acc], 0x3);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (!ok && any) {  // let issued MMAs finish before TMEM is released
      umma2_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, status);
    }
  } else if (warp >= 2) {
    pdl_wait();  // the epilogue reads and writes memory owned by earlier kernels
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool failed = false;  // after a timed-out wait the MMA has stopped: no further waits
    for (int t = pair; t < tiles; t += pairs) {
      int tm, tn;
      const int j = chain_tile(args, t, tm, tn);
      const ChainJob& J = args.job[j];
      const EpiArgs& epi = J.epi;
      const int m0 = tm * 2 * P_BM + (int)rank * P_BM, n0 = tn * P_BN;
      if (!failed) failed = !__all_sync(0xffffffffu, mbar_wait(&accf[acc], acc_phase, status));
      // already complete (the producer warp waited for it): acquires those rows' writes for this thread
      if (!failed && J.dep >= 0) failed = !__all_sync(0xffffffffu, rows_ready(j, tm));
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + acc * P_BN;
      const int kind = J.kind;
      const float rs = (kind == EPI_QKV_ROPE || kind == EPI_SWIGLU) && epi.ss_in && m0 + row < J.M
                           ? norm_row_scale(epi, m0 + row) : 1.f;
      float ssq = 0.f;
#pragma unroll 1
      for (int c = 0; c < P_BN / 32; ++c) {
        float v[32];
        if (!failed) {
          tmem_ld32(base + c * 32, v);
          if (n0 + c * 32 < J.N) {
            switch (kind) {
              case EPI_STORE_F32: ssq += chain_epi_row32<EPI_STORE_F32, T>(epi, m0 + row, n0 + c * 32, v, rs); break;
              case EPI_RESIDUAL: ssq += chain_epi_row32<EPI_RESIDUAL, T>(epi, m0 + row, n0 + c * 32, v, rs); break;
              case EPI_SWIGLU: ssq += chain_epi_row32<EPI_SWIGLU, T>(epi, m0 + row, n0 + c * 32, v, rs); break;
              default: ssq += chain_epi_row32<EPI_QKV_ROPE, T>(epi, m0 + row, n0 + c * 32, v, rs); break;
            }
          }
        }
      }
      if (kind == EPI_RESIDUAL && epi.ss_out && m0 + row < J.M) epi.ss_out[(size_t)(m0 + row) * epi.ss_n + n0 / P_BN] = ssq;
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(smem_u32(&acce[acc]), 0));
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      if (J.ready) {   // this CTA's 128 rows of the tile are written: publish them
        named_bar_sync(1, 128);
        if (warp == 2 && lane == 0) {
          __threadfence();
          atomicAdd(J.ready + 2 * tm + (int)rank, 1);
        }
      }
    }
  }
  tc_fence_before();
  cluster_sync_all();  // no MMA of the pair and no epilogue read is left when TMEM goes
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem, 512);
  }
}

// ---------------------------------------------------------------- skinny
// Stream-K over (weight tile, k-block) units: of the U = tiles * kb units
// (tile-major), CTA c of G takes [U*c/G, U*(c+1)/G), so every CTA streams the
// same number of weight bytes to within one 16 KB block. A CTA's range falls
// into pieces, one per tile it touches. A piece covering its whole tile runs
// the epilogue directly. A split tile is finished by its owner, the CTA whose
// piece holds k-block 0 (always the last piece of the owner's range); every
// other piece of the tile is the first piece of its CTA's range, stored in
// that CTA's workspace slot and counted in the tile's counter. The owner waits
// (bounded) for the count, adds the shares in CTA order, runs the epilogue and
// re-arms the counter: results do not depend on timing. Residual tiles are the
// exception: x += sum is linear, so every piece adds its share into x with
// vector atomics and nothing waits (measured faster on decode than the owner
// fixup, whose x read-modify-write lands at the end of the kernel); their
// summation order varies from run to run at fp32 rounding level. All CTAs of the grid
// (one per SM) are resident together and owners wait only for first pieces,
// which wait for nothing, so the waits end. Accumulators are double-buffered
// in TMEM so the MMA runs on while a piece drains.
template <int NT>
struct SkinnyCfg {
  static constexpr int B_BYTES = NT * BK * 2;
  static constexpr int STAGE_BYTES = S_A_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 8 ? 8 : (200 * 1024) / STAGE_BYTES;
  static constexpr int TRANS_LD = S_BM + 4;                 // padded row of the transpose buffer (floats)
  static constexpr int TRANS_BYTES = 32 * TRANS_LD * 4;      // 32 tokens x 128 features
  static constexpr int SMEM = STAGES * STAGE_BYTES + TRANS_BYTES + 1024 + 256;
  static constexpr uint32_t TMEM_COLS = 2 * NT <= 32 ? 32 : (2 * NT <= 64 ? 64 : (2 * NT <= 128 ? 128 : (2 * NT <= 256 ? 256 : 512)));
};

template <int KIND, typename T, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_skinny_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, int M,
                       int N, int K, EpiArgs epi, float* __restrict__ ws, int* __restrict__ counters,
                       int* status) {
  using C = SkinnyCfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  float* trans = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::TRANS_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = (N + S_BM - 1) / S_BM;
  const int kb = (K + BK - 1) / BK;
  const long long U = (long long)tiles * kb, G = gridDim.x;
  const long long u0 = sk_first(blockIdx.x, U, G), u1 = sk_first(blockIdx.x + 1, U, G);

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&accf[a], 1); mbar_init(&acce[a], 128); }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, C::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    const uint64_t pol_w = l2_policy_evict_first(), pol_x = l2_policy_evict_last();
    // Weight blocks do not depend on the previous kernel: the first stages are
    // requested before waiting for it, their activation halves after.
    const int pre = (int)((u1 - u0) < C::STAGES ? (u1 - u0) : C::STAGES);
    for (int i = 0; i < pre; ++i) {
      const long long u = u0 + i;
      mbar_arrive_expect_tx(&full[i], C::STAGE_BYTES);
      tma_load_2d(smem + i * C::STAGE_BYTES, &tmW, &full[i], (int)(u % kb) * BK, (int)(u / kb) * S_BM, pol_w);
    }
    pdl_wait();
    for (int i = 0; i < pre; ++i) {
      const long long u = u0 + i;
      tma_load_2d(smem + i * C::STAGE_BYTES + S_A_BYTES, &tmX, &full[i], (int)(u % kb) * BK, 0, pol_x);
    }
    int stage = pre % C::STAGES, issued = pre;
    uint32_t phase = pre == C::STAGES ? 1u : 0u;
    bool ok = true;
    for (long long u = u0 + pre; u < u1; ++u) {
      if (!mbar_wait(&empty[stage], phase ^ 1, status)) { ok = false; break; }
      uint8_t* sa = smem + stage * C::STAGE_BYTES;
      mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
      tma_load_2d(sa, &tmW, &full[stage], (int)(u % kb) * BK, (int)(u / kb) * S_BM, pol_w);
      tma_load_2d(sa + S_A_BYTES, &tmX, &full[stage], (int)(u % kb) * BK, 0, pol_x);
      ++issued;
      if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
    }
    if (!ok) drain_loads(full, stage, phase, issued, C::STAGES, status);
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = umma_idesc_16(UmmaFmt<T>::value, S_BM, NT);
    int stage = 0, buf = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true, any = false;
    for (long long u = u0; u < u1 && ok;) {
      const int klo = (int)(u % kb);
      const int n = (int)((u1 - u) < (kb - klo) ? (u1 - u) : (kb - klo));
      if (!mbar_wait(&acce[buf], acc_phase ^ 1, status)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem + buf * NT;
      for (int k = 0; k < n; ++k) {
        if (!mbar_wait(&full[stage], phase, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + stage * C::STAGE_BYTES);
        const uint32_t b_addr = a_addr + S_A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_bf16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32), idesc,
                    (k | kk) != 0);
        umma_commit(&empty[stage]);
        any = true;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      umma_commit(&accf[buf]);
      if (++buf == 2) { buf = 0; acc_phase ^= 1; }
      u += n;
    }
    if (!ok && any) {
      umma_commit(drain);
      mbar_wait(drain, 0, status);
    }
  } else if (warp >= 2) {
    pdl_wait();  // the epilogue reads and writes memory owned by earlier kernels
    // TMEM hands each thread one weight row (feature) across 32 tokens; the
    // tile is turned around in shared memory so that thread (token = lane,
    // 32-feature chunk = ew) runs the same row epilogue as the wide GEMM.
    const int quarter = warp & 3;          // TMEM lanes this warp may read
    const int ew = warp - 2;               // feature chunk in the row phase
    const int tid = ew * 32 + lane;        // 0..127
    int buf = 0;
    uint32_t acc_phase = 0;
    for (long long u = u0; u < u1;) {
      const int tile = (int)(u / kb), klo = (int)(u % kb);
      const int n = (int)((u1 - u) < (kb - klo) ? (u1 - u) : (kb - klo));
      const bool whole = klo == 0 && n == kb;
      // residual tiles: every piece adds its share into x atomically (linear,
      // no waiting at the end of the kernel; the summation order varies);
      // other split tiles: owner fixup
      const bool atomic_piece = KIND == EPI_RESIDUAL && !whole;
      const bool owner = !whole && !atomic_piece && klo == 0;   // k-block 0: the last piece of this CTA's range
      const bool share = !whole && !atomic_piece && klo != 0;   // the first piece of this CTA's range
      const int f0 = tile * S_BM + ew * 32;
      const long long t0 = (long long)tile * kb;
      long long c_own = 0, c_hi = 0;
      if (!whole) { c_own = sk_owner(t0, U, G); c_hi = sk_owner(t0 + kb - 1, U, G); }
      if (owner) {  // the other shares of this tile (their CTAs' first pieces) before the epilogue
        if (threadIdx.x == 64) {
          int need = 0;
          for (long long cc = c_own + 1; cc <= c_hi; ++cc) need += sk_first(cc + 1, U, G) > sk_first(cc, U, G);
          counter_wait_geq(&counters[tile], need, status);   // a timeout is latched in status
          counters[tile] = 0;
        }
        named_bar_sync(1, 128);
        __threadfence();
      }
      // all lanes of a warp take the same branch so the warp-wide TMEM loads stay converged
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&accf[buf], acc_phase, status));
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + buf * NT;
#pragma unroll 1
      for (int c = 0; c < NT / 32; ++c) {
        float v[32];
        if (ok) tmem_ld32(base + c * 32, v);
        else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
        if (c == NT / 32 - 1) {  // TMEM no longer needed: the MMA may refill this buffer
          tc_fence_before();
          mbar_arrive(&acce[buf]);
        }
        named_bar_sync(1, 128);  // earlier readers of the transpose buffer are done
#pragma unroll
        for (int j = 0; j < 32; ++j) trans[j * C::TRANS_LD + quarter * 32 + lane] = v[j];
        named_bar_sync(1, 128);
        const float4* src = reinterpret_cast<const float4*>(trans + lane * C::TRANS_LD + ew * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 x = src[j];
          v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
        }
        const int m = c * 32 + lane;
        if (atomic_piece) {
          if (m < epi.M) {
            float* dst = epi.out + (size_t)m * epi.ldo + f0;
            if (f0 + 32 <= epi.N && (epi.ldo & 3) == 0) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                atomicAdd(reinterpret_cast<float4*>(dst) + j, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (f0 + j < epi.N) atomicAdd(dst + j, v[j]);
            }
          }
          continue;
        }
        // a share: float4 (c*8 + j)*128 + tid of the CTA's slot, so a warp's
        // accesses are 512 contiguous bytes
        if (share) {
          float4* p4 = reinterpret_cast<float4*>(ws) + (size_t)blockIdx.x * (NT * S_BM / 4) + tid;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            __stcg(p4 + (c * 8 + j) * 128, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
          continue;
        }
        if (owner) {  // add the other shares in CTA order, four shares' loads in flight at a time
          for (long long c0 = c_own + 1; c0 <= c_hi; c0 += 4) {
            float4 x[4][8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const long long cc = c0 + q;
              if (cc <= c_hi && sk_first(cc + 1, U, G) > sk_first(cc, U, G)) {   // a CTA with units
                const float4* p4 = reinterpret_cast<const float4*>(ws) + (size_t)cc * (NT * S_BM / 4) + tid;
#pragma unroll
                for (int j = 0; j < 8; ++j) x[q][j] = __ldcg(p4 + (c * 8 + j) * 128);
              } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) x[q][j] = make_float4(0.f, 0.f, 0.f, 0.f);
              }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                v[4 * j] += x[q][j].x; v[4 * j + 1] += x[q][j].y; v[4 * j + 2] += x[q][j].z; v[4 * j + 3] += x[q][j].w;
              }
            }
          }
        }
        epi_row32<KIND, T>(epi, m, f0, v);
      }
      if (share) {  // publish the share
        __threadfence();
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) atomicAdd(&counters[tile], 1);
      }
      if (++buf == 2) { buf = 0; acc_phase ^= 1; }
      u += n;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// -------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

// 16-bit row-major [rows, cols] matrix with row pitch `pitch` elements, boxes
// of box_rows x 64 elements, 128-byte swizzle, zero fill outside the matrix.
int make_tmap_16(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t pitch, int box_rows,
                 bool is_f16) {
  auto fn = encode_fn();
  if (!fn) return LLAMA_ERR_CUDA;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (pitch * 2) % 16 != 0) return LLAMA_ERR_INVALID_ARG;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)(pitch * 2)};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, is_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), gdim, gstride, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LLAMA_OK : LLAMA_ERR_CUDA;
}

namespace {
PerDeviceValue<int> g_sm_count;
OncePerDevice g_smem_attr;
int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return dev;
}
}  // namespace

uint64_t context_key() {
  typedef CUresult (*GetCurrent)(CUcontext*);
  typedef CUresult (*GetId)(CUcontext, unsigned long long*);
  struct Fns {
    GetCurrent cur = nullptr;
    GetId id = nullptr;
  };
  static const Fns fns = [] {
    Fns f;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.cur = reinterpret_cast<GetCurrent>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.id = reinterpret_cast<GetId>(p);
    cudaGetLastError();
    return f;
  }();
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (fns.cur && fns.id && fns.cur(&c) == CUDA_SUCCESS && c != nullptr && fns.id(c, &id) == CUDA_SUCCESS)
    return id;
  return (1ull << 63) | (uint64_t)(uint32_t)current_device();
}

int num_sms() {
  const int dev = current_device();
  return g_sm_count.get(dev, [dev] {
    int n = 0;
    if (dev < 0 || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return n;
  }, 148);
}

int ensure_smem_attr(const void* kern, int bytes) {
  // Attributes belong to a context: key by the current one, so that a device
  // reset (new context) sets them again.
  const uint64_t key = context_key();
  return g_smem_attr.run(key, kern, [&] {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess) return 0;
    cudaGetLastError();
    return (int)LLAMA_ERR_CUDA;
  });
}

bool streamk_enabled() {
  static const bool on = getenv("LLAMA_NO_STREAMK") == nullptr;
  return on;
}

// Split of a wide GEMM of T output tiles over G SMs. With fewer tiles than
// SMs, every tile is cut into (tile, k-block) units spread over up to G CTAs
// (at least 8 k-blocks each), so all SMs stream the reduction dimension.
// With at least one full wave the tiles stay data-parallel: measured on the
// 8B prefill shapes, splitting the tail wave lost more (the fixup, and CTAs
// no longer walking K in step, which shares A and B slices in L2) than the
// idle SMs of the last wave cost.
WideSplit wide_split(int M, int N, int K) {
  WideSplit w;
  const int T = ((M + W_BM - 1) / W_BM) * ((N + W_BN - 1) / W_BN), G = num_sms(), kb = (K + BK - 1) / BK;
  int sk = 0;
  if (T < G && streamk_enabled()) sk = T;
  w.tiles = T;
  w.sk_tiles = sk;
  w.T_dp = T - sk;
  const long long U = (long long)sk * kb;
  w.G_sk = sk ? (int)std::min<long long>(G, std::max<long long>(1, U / 8)) : 0;
  w.grid = w.T_dp > 0 ? std::min(T, G) : w.G_sk;
  return w;
}

size_t wide_workspace_floats() { return (size_t)num_sms() * W_BM * W_BN; }

template <int KIND, typename T>
static int launch_wide(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K, const EpiArgs& e,
                       GemmScratch* scratch, int* status, cudaStream_t st) {
  auto kern = gemm_wide_kernel<KIND, T>;
  if (const int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), W_SMEM)) return rc;
  WideSplit w = wide_split(M, N, K);
  float* ws = nullptr;
  int* tickets = nullptr;
  if (w.sk_tiles > 0) {
    // partial-tile workspace and tickets; without them the tail wave stays data-parallel
    if (scratch && scratch->ws && scratch->ws_floats >= wide_workspace_floats() && scratch->tickets &&
        scratch->n_tickets >= w.sk_tiles) {
      ws = scratch->ws;
      tickets = scratch->tickets;
    } else {
      w.T_dp = w.tiles;
      w.G_sk = 0;
      w.grid = std::min(w.tiles, num_sms());
    }
  }
  const cudaError_t err = launch_k(kern, dim3(w.grid), dim3(kThreads), W_SMEM, st, ta, tb, M, N, K, e, w.T_dp,
                                   w.G_sk, ws, tickets, status);
  return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

bool pair_gemm_enabled() {
  static const bool on = getenv("LLAMA_NO_PAIR_GEMM") == nullptr;
  return on;
}

bool gemm16_uses_pair(int M, int N, int K) { return M > 128 && pair_gemm_enabled() && wide_split(M, N, K).sk_tiles == 0; }

// One persistent launch of the CTA-pair kernel over the jobs' tiles.
template <typename T>
static int launch_chain(const ChainJobDesc* jobs, int n, int* status, cudaStream_t st) {
  constexpr bool F16 = std::is_same<T, f16>::value;
  if (n <= 0 || n > kMaxJobs) return LLAMA_ERR_INVALID_ARG;
  ChainArgs args;
  memset(&args, 0, sizeof(args));
  int total = 0;
  for (int j = 0; j < n; ++j) {
    const ChainJobDesc& d = jobs[j];
    if (d.M <= 0 || d.N <= 0 || d.K <= 0) return LLAMA_ERR_SHAPE;
    if (d.K % 8 != 0 || d.lda % 8 != 0 || d.ldw % 8 != 0) return LLAMA_ERR_SHAPE;
    if (d.dep >= j || (d.dep >= 0 && !jobs[d.dep].ready)) return LLAMA_ERR_INVALID_ARG;
    int rc;
    if ((rc = make_tmap_16(&args.tmA[j], d.A, d.M, d.K, d.lda, P_BM, F16)) != LLAMA_OK) return rc;
    if ((rc = make_tmap_16(&args.tmB[j], d.W, d.N, d.K, d.ldw, P_BN / 2, F16)) != LLAMA_OK) return rc;
    ChainJob& J = args.job[j];
    J.M = d.M; J.N = d.N; J.K = d.K; J.kind = d.kind;
    J.m_tiles = (d.M + 2 * P_BM - 1) / (2 * P_BM);
    J.n_tiles = (d.N + P_BN - 1) / P_BN;
    J.kb = (d.K + BK - 1) / BK;
    J.G = d.m_group > 0 ? std::min(d.m_group, J.m_tiles) : J.m_tiles;
    J.m_group = J.G;
    J.tile0 = total;
    J.dep = d.dep;
    J.ready = d.ready;
    J.epi = d.epi;
    total += J.m_tiles * J.n_tiles;
  }
  args.n_jobs = n;
  args.total = total;
  auto kern = gemm_chain_kernel<T>;
  if (const int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), P_SMEM)) return rc;
  const int pairs = std::min(total, num_sms() / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = P_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  count_launches(1);
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, args, status);
  return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

template <int KIND, typename T, int NT>
static int launch_skinny_nt(const CUtensorMap& tw, const CUtensorMap& tx, int M, int N, int K, const EpiArgs& e,
                            float* ws, int* counters, int* status, cudaStream_t st) {
  using C = SkinnyCfg<NT>;
  auto kern = gemm_skinny_kernel<KIND, T, NT>;
  if (const int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM)) return rc;
  const cudaError_t err = launch_k(kern, dim3(num_sms()), dim3(kThreads), C::SMEM, st, tw, tx, M, N, K, e, ws,
                                   counters, status);
  return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

template <int KIND, typename T>
static int launch_skinny(const CUtensorMap& tw, const CUtensorMap& tx, int M, int N, int K, int NT, const EpiArgs& e,
                         float* ws, int* counters, int* status, cudaStream_t st) {
  switch (NT) {
    case 32: return launch_skinny_nt<KIND, T, 32>(tw, tx, M, N, K, e, ws, counters, status, st);
    case 64: return launch_skinny_nt<KIND, T, 64>(tw, tx, M, N, K, e, ws, counters, status, st);
    case 128: return launch_skinny_nt<KIND, T, 128>(tw, tx, M, N, K, e, ws, counters, status, st);
    case 256: return launch_skinny_nt<KIND, T, 256>(tw, tx, M, N, K, e, ws, counters, status, st);
  }
  return LLAMA_ERR_INVALID_ARG;
}

static int skinny_nt(int M) {
  int nt = 32;
  while (nt < M) nt *= 2;
  return nt;
}

size_t skinny_workspace_floats(int M) { return (size_t)num_sms() * S_BM * skinny_nt(M); }

bool pdl_enabled() {
  static const bool on = getenv("LLAMA_NO_PDL") == nullptr;
  return on;
}

template <typename T>
static int gemm16_t(const void* A, int M, int K, int lda, const void* W, int N, int ldw, int kind, const EpiArgs& e,
                    int variant, GemmScratch* scratch, int* status, cudaStream_t st) {
  constexpr bool F16 = std::is_same<T, f16>::value;
  if (M <= 0 || N <= 0 || K <= 0) return LLAMA_ERR_SHAPE;
  if (K % 8 != 0 || lda % 8 != 0 || ldw % 8 != 0) return LLAMA_ERR_SHAPE;
  const bool skinny = variant == GEMM_SKINNY || (variant == GEMM_AUTO && M <= 128);
  int rc;
  if (!skinny) {
    CUtensorMap ta, tb;
    if (gemm16_uses_pair(M, N, K)) {
      // at least one full wave of 128x256 tiles: CTA pairs on 256x256 tiles (a chain of one job)
      if (kind < EPI_STORE_F32 || kind > EPI_QKV_ROPE) return LLAMA_ERR_INVALID_ARG;
      ChainJobDesc d{A, lda, W, ldw, M, N, K, kind, 0, -1, nullptr, e};
      return launch_chain<T>(&d, 1, status, st);
    }
    if ((rc = make_tmap_16(&ta, A, M, K, lda, W_BM, F16)) != LLAMA_OK) return rc;
    if ((rc = make_tmap_16(&tb, W, N, K, ldw, W_BN, F16)) != LLAMA_OK) return rc;
    switch (kind) {
      case EPI_STORE_F32: return launch_wide<EPI_STORE_F32, T>(ta, tb, M, N, K, e, scratch, status, st);
      case EPI_RESIDUAL: return launch_wide<EPI_RESIDUAL, T>(ta, tb, M, N, K, e, scratch, status, st);
      case EPI_SWIGLU: return launch_wide<EPI_SWIGLU, T>(ta, tb, M, N, K, e, scratch, status, st);
      case EPI_QKV_ROPE: return launch_wide<EPI_QKV_ROPE, T>(ta, tb, M, N, K, e, scratch, status, st);
    }
    return LLAMA_ERR_INVALID_ARG;
  }
  if (M > 256) return LLAMA_ERR_SHAPE;
  const int NT = skinny_nt(M);
  const int tiles = (N + S_BM - 1) / S_BM;
  if (!scratch || !scratch->ws || scratch->ws_floats < skinny_workspace_floats(M) || !scratch->tickets ||
      scratch->n_tickets < tiles)
    return LLAMA_ERR_INVALID_ARG;
  CUtensorMap tw, tx;
  if ((rc = make_tmap_16(&tw, W, N, K, ldw, S_BM, F16)) != LLAMA_OK) return rc;
  if ((rc = make_tmap_16(&tx, A, M, K, lda, NT, F16)) != LLAMA_OK) return rc;
  float* ws = scratch->ws;
  int* tk = scratch->tickets;
  switch (kind) {
    case EPI_STORE_F32: return launch_skinny<EPI_STORE_F32, T>(tw, tx, M, N, K, NT, e, ws, tk, status, st);
    case EPI_RESIDUAL: return launch_skinny<EPI_RESIDUAL, T>(tw, tx, M, N, K, NT, e, ws, tk, status, st);
    case EPI_SWIGLU: return launch_skinny<EPI_SWIGLU, T>(tw, tx, M, N, K, NT, e, ws, tk, status, st);
    case EPI_QKV_ROPE: return launch_skinny<EPI_QKV_ROPE, T>(tw, tx, M, N, K, NT, e, ws, tk, status, st);
  }
  return LLAMA_ERR_INVALID_ARG;
}

int gemm16_chain(const ChainJobDesc* jobs, int n, int elt, int* status, cudaStream_t st) {
  for (int j = 0; j < n; ++j)
    if (!gemm16_uses_pair(jobs[j].M, jobs[j].N, jobs[j].K)) return LLAMA_ERR_UNSUPPORTED;
  if (elt == LLAMA_F16) return launch_chain<f16>(jobs, n, status, st);
  if (elt == LLAMA_BF16) return launch_chain<bf16>(jobs, n, status, st);
  return LLAMA_ERR_INVALID_ARG;
}

int gemm16(const void* A, int M, int K, int lda, const void* W, int N, int ldw, int elt, int kind, const EpiArgs& e,
           int variant, GemmScratch* scratch, int* status, cudaStream_t st) {
  if (elt == LLAMA_F16) return gemm16_t<f16>(A, M, K, lda, W, N, ldw, kind, e, variant, scratch, status, st);
  if (elt == LLAMA_BF16) return gemm16_t<bf16>(A, M, K, lda, W, N, ldw, kind, e, variant, scratch, status, st);
  return LLAMA_ERR_INVALID_ARG;
}

}  // namespace llama
