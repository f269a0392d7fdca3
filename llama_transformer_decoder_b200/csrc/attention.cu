// Causal grouped-query attention over the KV cache.
//
//  * prefill (bf16 / fp16): the tcgen05 flash-attention kernel in attention_tc.cu.
//  * prefill (fp32): one warp per query row on the CUDA cores.
//  * decode (both dtypes): split over the cached keys. Each CTA serves the
//    H/Hk query heads of one kv head, streams its key range through shared
//    memory with bulk async copies (the step is bound by HBM reads of the
//    cache), keeps (max, sum, o) per head, and a combine kernel merges the
//    splits with the log-sum-exp rule.
#include <cstdlib>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace llama {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------ mma.sync helpers (decode)

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Tile rows are 256 B (128 16-bit values); 16-byte chunk c of row r lives at chunk c ^ (r & 7).
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 256 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr));
}
// m16n8k16 tensor-core product, fp32 accumulate; T = bf16 or fp16 operands.
template <typename T>
__device__ __forceinline__ void mma16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1) {
  if constexpr (std::is_same<T, f16>::value) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

// ------------------------------------------------------ fp32 prefill (SIMT)
template <int D>
__global__ void __launch_bounds__(32) attn_prefill_f32_kernel(const float* __restrict__ q,
                                                              const float* __restrict__ kc,
                                                              const float* __restrict__ vc, float* __restrict__ o,
                                                              const int32_t* __restrict__ pos0, int S, int H,
                                                              int Hk, int Smax, float scale_log2) {
  pdl_wait();
  constexpr int DPL = D / 32;
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z, lane = threadIdx.x;
  const int g = h / (H / Hk);
  const int qp = (pos0 ? pos0[b] : 0) + s;
  const float* qv = q + (((size_t)b * H + h) * S + s) * D;
  const float* kb = kc + ((size_t)b * Hk + g) * Smax * D;
  const float* vb = vc + ((size_t)b * Hk + g) * Smax * D;
  float acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int j0 = 0; j0 <= qp; j0 += 32) {
    const int j = j0 + lane;
    float sc = -INFINITY;
    if (j <= qp) {
      float dot = 0.f;
      for (int t = 0; t < D; ++t) dot = fmaf(qv[t], kb[(size_t)j * D + t], dot);
      sc = dot * scale_log2;
    }
    float cm = sc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
    const float mn = fmaxf(m, cm);
    const float corr = exp2f(m - mn);
    const float p = (j <= qp) ? exp2f(sc - mn) : 0.f;
    float ps = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * corr + ps;
    m = mn;
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] *= corr;
    const int nk = min(32, qp + 1 - j0);
    for (int jj = 0; jj < nk; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[i] = fmaf(pj, vb[(size_t)(j0 + jj) * D + lane + 32 * i], acc[i]);
    }
  }
  float* dst = o + ((size_t)b * S + s) * H * D + h * D;
#pragma unroll
  for (int i = 0; i < DPL; ++i) dst[lane + 32 * i] = acc[i] / l;
}

// ------------------------------------------------------------ decode
constexpr int DEC_STAGES = 3;
// keys per shared-memory stage: K and V rows of one stage fill at most 64 KB
template <typename T, int D>
__host__ __device__ constexpr int dec_sub() { return (32768 / (D * (int)sizeof(T))) < 128 ? (32768 / (D * (int)sizeof(T))) : 128; }
constexpr int DEC_MAXG = 8;      // query heads per kv head supported

template <typename T, int D>
__global__ void __launch_bounds__(128) attn_decode_part_kernel(const T* __restrict__ q, const T* __restrict__ kc,
                                                               const T* __restrict__ vc,
                                                               const int32_t* __restrict__ nkeys, int add_keys,
                                                               float* __restrict__ part, int H, int Hk, int Smax,
                                                               int chunk, float scale_log2, int* status) {
  constexpr int DPL = D / 32;                       // dims per lane
  constexpr int DEC_SUB = dec_sub<T, D>();
  constexpr int ROW = D * (int)sizeof(T);           // bytes per cached key
  constexpr int STAGE = 2 * DEC_SUB * ROW;          // K and V rows of one stage
  extern __shared__ __align__(128) uint8_t sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + DEC_STAGES * STAGE);
  float* red = reinterpret_cast<float*>(bars + DEC_STAGES);   // [4 warps][G][D + 2]

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z, splits = gridDim.x;
  const int G = H / Hk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = nkeys[b] + add_keys;
  const int k_lo = split * chunk;
  const int k_hi = min(n, k_lo + chunk);
  const int nsub = k_hi > k_lo ? (k_hi - k_lo + DEC_SUB - 1) / DEC_SUB : 0;
  const T* ksrc = kc + ((size_t)b * Hk + g) * Smax * D;
  const T* vsrc = vc + ((size_t)b * Hk + g) * Smax * D;

  if ((n < 1 || n > Smax) && split == 0 && threadIdx.x == 0) set_status(status, LLAMA_ERR_DEVICE_BOUNDS);

  // this lane's slice of the G query vectors, pre-scaled for exp2
  float qr[DEC_MAXG][DPL];
#pragma unroll
  for (int gg = 0; gg < DEC_MAXG; ++gg)
#pragma unroll
    for (int i = 0; i < DPL; ++i)
      qr[gg][i] = gg < G ? to_f<T>(q[((size_t)b * H + g * G + gg) * D + lane * DPL + i]) * scale_log2 : 0.f;

  if (threadIdx.x == 0) {
    for (int s = 0; s < DEC_STAGES; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](int sub) {
    const int st = sub % DEC_STAGES;
    const int k0 = k_lo + sub * DEC_SUB;
    const int rows = min(DEC_SUB, k_hi - k0);
    uint8_t* dst = sm + st * STAGE;
    mbar_arrive_expect_tx(&bars[st], 2 * rows * ROW);
    bulk_load(dst, ksrc + (size_t)k0 * D, rows * ROW, &bars[st]);
    bulk_load(dst + DEC_SUB * ROW, vsrc + (size_t)k0 * D, rows * ROW, &bars[st]);
  };
  if (threadIdx.x == 0 && n <= Smax)
    for (int s = 0; s < DEC_STAGES && s < nsub; ++s) issue(s);

  float m[DEC_MAXG], l[DEC_MAXG], acc[DEC_MAXG][DPL];
#pragma unroll
  for (int gg = 0; gg < DEC_MAXG; ++gg) {
    m[gg] = -INFINITY;
    l[gg] = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[gg][i] = 0.f;
  }
  bool ok = n <= Smax;
  int fail_sub = nsub;
  for (int sub = 0; sub < nsub && ok; ++sub) {
    const int st = sub % DEC_STAGES;
    const bool arrived = mbar_wait(&bars[st], (sub / DEC_STAGES) & 1, status);
    if (!__syncthreads_and(arrived)) { ok = false; fail_sub = sub; break; }
    const int k0 = k_lo + sub * DEC_SUB;
    const int rows = min(DEC_SUB, k_hi - k0);
    const T* sk = reinterpret_cast<const T*>(sm + st * STAGE);
    const T* sv = reinterpret_cast<const T*>(sm + st * STAGE + DEC_SUB * ROW);
    // this warp's 32 keys of the stage: lane kk keeps the scores of key kk
    const int kw = warp * 32;
    float mine[DEC_MAXG];
#pragma unroll
    for (int gg = 0; gg < DEC_MAXG; ++gg) mine[gg] = -INFINITY;
    const int nk = min(32, rows - kw);
    for (int kk = 0; kk < nk; ++kk) {
      float kv[DPL];
#pragma unroll
      for (int i = 0; i < DPL; ++i) kv[i] = to_f<T>(sk[(size_t)(kw + kk) * D + lane * DPL + i]);
#pragma unroll
      for (int gg = 0; gg < DEC_MAXG; ++gg) {
        if (gg < G) {
          float dot = 0.f;
#pragma unroll
          for (int i = 0; i < DPL; ++i) dot = fmaf(qr[gg][i], kv[i], dot);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
          if (lane == kk) mine[gg] = dot;
        }
      }
    }
    float p[DEC_MAXG];
#pragma unroll
    for (int gg = 0; gg < DEC_MAXG; ++gg) {
      if (gg < G && nk > 0) {
        float cm = mine[gg];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
        const float mn = fmaxf(m[gg], cm);
        const float corr = exp2f(m[gg] - mn);
        p[gg] = lane < nk ? exp2f(mine[gg] - mn) : 0.f;
        float ps = p[gg];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l[gg] = l[gg] * corr + ps;
        m[gg] = mn;
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[gg][i] *= corr;
      } else {
        p[gg] = 0.f;
      }
    }
    for (int kk = 0; kk < nk; ++kk) {
      float vv[DPL];
#pragma unroll
      for (int i = 0; i < DPL; ++i) vv[i] = to_f<T>(sv[(size_t)(kw + kk) * D + lane * DPL + i]);
#pragma unroll
      for (int gg = 0; gg < DEC_MAXG; ++gg) {
        if (gg < G) {
          const float pk = __shfl_sync(0xffffffffu, p[gg], kk);
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc[gg][i] = fmaf(pk, vv[i], acc[gg][i]);
        }
      }
    }
    __syncthreads();  // every warp is done with this stage before it is refilled
    if (threadIdx.x == 0 && sub + DEC_STAGES < nsub) issue(sub + DEC_STAGES);
  }
  if (!ok && threadIdx.x == 0) {
    // do not leave copies in flight: wait (bounded) for every issued stage
    for (int sub = fail_sub; sub < nsub && sub < fail_sub + DEC_STAGES; ++sub)
      mbar_wait(&bars[sub % DEC_STAGES], (sub / DEC_STAGES) & 1, status);
  }
  // merge the 4 warps' states, then write this split's (o, max, sum) per head
  for (int gg = 0; gg < G; ++gg) {
    float* r = red + ((size_t)warp * DEC_MAXG + gg) * (D + 2);
#pragma unroll
    for (int i = 0; i < DPL; ++i) r[lane * DPL + i] = acc[gg][i];
    if (lane == 0) { r[D] = m[gg]; r[D + 1] = l[gg]; }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += 128) {
    const int gg = idx / D, dd = idx - gg * D;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, red[((size_t)w * DEC_MAXG + gg) * (D + 2) + D]);
    float L = 0.f, O = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float* r = red + ((size_t)w * DEC_MAXG + gg) * (D + 2);
      const float f = r[D] == -INFINITY ? 0.f : exp2f(r[D] - M);
      L += r[D + 1] * f;
      O += r[dd] * f;
    }
    float* dst = part + (((size_t)b * H + g * G + gg) * splits + split) * (D + 2);
    dst[dd] = O;
    if (dd == 0) { dst[D] = M; dst[D + 1] = L; }
  }
}

template <typename T, int D>
__global__ void attn_decode_combine_kernel(const float* __restrict__ part, T* __restrict__ o, int H, int splits) {
  const int h = blockIdx.x, b = blockIdx.y;
  const float* base = part + ((size_t)b * H + h) * splits * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, base[(size_t)s * (D + 2) + D]);
  for (int dd = threadIdx.x; dd < D; dd += blockDim.x) {
    float L = 0.f, O = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float* r = base + (size_t)s * (D + 2);
      const float f = r[D] == -INFINITY ? 0.f : exp2f(r[D] - M);
      L += r[D + 1] * f;
      O += r[dd] * f;
    }
    o[((size_t)b * H + h) * D + dd] = from_f<T>(O / L);
  }
}


// ---------------------------------------- decode, 16-bit d = 128 (mma)
// The work is the sequence of (sequence b, kv head g, 32-key tile t) triples
// in that order, T tiles in all, split into W ranges r = [T r / W, T (r+1) / W),
// one per decoding warp. When every warp has enough tiles, the last 25% of
// each range is cut into two sub-chunks (15% and 10% of the range) that warps
// claim from a counter once their own 75% is done: the first sub-chunks of all
// ranges, then the second ones, so the last claims are the short ones. Warps on SMs that stream slower than the others (measured: the same
// SMs every run, finishing 12-15 us after the median of a ~100 us launch)
// thereby stream less of the tail. Each claim is issued a few tiles before the
// warp needs it. Sub-chunk boundaries depend only on T and the chunk index,
// never on timing. Chunk id k = r * DM_SUB + s (s = 0: the owner's part)
// increases with tile position; cutting the chunks at (b, g) boundaries gives
// pieces, and the piece of (b, g) in chunk k is stored in slot (b*Hk + g) + k,
// which is unique since chunks and (b, g) ranges are both in tile order. The
// partials need B*Hk + W * DM_SUB slots (B*Hk + W without claimed
// sub-chunks), and the merge order is the same whichever warp ran a chunk.
//
// A warp streams its tiles through a private 3-stage ring of swizzled shared
// memory (cp.async, zero fill past the last key) without draining at chunk or
// piece boundaries, computes S^T = K Q^T and O^T += V^T P^T with mma.sync (the
// G query heads of the kv head are columns 0..G-1 of 8) and writes
// (o, max, sum) of every piece for the combine kernel.
constexpr int DM_KEYS = 32;
constexpr int DM_STAGES = 3;
constexpr int DM_WARPS = 4;
constexpr int DM_TILE = DM_KEYS * 256;             // one K (or V) tile: 32 rows x 256 B
constexpr int DM_STAGE = 2 * DM_TILE;
constexpr int DM_RING = DM_WARPS * DM_STAGES * DM_STAGE;
// Per-sequence tile prefix and key counts in shared memory (for B up to
// DM_SEEK_B), so that moving to a claimed chunk is a binary search, not a walk
// over every sequence's length in global memory.
constexpr int DM_SEEK_B = 128;
constexpr int DM_SMEM = DM_RING + (DM_SEEK_B + 1) * 8 + DM_SEEK_B * 4;
constexpr int DM_CLAIM_AHEAD = 3;                  // tiles before a chunk's end its successor is claimed
static_assert(DM_STAGES == 3, "the chunk queue holds the DM_STAGES - 1 chunks the loader may run ahead, plus one");
constexpr int DM_SUB = 3;                          // sub-chunks of a range (the owner's, then two claimed)
// Tiles per warp for claimed sub-chunks. Below ~128 (launches under ~200 us
// at batch 32) they measured slower inside the decode step, though faster
// alone; above it they gain 5-7% (batch 8-32, 16k-64k keys).
constexpr int DM_TAIL_MIN = 128;
__host__ __device__ constexpr int dm_cut(int s) { return s == 0 ? 0 : s == 1 ? 75 : s == 2 ? 90 : 100; }
// The last 16 bytes of the decode scratch hold the two tail counters
// (sub-chunks claimed, warps finished; zero between launches: the last warp to
// finish re-arms them); the partials of every decode path start at its front.
constexpr size_t kDecodeCounterFloats = 4;

// Chunk geometry of T tiles over W warps for B*Hk (sequence, kv head) pairs.
struct DmSplit {
  long long T, W;
  bool tail;   // claimed sub-chunks: enough tiles per warp, and few enough ranges per (b, g) for the merge
};
__host__ __device__ inline DmSplit dm_split(long long T, long long W, long long BHk) {
  return DmSplit{T, W, T >= DM_TAIL_MIN * W && BHk * 24 >= W};   // <= 24 ranges (72 pieces) per (b, g)
}
__host__ __device__ inline long long dm_chunks(const DmSplit& s) { return s.tail ? s.W * DM_SUB : s.W; }
// First tile of chunk k (k = dm_chunks gives T).
__device__ __forceinline__ long long dm_chunk_start(const DmSplit& s, long long k) {
  if (!s.tail) return s.T * k / s.W;
  const long long r = k / DM_SUB;
  const int sub = (int)(k - r * DM_SUB);
  const long long a = s.T * r / s.W;
  if (sub == 0) return a;
  return a + (s.T * (r + 1) / s.W - a) * dm_cut(sub) / 100;
}
// Chunk holding tile x < T.
__device__ inline long long dm_chunk_of(const DmSplit& s, long long x) {
  const long long r = ((x + 1) * s.W - 1) / s.T;
  if (!s.tail) return r;
  const long long a = s.T * r / s.W, len = s.T * (r + 1) / s.W - a;
  int sub = 0;
  while (sub < DM_SUB - 1 && a + len * dm_cut(sub + 1) / 100 <= x) ++sub;
  return r * DM_SUB + sub;
}
__device__ __forceinline__ int dm_keys(const int32_t* nkeys, int b, int add, int nmax) {
  return min(nkeys[b] + add, nmax);
}
__device__ __forceinline__ int dm_tiles(int n) { return n > 0 ? (n + DM_KEYS - 1) / DM_KEYS : 0; }

// Sequence lengths as the cursors read them: from shared memory (the CTA's
// prefix table) when B <= DM_SEEK_B, else from global memory.
struct DmLens {
  const int32_t* nkeys;
  int add, nmax, B, Hk;
  const long long* cum;   // [B + 1] tiles before sequence b, or null
  const int* keys;        // [B] keys of sequence b (clamped), or null
  __device__ int n(int b) const { return keys ? keys[b] : dm_keys(nkeys, b, add, nmax); }
};

struct TileCursor {
  int b, g, t;          // sequence, kv head, tile of (b, g)
  int n, nt;            // keys and tiles of sequence b
  long long left;       // tiles left in this warp's range, counting the current one
};

__device__ void tc_seek(TileCursor& c, long long x, long long count, const DmLens& Ls) {
  c.left = count;
  int b = -1;
  long long acc = 0;
  if (Ls.cum) {   // the last sequence whose first tile is at or before x (it holds x: empty ones are skipped)
    int lo = 0, hi = Ls.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (Ls.cum[mid] <= x) lo = mid;
      else hi = mid - 1;
    }
    if (x < Ls.cum[lo + 1]) { b = lo; acc = Ls.cum[lo]; }
  } else {
    for (int bb = 0; bb < Ls.B; ++bb) {
      const long long cnt = (long long)Ls.Hk * dm_tiles(Ls.n(bb));
      if (x < acc + cnt) { b = bb; break; }
      acc += cnt;
    }
  }
  if (b < 0) {
    c.left = 0;
    return;
  }
  const int n = Ls.n(b), nt = dm_tiles(n);
  const int r = (int)(x - acc);
  c.b = b; c.n = n; c.nt = nt; c.g = r / nt; c.t = r - c.g * nt;
}

// Advance one tile; true when the piece (this warp's part of one (b, g)) ended.
__device__ bool tc_next(TileCursor& c, const DmLens& Ls) {
  const bool last_in_range = --c.left <= 0;
  if (++c.t < c.nt) return last_in_range;
  c.t = 0;
  if (++c.g == Ls.Hk) {
    c.g = 0;
    do {
      ++c.b;
      c.n = c.b < Ls.B ? Ls.n(c.b) : 0;
      c.nt = dm_tiles(c.n);
    } while (c.nt == 0 && c.b < Ls.B);
  }
  return true;
}

template <typename T>
__device__ __forceinline__ void dm_load_tile(uint8_t* stage, const T* kc, const T* vc, const TileCursor& c,
                                             int Hk, const KvLayout& L, int lane) {
  const int key0 = c.t * DM_KEYS;
  const int valid = min(DM_KEYS, c.n - key0);
  const size_t row0 = kv_row(L, Hk, c.b, c.g, key0);   // a 32-key tile never crosses a 128-key page
  const T* ks = kc + row0 * 128;
  const T* vs = vc + row0 * 128;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int idx = i * 32 + lane;
    const int r = idx >> 4, ch = idx & 15;
    const bool ok = r < valid;
    const size_t off = (size_t)(ok ? r : 0) * 128 + ch * 8;
    cp_async16(stage + swz(r, ch), ks + off, ok);
    cp_async16(stage + DM_TILE + swz(r, ch), vs + off, ok);
  }
}

// TAIL = false compiles the claims and the seek table out (the launch's size
// bound rules claimed sub-chunks out); with TAIL = true they are used when
// this launch's T calls for them.
template <typename T, bool TAIL>
__global__ void __launch_bounds__(DM_WARPS * 32, 1)
    attn_decode_mma_kernel(const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
                           const int32_t* __restrict__ nkeys, int add_keys, int nmax, float* __restrict__ part,
                           int* __restrict__ counters, int B, int H, int Hk, KvLayout L, float scale_log2,
                           int* status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(128) uint8_t sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = H / Hk;
  uint8_t* ring = sm + warp * DM_STAGES * DM_STAGE;
  long long* s_cum = reinterpret_cast<long long*>(sm + DM_RING);
  int* s_keys = reinterpret_cast<int*>(sm + DM_RING + (DM_SEEK_B + 1) * 8);

  long long total = 0;
  for (int b = 0; b < B; ++b) {
    const int nb = nkeys[b] + add_keys;
    if ((nb < 1 || nb > nmax) && blockIdx.x == 0 && threadIdx.x == 0) set_status(status, LLAMA_ERR_DEVICE_BOUNDS);
    total += (long long)Hk * dm_tiles(dm_keys(nkeys, b, add_keys, nmax));
  }
  const long long W = (long long)gridDim.x * DM_WARPS;
  const int w = blockIdx.x * DM_WARPS + warp;
  DmSplit sp = dm_split(total, W, (long long)B * Hk);
  if (!TAIL) sp.tail = false;   // never taken: the host's bound excludes it
  const bool tail = sp.tail;
  DmLens Ls{nkeys, add_keys, nmax, B, Hk, nullptr, nullptr};
  if (tail && B <= DM_SEEK_B) {   // the prefix table: keys by thread, tile prefix by a scan in warp 0
    for (int b = threadIdx.x; b < B; b += blockDim.x) s_keys[b] = dm_keys(nkeys, b, add_keys, nmax);
    __syncthreads();
    if (warp == 0) {
      long long carry = 0;
      for (int b0 = 0; b0 < B; b0 += 32) {
        const int b = b0 + lane;
        long long v = b < B ? (long long)Hk * dm_tiles(s_keys[b]) : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const long long u = __shfl_up_sync(0xffffffffu, v, off);
          if (lane >= off) v += u;
        }
        if (b < B) s_cum[b + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
      if (lane == 0) s_cum[0] = 0;
    }
    __syncthreads();
    Ls.cum = s_cum;
    Ls.keys = s_keys;
  }
  const long long k_first = tail ? (long long)w * DM_SUB : w;   // the warp's own part of its range
  const long long x0 = dm_chunk_start(sp, k_first), x1 = dm_chunk_start(sp, k_first + 1);
  if (x1 <= x0) return;   // only without a tail (T < W): with one, every range holds >= DM_TAIL_MIN tiles
  const int n_claims = tail ? (DM_SUB - 1) * (int)W : 0;

  TileCursor ld, cp;
  tc_seek(ld, x0, x1 - x0, Ls);
  cp = ld;
  long long k_cp = k_first;         // the consumer's chunk
  long long k_q0 = 0, k_q1 = 0, k_q2 = 0;   // chunks the loader moved on to, not yet reached by the consumer
  int n_q = 0;                              // (it runs at most DM_STAGES - 1 = 2 tiles ahead)
  int pending = 0;                  // lane 0: the claim issued for the loader's next chunk
  bool claimed = false, ld_done = false;
  int issued = 0;
  auto maybe_claim = [&]() {
    if (tail && !claimed && ld.left <= DM_CLAIM_AHEAD) {
      if (lane == 0) pending = atomicAdd(&counters[0], 1);
      claimed = true;
    }
  };
  // one tile into the ring, then step the loader (to its claimed chunk at a chunk's end)
  auto issue = [&]() {
    dm_load_tile(ring + (issued % DM_STAGES) * DM_STAGE, kc, vc, ld, Hk, L, lane);
    ++issued;
    tc_next(ld, Ls);
    if (ld.left > 0) {
      maybe_claim();
      return;
    }
    const int c = tail ? __shfl_sync(0xffffffffu, pending, 0) : 0;
    claimed = false;
    if (!tail || c >= n_claims) {
      ld_done = true;
      return;
    }
    // claim c: sub-chunk 1 + c / W of range c % W
    const long long k = (long long)(c % (int)W) * DM_SUB + 1 + c / (int)W, a = dm_chunk_start(sp, k);
    tc_seek(ld, a, dm_chunk_start(sp, k + 1) - a, Ls);
    if (n_q == 0) k_q0 = k;
    else if (n_q == 1) k_q1 = k;
    else k_q2 = k;
    ++n_q;
    maybe_claim();
  };
  const int row = lane >> 2, tq = lane & 3;   // fragment row (query head within the group), column pair
  const bool real = row < G;
  uint32_t qa[8][2];
  auto load_q = [&](const TileCursor& c) {   // the G query rows of (b, g)
    const T* qr = q + ((size_t)c.b * H + c.g * G + (real ? row : 0)) * 128;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa[ks][0] = real ? *reinterpret_cast<const uint32_t*>(qr + ks * 16 + 2 * tq) : 0u;
      qa[ks][1] = real ? *reinterpret_cast<const uint32_t*>(qr + ks * 16 + 8 + 2 * tq) : 0u;
    }
  };
  // the first piece's query rows before the ring fills, so that they do not
  // queue behind every warp's first K/V tiles
  load_q(cp);
  maybe_claim();
  for (int i = 0; i < DM_STAGES - 1; ++i) {
    if (!ld_done) issue();
    cp_async_commit();
  }

  // Keys and head dims take the 16-row side of mma.m16n8k16 and the (padded)
  // query heads its 8 columns: S^T = K Q^T, then O^T += V^T P^T, 32 products
  // per 32-key tile where query rows padded to 16 would take 64. A thread
  // holds the two query columns 2 tq and 2 tq + 1.
  float oacc[8][4];          // O^T: d = 16 i + row (+8), queries 2 tq, 2 tq + 1
  float m_r[2], l_r[2];
  int consumed = 0;
  bool start = true, first_piece = true;
  for (;;) {
    if (start) {   // new piece: reset the state and fetch the G query rows of (b, g)
      if (!first_piece) load_q(cp);
      first_piece = false;
#pragma unroll
      for (int i = 0; i < 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
      m_r[0] = m_r[1] = -INFINITY;
      l_r[0] = l_r[1] = 0.f;
      start = false;
    }
    if (!ld_done) issue();   // keep DM_STAGES-1 tiles in flight
    cp_async_commit();
    cp_async_wait<DM_STAGES - 1>();
    __syncwarp();
    const uint8_t* st = ring + (consumed % DM_STAGES) * DM_STAGE;
    const uint32_t kb = smem_u32(st), vb = smem_u32(st + DM_TILE);
    const int valid = min(DM_KEYS, cp.n - cp.t * DM_KEYS);
    // S^T = K Q^T: two 16-key row tiles; the Q fragments serve as B as they are
    float s[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) s[mt][0] = s[mt][1] = s[mt][2] = s[mt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int r = mt * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int c = ks * 2 + (lane >> 4);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kb + swz(r, c), a0, a1, a2, a3);
        mma16<T>(s[mt], a0, a1, a2, a3, qa[ks][0], qa[ks][1]);
      }
    }
    // online softmax per query column over the tile's keys (rows row, row + 8
    // of both row tiles here; the other rows sit in lanes row' = lane >> 2)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int kk = mt * 16 + row + ((i >> 1) << 3);
        const float v = kk < valid ? s[mt][i] * scale_log2 : -INFINITY;
        s[mt][i] = v;
        mx[i & 1] = fmaxf(mx[i & 1], v);
      }
    }
    float corr[2], ls[2] = {0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], off));
      const float mnew = fmaxf(m_r[e], mx[e]);
      corr[e] = exp2f(m_r[e] - mnew);
      m_r[e] = mnew;
    }
    // P^T as B fragments: each packed pair is a row of an 8x8 block (keys x
    // queries) that movmatrix turns into the block's transpose
    uint32_t pb[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float p0 = exp2f(s[mt][2 * h] - m_r[0]), p1 = exp2f(s[mt][2 * h + 1] - m_r[1]);
        ls[0] += p0;
        ls[1] += p1;
        const uint32_t pk = pack2<T>(p0, p1);
        asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(pb[mt][h]) : "r"(pk));
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) ls[e] += __shfl_xor_sync(0xffffffffu, ls[e], off);
      l_r[e] = l_r[e] * corr[e] + ls[e];
    }
    // O^T = O^T corr + V^T P^T: eight 16-dim row tiles, two 16-key steps
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      oacc[i][0] *= corr[0]; oacc[i][1] *= corr[1];
      oacc[i][2] *= corr[0]; oacc[i][3] *= corr[1];
    }
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = kt * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int c = i * 2 + ((lane >> 3) & 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vb + swz(r, c), a0, a1, a2, a3);
        mma16<T>(oacc[i], a0, a1, a2, a3, pb[kt][0], pb[kt][1]);
      }
    }
    __syncwarp();   // the stage may be refilled from the next iteration on
    ++consumed;
    const int b_done = cp.b, g_done = cp.g;
    if (tc_next(cp, Ls)) {
      const size_t slot = (size_t)b_done * Hk + g_done + k_cp;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int qh = 2 * tq + e;   // query head within the group
        if (qh < G) {
          float* dst = part + (slot * G + qh) * 130;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            dst[i * 16 + row] = oacc[i][e];
            dst[i * 16 + row + 8] = oacc[i][2 + e];
          }
          if (row == 0) { dst[128] = m_r[e]; dst[129] = l_r[e]; }
        }
      }
      start = true;
      if (cp.left <= 0) {   // the chunk is done: on to the next one the loader reached, if any
        if (n_q == 0) break;
        k_cp = k_q0;
        k_q0 = k_q1;
        k_q1 = k_q2;
        --n_q;
        const long long a = dm_chunk_start(sp, k_cp);
        tc_seek(cp, a, dm_chunk_start(sp, k_cp + 1) - a, Ls);
      }
    }
  }
  cp_async_wait<0>();
  if (tail && lane == 0) {   // every warp has made its last claim: the last one out re-arms the counters
    __threadfence();
    if (atomicAdd(&counters[1], 1) == (int)W - 1) {
      counters[0] = 0;
      counters[1] = 0;
    }
  }
}

// Merge the pieces of every (b, h). The chunks holding tiles of (b, g) are
// chunk(t0) .. chunk(t0 + nt - 1): when every range holds tiles (T >= W;
// claimed sub-chunks then always do) these are every chunk between the two;
// otherwise (T < W, no claimed sub-chunks) every warp holds at most one tile,
// so piece k is the warp of tile t0 + k. A block of CW warps serves CW / wh
// heads (flattened b*H + h), wh warps each: warp j of a head merges its pieces
// [cnt j / wh, cnt (j+1) / wh), loading CB pieces at a time with every load in
// flight and keeping a running (max, sum, o) rescaled as the maximum grows;
// the wh warps' results are then merged in warp order. The order is fixed, so
// results do not depend on timing. wh (1, 2, 4 or 8) and CB are chosen on
// the host from the pieces a head is expected to have: many pieces per head
// when B * Hk is small, few when it is large (a smaller CB then holds fewer
// registers, leaving room on the SM for the next kernel's early blocks).
constexpr int CW = 8;        // warps of a combine block
constexpr int CB_MAX = 12;   // pieces a warp loads per round, at most

template <typename T, int D, int CB>
__global__ void __launch_bounds__(CW * 32) attn_decode_combine_pieces_kernel(
    const float* __restrict__ part, const int32_t* __restrict__ nkeys, int add_keys, int nmax, T* __restrict__ o,
    int B, int H, int Hk, long long W, int wh) {
  static_assert(D == 128, "one 4-dim slice per lane");
  pdl_trigger();
  pdl_wait();
  __shared__ float s_mq[CW], s_lq[CW];
  __shared__ float s_acc[CW][D];
  __shared__ int s_bad[CW];
  const int q = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hpb = CW / wh;   // heads per block
  const long long bh = (long long)blockIdx.x * hpb + q / wh;
  const int j = q % wh;
  const int G = H / Hk;
  float M = -INFINITY, L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (bh < (long long)B * H) {
    const int b = (int)(bh / H), h = (int)(bh - (long long)b * H);
    const int g = h / G, row = h - g * G;
    // T and the tiles of the sequences before b, the lengths loaded 32 at a time
    long long total = 0, t0 = 0;
    for (int bb = lane; bb < B; bb += 32) {
      const long long c = (long long)Hk * dm_tiles(dm_keys(nkeys, bb, add_keys, nmax));
      total += c;
      if (bb < b) t0 += c;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      total += __shfl_xor_sync(0xffffffffu, total, off);
      t0 += __shfl_xor_sync(0xffffffffu, t0, off);
    }
    const int nb = nkeys[b] + add_keys;
    const int nt_b = dm_tiles(dm_keys(nkeys, b, add_keys, nmax));
    t0 += (long long)g * nt_b;
    // no keys, or more keys than the cache holds (clamped for the other
    // sequences' sake, latched by the decode kernel): NaN rows, as the split path
    const bool bad = nt_b == 0 || total == 0 || nb < 1 || nb > nmax;
    if (j == 0 && lane == 0) s_bad[q / wh] = bad;
    if (!bad) {
      const DmSplit sp = dm_split(total, W, (long long)B * Hk);
      const long long w_lo = dm_chunk_of(sp, t0);
      const bool dense = total >= W;
      const int cnt = dense ? (int)(dm_chunk_of(sp, t0 + nt_b - 1) - w_lo + 1) : nt_b;
      const size_t bg = (size_t)b * Hk + g;
      const int k0 = cnt * j / wh, k1 = cnt * (j + 1) / wh;
      for (int kb = k0; kb < k1; kb += CB) {
        float2 a[CB], c[CB], ml[CB];   // rows are D + 2 floats apart: 8-byte aligned
#pragma unroll
        for (int u = 0; u < CB; ++u) {
          if (kb + u < k1) {
            const long long k = kb + u;
            const long long w = dense ? w_lo + k : ((t0 + k + 1) * W - 1) / total;
            const float* r = part + ((bg + w) * G + row) * (D + 2);
            a[u] = *reinterpret_cast<const float2*>(r + 4 * lane);
            c[u] = *reinterpret_cast<const float2*>(r + 4 * lane + 2);
            ml[u] = *reinterpret_cast<const float2*>(r + D);
          } else {
            a[u] = c[u] = make_float2(0.f, 0.f);
            ml[u] = make_float2(-INFINITY, 0.f);
          }
        }
        float Mc = M;
#pragma unroll
        for (int u = 0; u < CB; ++u) Mc = fmaxf(Mc, ml[u].x);
        const float s = M == -INFINITY ? 0.f : exp2f(M - Mc);
        L *= s;
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] *= s;
#pragma unroll
        for (int u = 0; u < CB; ++u) {
          const float f = exp2f(ml[u].x - Mc);   // 0 for the padding
          L += ml[u].y * f;
          acc[0] += a[u].x * f;
          acc[1] += a[u].y * f;
          acc[2] += c[u].x * f;
          acc[3] += c[u].y * f;
        }
        M = Mc;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) s_acc[q][4 * lane + i] = acc[i];
  if (lane == 0) { s_mq[q] = M; s_lq[q] = L; }
  __syncthreads();
  for (int idx = threadIdx.x; idx < hpb * D; idx += blockDim.x) {
    const int hh = idx / D, dd = idx - hh * D;
    const long long bh2 = (long long)blockIdx.x * hpb + hh;
    if (bh2 >= (long long)B * H) break;
    float r;
    if (s_bad[hh]) {
      r = NAN;
    } else {
      const int q0 = hh * wh;
      float Mt = -INFINITY;
      for (int i = 0; i < wh; ++i) Mt = fmaxf(Mt, s_mq[q0 + i]);
      float O = 0.f, Lt = 0.f;
      for (int i = 0; i < wh; ++i) {
        const float wq = s_mq[q0 + i] == -INFINITY ? 0.f : exp2f(s_mq[q0 + i] - Mt);   // a warp without pieces weighs nothing
        Lt += s_lq[q0 + i] * wq;
        O += s_acc[q0 + i][dd] * wq;
      }
      r = O / Lt;
    }
    o[bh2 * D + dd] = from_f<T>(r);
  }
}

template <typename T, int D>
int decode_launch(const void* q, const void* kc, const void* vc, const int32_t* nkeys, int add_keys, void* o, int B,
                  int cmax, int H, int Hk, int Smax, float* part, int splits, int* status, cudaStream_t st) {
  constexpr int ROW = D * (int)sizeof(T);
  constexpr int DEC_SUB = dec_sub<T, D>();
  constexpr int SMEM = DEC_STAGES * 2 * DEC_SUB * ROW + DEC_STAGES * 8 + 4 * DEC_MAXG * (D + 2) * 4;
  auto kern = attn_decode_part_kernel<T, D>;
  if (const int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), SMEM)) return rc;
  int chunk = (cmax + splits - 1) / splits;
  chunk = (chunk + 127) / 128 * 128;
  const float scale_log2 = kLog2e / sqrtf((float)D);
  count_launches(2);
  kern<<<dim3(splits, Hk, B), 128, SMEM, st>>>(static_cast<const T*>(q), static_cast<const T*>(kc),
                                               static_cast<const T*>(vc), nkeys, add_keys, part, H, Hk, Smax, chunk,
                                               scale_log2, status);
  attn_decode_combine_kernel<T, D><<<dim3(H, B), D < 128 ? D : 128, 0, st>>>(part, static_cast<T*>(o), H, splits);
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

}  // namespace

int attention_prefill(const void* q, const void* kc, const void* vc, void* o, const int32_t* pos0, int B, int S,
                      int H, int Hk, int d, int Smax, int dtype, int* status, cudaStream_t st, const int32_t* kv_table,
                      int kv_max_pages, int kv_pages) {
  (void)status;
  if (B <= 0 || S <= 0) return LLAMA_OK;
  if (H % Hk != 0) return LLAMA_ERR_SHAPE;
  const float scale_log2 = kLog2e / sqrtf((float)d);
  if (dtype == LLAMA_BF16 || dtype == LLAMA_F16) {
    if (d != 128) return LLAMA_ERR_UNSUPPORTED;
    return attention_prefill_tc(q, kc, vc, o, pos0, B, S, H, Hk, Smax, dtype, status, st, kv_table, kv_max_pages,
                                kv_pages);
  } else {
    if (kv_table) return LLAMA_ERR_UNSUPPORTED;   // paged caches: 16-bit, head_dim 128 only
    dim3 grid(S, H, B);
    count_launches(1);
#define LLAMA_F32_PREFILL(DD)                                                                                  \
  attn_prefill_f32_kernel<DD><<<grid, 32, 0, st>>>(static_cast<const float*>(q), static_cast<const float*>(kc), \
                                                   static_cast<const float*>(vc), static_cast<float*>(o), pos0, S, \
                                                   H, Hk, Smax, scale_log2)
    switch (d) {
      case 32: LLAMA_F32_PREFILL(32); break;
      case 64: LLAMA_F32_PREFILL(64); break;
      case 128: LLAMA_F32_PREFILL(128); break;
      default: return LLAMA_ERR_UNSUPPORTED;
    }
#undef LLAMA_F32_PREFILL
  }
  return cudaGetLastError() == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

namespace {
int decode_splits(int cmax, int B, int Hk) {
  const int target = 2 * num_sms();
  int s = (target + B * Hk - 1) / (B * Hk);
  const int max_s = (cmax + 511) / 512;  // at least ~512 keys per split
  if (s > max_s) s = max_s;
  return s < 1 ? 1 : s;
}

bool use_mma_decode(int d, int dtype) { return (dtype == LLAMA_BF16 || dtype == LLAMA_F16) && d == 128; }
}  // namespace

namespace {
// Chunk geometry of a launch whose sequences hold at most cmax keys (claimed
// sub-chunks only come in as T grows, so this bounds every launch within cmax).
DmSplit decode_split_bound(int cmax, int B, int Hk) {
  const long long T = (long long)B * Hk * ((cmax + DM_KEYS - 1) / DM_KEYS);
  return dm_split(T, (long long)num_sms() * DM_WARPS, (long long)B * Hk);
}
}  // namespace

size_t decode_scratch_floats(int cmax, int B, int H, int Hk, int d, int dtype) {
  if (use_mma_decode(d, dtype))
    return kDecodeCounterFloats +
           ((size_t)B * Hk + (size_t)dm_chunks(decode_split_bound(cmax, B, Hk))) * (H / Hk) * (d + 2);
  return kDecodeCounterFloats + (size_t)B * H * decode_splits(cmax, B, Hk) * (d + 2);
}

template <typename T>
static int mma_decode_launch(const void* q, const void* kc, const void* vc, const int32_t* nkeys, int add_keys,
                             void* o, int B, int cmax, int H, int Hk, int Smax, const KvLayout& L,
                             DecodeScratch* scratch, int* status, cudaStream_t st) {
  const int grid = num_sms();
  const float scale_log2 = kLog2e / sqrtf(128.f);
  const int nmax = cmax < Smax ? cmax : Smax;
  const DmSplit bound = decode_split_bound(nmax, B, Hk);
  auto kern = bound.tail ? attn_decode_mma_kernel<T, true> : attn_decode_mma_kernel<T, false>;
  if (const int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), bound.tail ? DM_SMEM : DM_RING)) return rc;
  // warps per head of the combine: enough that each loads about CB_MAX pieces
  const long long W = (long long)grid * DM_WARPS;
  long long pieces = dm_chunks(bound) / ((long long)B * Hk) + (bound.tail ? DM_SUB + 1 : 2);
  const long long tiles = (nmax + DM_KEYS - 1) / DM_KEYS;
  if (!bound.tail && pieces > tiles) pieces = tiles;
  int wh = 1;
  while (wh < CW && (long long)wh * CB_MAX < pieces) wh *= 2;
  auto combine = pieces <= 6 ? attn_decode_combine_pieces_kernel<T, 128, 6>
                             : attn_decode_combine_pieces_kernel<T, 128, CB_MAX>;
  int* counters = reinterpret_cast<int*>(scratch->part + scratch->floats - kDecodeCounterFloats);
  float* part = scratch->part;
  // the seek table's shared memory only where claimed sub-chunks may be used
  cudaError_t err = launch_k(kern, dim3(grid), dim3(DM_WARPS * 32), bound.tail ? DM_SMEM : DM_RING, st,
                             static_cast<const T*>(q), static_cast<const T*>(kc), static_cast<const T*>(vc), nkeys,
                             add_keys, nmax, part, counters, B, H, Hk, L, scale_log2, status);
  if (err == cudaSuccess)
    err = launch_k(combine, dim3((unsigned)((B * H + CW / wh - 1) / (CW / wh))), dim3(CW * 32), 0, st,
                   (const float*)part, nkeys, add_keys, nmax, static_cast<T*>(o), B, H, Hk, W, wh);
  return err == cudaSuccess ? LLAMA_OK : LLAMA_ERR_CUDA;
}

int attention_decode(const void* q, const void* kc, const void* vc, const int32_t* nkeys, int add_keys, void* o,
                     int B, int cmax, int H, int Hk, int d, int Smax, int dtype, DecodeScratch* scratch, int* status,
                     cudaStream_t st, const int32_t* kv_table, int kv_max_pages, int kv_pages) {
  if (B <= 0) return LLAMA_OK;
  if (H % Hk != 0 || H / Hk > DEC_MAXG) return LLAMA_ERR_SHAPE;
  if (!scratch || !scratch->part || scratch->floats < decode_scratch_floats(cmax, B, H, Hk, d, dtype))
    return LLAMA_ERR_INVALID_ARG;
  const KvLayout L{kv_table, kv_max_pages, Smax, kv_pages};
  if (use_mma_decode(d, dtype)) {
    if (dtype == LLAMA_F16)
      return mma_decode_launch<f16>(q, kc, vc, nkeys, add_keys, o, B, cmax, H, Hk, Smax, L, scratch, status, st);
    return mma_decode_launch<bf16>(q, kc, vc, nkeys, add_keys, o, B, cmax, H, Hk, Smax, L, scratch, status, st);
  }
  if (kv_table) return LLAMA_ERR_UNSUPPORTED;   // paged caches: 16-bit, head_dim 128 only
  const int splits = decode_splits(cmax, B, Hk);
  float* part = scratch->part;
  if (dtype == LLAMA_BF16) {
    if (d == 64) return decode_launch<bf16, 64>(q, kc, vc, nkeys, add_keys, o, B, cmax, H, Hk, Smax, part,
                                                splits, status, st);
  } else if (dtype == LLAMA_F16) {
    if (d == 64) return decode_launch<f16, 64>(q, kc, vc, nkeys, add_keys, o, B, cmax, H, Hk, Smax, part,
                                               splits, status, st);
  } else {
    if (d == 128) return decode_launch<float, 128>(q, kc, vc, nkeys, add_keys, o, B, cmax, H, Hk, Smax,
                                                   part, splits, status, st);
    if (d == 64) return decode_launch<float, 64>(q, kc, vc, nkeys, add_keys, o, B, cmax, H, Hk, Smax, part,
                                                 splits, status, st);
    if (d == 32) return decode_launch<float, 32>(q, kc, vc, nkeys, add_keys, o, B, cmax, H, Hk, Smax, part,
                                                 splits, status, st);
  }
  return LLAMA_ERR_UNSUPPORTED;
}

}  // namespace llama
