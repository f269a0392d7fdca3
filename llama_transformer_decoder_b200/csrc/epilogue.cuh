// GEMM epilogues shared by the tcgen05 GEMMs and the fp32 SIMT GEMM.
//
// A GEMM computes acc[m][n] = sum_k A[m][k] * W[n][k] (y = x W^T, the [out, in]
// weight convention of the checkpoint). The epilogue turns acc into one of:
//   STORE_F32  out[m][n] = acc                      (LM-head logits, tests)
//   RESIDUAL   out[m][n] += acc                     (Wo and w2: h = x + delta)
//   SWIGLU     g[m][f] = silu(acc[m][2f]) * acc[m][2f+1]
//              (w1 and w3 rows are interleaved: row 2f = w1[f], 2f+1 = w3[f])
//   QKV_ROPE   columns [0,H*d) are q, [H*d,(H+Hk)*d) k, then v. Adjacent
//              pairs of q and k are rotated by angle pos*theta^(-2i/d); q goes
//              to q_out[b][h][s][:], k and v into the KV cache at pos.
#pragma once
#include "common.cuh"

namespace llama {

enum EpiKind { EPI_STORE_F32 = 0, EPI_RESIDUAL = 1, EPI_SWIGLU = 2, EPI_QKV_ROPE = 3 };

struct EpiArgs {
  int M, N;           // logical output extent (rows = tokens, columns = features)
  float* out;         // STORE_F32 / RESIDUAL target, row pitch ldo (floats)
  int ldo;
  void* g;            // SWIGLU output (T = model dtype), row pitch ldg
  int ldg;
  void* q;            // QKV_ROPE: q output [B][H][S][d]
  void* kc;           // K cache of this layer: [Bmax][Hk][Smax][d], or paged [pages][Hk][128][d]
  void* vc;           // V cache of this layer
  const float2* rope; // (cos, sin) table [Smax][d/2]
  const int* pos0;    // per-sequence position of the call's first token
  int S, H, Hk, d, Smax;
  const int32_t* kv_table;  // paged cache block table (nullptr: contiguous)
  int kv_max_pages, kv_pages;
  // RMSNorm folded into the GEMMs around it (prefill): rmsnorm(x) W^T equals
  // r * ((x * g) W^T) with r = rsqrt(mean(x^2) + eps) per row. A RESIDUAL
  // epilogue with g_next also writes y = x_new * g_next (16-bit, row pitch
  // ldo) to y_out and the sum of x_new^2 over its 256-column tile to
  // ss_out[m * ss_n + n0 / 256]; a QKV or SwiGLU epilogue with ss_in scales
  // its accumulators by r = rsqrt(sum_t ss_in[m * ss_n + t] * norm_inv_d + norm_eps).
  const float* g_next;
  void* y_out;
  float* ss_out;
  const float* ss_in;
  int ss_n;
  float norm_inv_d, norm_eps;
  // Status word for LLAMA_ERR_RANGE: a 16-bit output (q/k/v, the SwiGLU
  // product, y = x * g) that is not finite after rounding (nullptr: unchecked).
  int* status;
};

// One GEMM of a chain of CTA-pair GEMMs run by one persistent launch
// (gemm16_chain): acc = A W^T with A [M][K] (row pitch lda), W [N][K] (ldw),
// epilogue `kind` with `epi`. Tiles are taken in groups of m_group 256-row
// blocks (column by column inside a group; 0 = all blocks in one group).
// With `ready`, every CTA adds 1 to ready[r] once it has written the 128
// output rows r*128 .. r*128+127 of a tile (zero before the launch). A job
// with dep = d reads rows that job d writes: before touching rows of block r
// it waits until job d has published all of its column tiles of r.
struct ChainJobDesc {
  const void* A;
  int lda;
  const void* W;
  int ldw;
  int M, N, K, kind, m_group, dep;
  int* ready;
  EpiArgs epi;
};

// r of row m from its partial sums of squares (added in a fixed order).
__device__ __forceinline__ float norm_row_scale(const EpiArgs& e, int m) {
  const float* p = e.ss_in + (size_t)m * e.ss_n;
  float t = 0.f;
  for (int i = 0; i < e.ss_n; ++i) t += p[i];
  return rsqrtf(t * e.norm_inv_d + e.norm_eps);
}

// Element offset of (sequence b, kv head g, position pos, dim 0) in a K/V cache.
__device__ __forceinline__ size_t kv_elem(const EpiArgs& e, int b, int g, int pos) {
  const KvLayout L{e.kv_table, e.kv_max_pages, e.Smax, e.kv_pages};
  return kv_row(L, e.Hk, b, g, pos) * (size_t)e.d;
}

// One rotated (or plain) value of the q/k/v block. n is the column, v its
// accumulator and partner the accumulator of column n^1.
template <typename T>
__device__ __forceinline__ void qkv_store(const EpiArgs& e, int m, int n, float v, float partner) {
  const int b = m / e.S, s = m - b * e.S;
  const int pos = e.pos0[b] + s;
  const int hd = e.H * e.d;
  float r = v;
  if (n < hd + e.Hk * e.d) {
    const int i = (n % e.d) >> 1;
    const float2 cs = e.rope[(size_t)pos * (e.d >> 1) + i];
    r = (n & 1) ? (partner * cs.y + v * cs.x) : (v * cs.x - partner * cs.y);
  }
  if (nonfinite16<T>(r)) set_status(e.status, LLAMA_ERR_RANGE);
  if (n < hd) {
    const int h = n / e.d, dd = n - h * e.d;
    static_cast<T*>(e.q)[(((size_t)b * e.H + h) * e.S + s) * e.d + dd] = from_f<T>(r);
  } else {
    const bool is_k = n < hd + e.Hk * e.d;
    const int nn = n - hd - (is_k ? 0 : e.Hk * e.d);
    const int g = nn / e.d, dd = nn - g * e.d;
    T* dst = static_cast<T*>(is_k ? e.kc : e.vc);
    dst[kv_elem(e, b, g, pos) + dd] = from_f<T>(r);
  }
}

// Element-wise form (used when consecutive columns live in neighbouring lanes).
template <int KIND, typename T>
__device__ __forceinline__ void epi_elem(const EpiArgs& e, int m, int n, float v, float partner) {
  if (m >= e.M || n >= e.N) return;
  if (KIND == EPI_STORE_F32) {
    e.out[(size_t)m * e.ldo + n] = v;
  } else if (KIND == EPI_RESIDUAL) {
    float* p = e.out + (size_t)m * e.ldo + n;
    *p = *p + v;
  } else if (KIND == EPI_SWIGLU) {
    if ((n & 1) == 0) {
      const float r = silu_f(v) * partner;
      if (nonfinite16<T>(r)) set_status(e.status, LLAMA_ERR_RANGE);
      static_cast<T*>(e.g)[(size_t)m * e.ldg + (n >> 1)] = from_f<T>(r);
    }
  } else {
    qkv_store<T>(e, m, n, v, partner);
  }
}

// Row-chunk form: one thread holds 32 consecutive columns [n0, n0+32) of row m
// (n0 % 32 == 0). Full chunks use 16-byte stores. rs scales the accumulators
// (the folded RMSNorm's r; 1 otherwise). Returns the chunk's sum of x_new^2
// for a RESIDUAL epilogue with g_next, else 0.
template <int KIND, typename T>
__device__ __forceinline__ float epi_row32(const EpiArgs& e, int m, int n0, const float (&v)[32], float rs = 1.f) {
  if (m >= e.M) return 0.f;
  const bool full = (n0 + 32 <= e.N);
  float ssq = 0.f;
  bool bad = false;   // a 16-bit output of this chunk is not finite
  if (KIND == EPI_STORE_F32 || KIND == EPI_RESIDUAL) {
    const bool norm_out = KIND == EPI_RESIDUAL && e.g_next != nullptr;
    float* p = e.out + (size_t)m * e.ldo + n0;
    T* yp = norm_out ? static_cast<T*>(e.y_out) + (size_t)m * e.ldo + n0 : nullptr;
    if (full && ((e.ldo & 3) == 0) && ((reinterpret_cast<uintptr_t>(e.out) & 15) == 0) &&
        (!norm_out || (sizeof(T) == 2 && (e.ldo & 7) == 0))) {
      float4* p4 = reinterpret_cast<float4*>(p);
      float4 x[8];
      if (KIND == EPI_RESIDUAL) {  // all loads before any store: they do not wait on one another
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = p4[j];
      }
      uint32_t yw[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 o = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        if (KIND == EPI_RESIDUAL) { o.x += x[j].x; o.y += x[j].y; o.z += x[j].z; o.w += x[j].w; }
        p4[j] = o;
        if (norm_out) {
          const float4 gg = __ldg(reinterpret_cast<const float4*>(e.g_next + n0) + j);
          ssq += o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
          yw[2 * j] = pack2<T>(o.x * gg.x, o.y * gg.y);
          yw[2 * j + 1] = pack2<T>(o.z * gg.z, o.w * gg.w);
        }
      }
      if (norm_out) {
        uint4* y4 = reinterpret_cast<uint4*>(yp);
#pragma unroll
        for (int j = 0; j < 4; ++j) y4[j] = make_uint4(yw[4 * j], yw[4 * j + 1], yw[4 * j + 2], yw[4 * j + 3]);
        if (sizeof(T) == 2) {
#pragma unroll
          for (int j = 0; j < 16; ++j) bad |= packed_nonfinite<T>(yw[j]);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (n0 + j < e.N) {
          if (KIND == EPI_RESIDUAL) p[j] += v[j];
          else p[j] = v[j];
          if (norm_out) {
            ssq += p[j] * p[j];
            const float y = p[j] * e.g_next[n0 + j];
            bad |= nonfinite16<T>(y);
            yp[j] = from_f<T>(y);
          }
        }
      }
    }
  } else if (KIND == EPI_SWIGLU) {
    T* p = static_cast<T*>(e.g) + (size_t)m * e.ldg + (n0 >> 1);
    if (sizeof(T) == 2 && full && ((e.ldg & 7) == 0)) {
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        w[j] = pack2<T>(silu_f(rs * v[4 * j]) * (rs * v[4 * j + 1]), silu_f(rs * v[4 * j + 2]) * (rs * v[4 * j + 3]));
      uint4* p4 = reinterpret_cast<uint4*>(p);
      p4[0] = make_uint4(w[0], w[1], w[2], w[3]);
      p4[1] = make_uint4(w[4], w[5], w[6], w[7]);
#pragma unroll
      for (int j = 0; j < 8; ++j) bad |= packed_nonfinite<T>(w[j]);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (n0 + 2 * j + 1 < e.N) {
          const float r = silu_f(rs * v[2 * j]) * (rs * v[2 * j + 1]);
          bad |= nonfinite16<T>(r);
          p[j] = from_f<T>(r);
        }
    }
  } else {  // QKV_ROPE: a 32-column chunk never straddles a head when d % 32 == 0
    if (!full || (e.d & 31) != 0 || sizeof(T) != 2) {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (n0 + j < e.N) qkv_store<T>(e, m, n0 + j, rs * v[j], rs * v[j ^ 1]);
      return 0.f;
    }
    const int b = m / e.S, s = m - b * e.S;
    const int pos = e.pos0[b] + s;
    const int hd = e.H * e.d;
    T* dst;
    int dd0;
    float r[32];
    if (n0 < hd + e.Hk * e.d) {
      const float2* cs = e.rope + (size_t)pos * (e.d >> 1) + ((n0 % e.d) >> 1);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 c = cs[j];
        const float a = rs * v[2 * j], b = rs * v[2 * j + 1];
        r[2 * j] = a * c.x - b * c.y;
        r[2 * j + 1] = a * c.y + b * c.x;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = rs * v[j];
    }
    if (n0 < hd) {
      const int h = n0 / e.d;
      dd0 = n0 - h * e.d;
      dst = static_cast<T*>(e.q) + (((size_t)b * e.H + h) * e.S + s) * e.d + dd0;
    } else {
      const bool is_k = n0 < hd + e.Hk * e.d;
      const int nn = n0 - hd - (is_k ? 0 : e.Hk * e.d);
      const int g = nn / e.d;
      dd0 = nn - g * e.d;
      dst = static_cast<T*>(is_k ? e.kc : e.vc) + kv_elem(e, b, g, pos) + dd0;
    }
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = pack2<T>(r[2 * j], r[2 * j + 1]);
    uint4* p4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int j = 0; j < 4; ++j) p4[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
#pragma unroll
    for (int j = 0; j < 16; ++j) bad |= packed_nonfinite<T>(w[j]);
  }
  if (bad) set_status(e.status, LLAMA_ERR_RANGE);
  return ssq;
}

}  // namespace llama
