// Causal grouped-query flash attention, forward and backward, for the
// decoder layer's attention step (head_dim 64 or 128).
//
// The score and value contractions run on the tensor cores through
// mma.sync.m16n8k16 (bf16 in, fp32 accumulate) with ldmatrix fragment loads
// from XOR-swizzled shared-memory tiles; softmax statistics stay in
// registers (online softmax, log2 domain). Nothing of size T x T is stored.
//
// The backward is deterministic: one kernel computes dQ per query block
// (looping over key blocks), another computes dK and dV per key block,
// looping over the query heads of its group in a fixed order and over the
// query blocks at or after the diagonal. No atomics are used.
#include <cstdlib>
#include <mutex>
#include <string>

#include "mt_internal.h"

namespace mt {

mt_status attn_bwd_tc_launch(const mt_bf16* qkv, int64_t ld, const mt_bf16* d_o, int64_t ld_o, const float* lse,
                             const float* delta, mt_bf16* dqkv, int B, int T, int nq, int nkv, const float* rope_tab,
                             cudaStream_t st);

namespace {

constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of 16-byte chunk `ch` of row `r` in a [rows][D] bf16 tile.
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return static_cast<uint32_t>(r * (D * 2) + ((ch ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Loads `rows` rows x D columns (bf16) starting at token row `t0` of a
// sequence into a swizzled tile; rows at or past T are zero-filled.
template <int D, int NT>
__device__ __forceinline__ void load_tile(uint8_t* tile, const __nv_bfloat16* base, int64_t ld, int t0, int T,
                                          int rows) {
  constexpr int CH = D / 8;
  const uint32_t s = smem_u32(tile);
  for (int id = threadIdx.x; id < rows * CH; id += NT) {
    const int r = id / CH, ch = id % CH;
    const int t = t0 + r;
    const bool valid = t < T;
    const __nv_bfloat16* src = base + static_cast<int64_t>(valid ? t : 0) * ld + ch * 8;
    cp_async16(s + swz<D>(r, ch), src, valid);
  }
}

// A fragment (16 x 16) of rows [r0, r0+16), k-step kk, from a row-major tile.
template <int D>
__device__ __forceinline__ void lda_frag(const uint8_t* tile, int r0, int kk, uint32_t (&a)[4]) {
  const int lane = threadIdx.x & 31, mat = lane >> 3;
  const int r = r0 + (lane & 7) + (mat & 1) * 8;
  const int ch = kk * 2 + (mat >> 1);
  ldsm_x4(smem_u32(tile) + swz<D>(r, ch), a);
}

// B fragments of two n8 tiles (rows n0..n0+15 of a [n][k] tile), k-step kk:
// b[0], b[1] for rows n0..n0+7 and b[2], b[3] for rows n0+8..n0+15.
template <int D>
__device__ __forceinline__ void ldb_frag(const uint8_t* tile, int n0, int kk, uint32_t (&b)[4]) {
  const int lane = threadIdx.x & 31, mat = lane >> 3;
  const int r = n0 + (lane & 7) + (mat >> 1) * 8;
  const int ch = kk * 2 + (mat & 1);
  ldsm_x4(smem_u32(tile) + swz<D>(r, ch), b);
}

// B fragments of two n8 tiles (columns c0..c0+15 of a [k][n] tile), k rows
// k0..k0+15: b[0], b[1] for columns c0..c0+7 and b[2], b[3] for c0+8..c0+15.
template <int D>
__device__ __forceinline__ void ldb_frag_t(const uint8_t* tile, int k0, int c0, uint32_t (&b)[4]) {
  const int lane = threadIdx.x & 31, mat = lane >> 3;
  const int r = k0 + (lane & 7) + (mat & 1) * 8;
  const int ch = c0 / 8 + (mat >> 1);
  ldsm_x4_t(smem_u32(tile) + swz<D>(r, ch), b);
}

// ============================================================== forward
template <int D>
struct FwdCfg {
  static constexpr int BQ = 128, BKV = 64, WARPS = 8, NT = WARPS * 32;
  static constexpr int TILE_Q = BQ * D * 2, TILE_KV = BKV * D * 2;
  static constexpr int SMEM = TILE_Q + 4 * TILE_KV;
};

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::NT, 1)
    attn_fwd_kernel(const __nv_bfloat16* __restrict__ qkv, int64_t ld, __nv_bfloat16* __restrict__ o, int64_t ld_o,
                    float* __restrict__ lse, int T, int nq, int nkv, float scale_log2) {
  using C = FwdCfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::TILE_Q;
  uint8_t* sV = sK + 2 * C::TILE_KV;

  const int qb = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int c = (h * nkv) / nq;
  const int q0 = qb * C::BQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int r0 = warp * 16;

  const int64_t seq = static_cast<int64_t>(b) * T;
  const __nv_bfloat16* Qb = qkv + seq * ld + h * D;
  const __nv_bfloat16* Kb = qkv + seq * ld + static_cast<int64_t>(nq) * D + c * D;
  const __nv_bfloat16* Vb = qkv + seq * ld + static_cast<int64_t>(nq + nkv) * D + c * D;

  const int n_kv = min((T + C::BKV - 1) / C::BKV, (q0 + C::BQ + C::BKV - 1) / C::BKV);

  load_tile<D, C::NT>(sQ, Qb, ld, q0, T, C::BQ);
  load_tile<D, C::NT>(sK, Kb, ld, 0, T, C::BKV);
  load_tile<D, C::NT>(sV, Vb, ld, 0, T, C::BKV);
  cp_commit();

  float acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  uint32_t qf[D / 16][4];

  const int row_a = q0 + r0 + g, row_b = row_a + 8;

  for (int j = 0; j < n_kv; ++j) {
    if (j + 1 < n_kv) {
      const int nb = (j + 1) & 1;
      load_tile<D, C::NT>(sK + nb * C::TILE_KV, Kb, ld, (j + 1) * C::BKV, T, C::BKV);
      load_tile<D, C::NT>(sV + nb * C::TILE_KV, Vb, ld, (j + 1) * C::BKV, T, C::BKV);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) lda_frag<D>(sQ, r0, kk, qf[kk]);
    }
    const uint8_t* tK = sK + (j & 1) * C::TILE_KV;
    const uint8_t* tV = sV + (j & 1) * C::TILE_KV;
    const int k0 = j * C::BKV;

    float s[C::BKV / 8][4];
#pragma unroll
    for (int i = 0; i < C::BKV / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < C::BKV / 16; ++np) {
        uint32_t bb[4];
        ldb_frag<D>(tK, np * 16, kk, bb);
        mma16816(s[2 * np], qf[kk], bb[0], bb[1]);
        mma16816(s[2 * np + 1], qf[kk], bb[2], bb[3]);
      }
    }
    const bool need_mask = k0 + C::BKV - 1 > q0 + r0;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < C::BKV / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = s[nt][e] * scale_log2;
        if (need_mask) {
          const int col = k0 + nt * 8 + 2 * tq + (e & 1);
          const int row = (e < 2) ? row_a : row_b;
          if (col > row) v = -INFINITY;
        }
        s[nt][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
    float alpha[2], m_use[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
      const float mn = fmaxf(m_r[i], mx[i]);
      m_use[i] = (mn == -INFINITY) ? 0.f : mn;
      alpha[i] = exp2f(m_r[i] - m_use[i]);
      m_r[i] = mn;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < C::BKV / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[nt][e] - m_use[e >> 1]);
        s[nt][e] = p;
        rs[e >> 1] += p;
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) l_r[i] = l_r[i] * alpha[i] + rs[i];
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) {
      acc[dt][0] *= alpha[0];
      acc[dt][1] *= alpha[0];
      acc[dt][2] *= alpha[1];
      acc[dt][3] *= alpha[1];
    }
#pragma unroll
    for (int kk = 0; kk < C::BKV / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t bb[4];
        ldb_frag_t<D>(tV, kk * 16, dp * 16, bb);
        mma16816(acc[2 * dp], pa, bb[0], bb[1]);
        mma16816(acc[2 * dp + 1], pa, bb[2], bb[3]);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 1);
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 2);
  }
  const float inv_a = 1.f / l_r[0], inv_b = 1.f / l_r[1];
  if (row_a < T) {
    __nv_bfloat16* op = o + (seq + row_a) * ld_o + h * D;
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt)
      *reinterpret_cast<uint32_t*>(op + dt * 8 + 2 * tq) = pack_bf16(acc[dt][0] * inv_a, acc[dt][1] * inv_a);
    if (tq == 0) lse[(static_cast<int64_t>(b) * nq + h) * T + row_a] = (m_r[0] + log2f(l_r[0])) * LN2;
  }
  if (row_b < T) {
    __nv_bfloat16* op = o + (seq + row_b) * ld_o + h * D;
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt)
      *reinterpret_cast<uint32_t*>(op + dt * 8 + 2 * tq) = pack_bf16(acc[dt][2] * inv_b, acc[dt][3] * inv_b);
    if (tq == 0) lse[(static_cast<int64_t>(b) * nq + h) * T + row_b] = (m_r[1] + log2f(l_r[1])) * LN2;
  }
}

// ============================================================== backward
// Delta[b,h,t] = sum_j dO[b,t,h,j] * O[b,t,h,j]
template <int D>
__global__ void attn_delta_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ d_o,
                                  int64_t ld_o, float* __restrict__ delta, int64_t rows, int T, int nq) {
  const int64_t id = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (id >= rows * nq) return;
  const int64_t row = id / nq;
  const int h = static_cast<int>(id % nq);
  const uint4* a = reinterpret_cast<const uint4*>(o + row * ld_o + h * D);
  const uint4* bq = reinterpret_cast<const uint4*>(d_o + row * ld_o + h * D);
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    uint4 u = a[c], v = bq[c];
    const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&u);
    const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 p = __bfloat1622float2(x[i]), q = __bfloat1622float2(y[i]);
      s += p.x * q.x + p.y * q.y;
    }
  }
  const int64_t b = row / T, t = row % T;
  delta[(b * nq + h) * T + t] = s;
}

template <int D>
struct BwdCfg {
  static constexpr int BQ = 64, BKV = 64, WARPS = 4, NT = WARPS * 32;
  static constexpr int TILE = 64 * D * 2;
  static constexpr int SMEM = 6 * TILE + 4 * 64 * 4;
};

// dQ for one query block of one head.
template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::NT, 1)
    attn_bwd_dq_kernel(const __nv_bfloat16* __restrict__ qkv, int64_t ld, const __nv_bfloat16* __restrict__ d_o,
                       int64_t ld_o, const float* __restrict__ lse, const float* __restrict__ delta,
                       __nv_bfloat16* __restrict__ dqkv, int T, int nq, int nkv, float scale_log2, float scale) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sO = smem + C::TILE;
  uint8_t* sK = smem + 2 * C::TILE;
  uint8_t* sV = smem + 4 * C::TILE;

  const int qb = gridDim.x - 1 - blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int c = (h * nkv) / nq;
  const int q0 = qb * C::BQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int r0 = warp * 16;
  const int64_t seq = static_cast<int64_t>(b) * T;
  const __nv_bfloat16* Qb = qkv + seq * ld + h * D;
  const __nv_bfloat16* Ob = d_o + seq * ld_o + h * D;
  const __nv_bfloat16* Kb = qkv + seq * ld + static_cast<int64_t>(nq) * D + c * D;
  const __nv_bfloat16* Vb = qkv + seq * ld + static_cast<int64_t>(nq + nkv) * D + c * D;
  const int n_kv = min((T + C::BKV - 1) / C::BKV, (q0 + C::BQ + C::BKV - 1) / C::BKV);

  load_tile<D, C::NT>(sQ, Qb, ld, q0, T, C::BQ);
  load_tile<D, C::NT>(sO, Ob, ld_o, q0, T, C::BQ);
  load_tile<D, C::NT>(sK, Kb, ld, 0, T, C::BKV);
  load_tile<D, C::NT>(sV, Vb, ld, 0, T, C::BKV);
  cp_commit();

  const int row_a = q0 + r0 + g, row_b = row_a + 8;
  const int64_t sb = (static_cast<int64_t>(b) * nq + h) * T;
  const float lse_a = row_a < T ? lse[sb + row_a] * LOG2E : 0.f;
  const float lse_b = row_b < T ? lse[sb + row_b] * LOG2E : 0.f;
  const float dl_a = row_a < T ? delta[sb + row_a] : 0.f;
  const float dl_b = row_b < T ? delta[sb + row_b] : 0.f;

  float dq[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;

  for (int j = 0; j < n_kv; ++j) {
    if (j + 1 < n_kv) {
      const int nb = (j + 1) & 1;
      load_tile<D, C::NT>(sK + nb * C::TILE, Kb, ld, (j + 1) * C::BKV, T, C::BKV);
      load_tile<D, C::NT>(sV + nb * C::TILE, Vb, ld, (j + 1) * C::BKV, T, C::BKV);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const uint8_t* tK = sK + (j & 1) * C::TILE;
    const uint8_t* tV = sV + (j & 1) * C::TILE;
    const int k0 = j * C::BKV;

    float s[C::BKV / 8][4], dp[C::BKV / 8][4];
#pragma unroll
    for (int i = 0; i < C::BKV / 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[i][e] = dp[i][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t qa[4], oa[4];
      lda_frag<D>(sQ, r0, kk, qa);
      lda_frag<D>(sO, r0, kk, oa);
#pragma unroll
      for (int np = 0; np < C::BKV / 16; ++np) {
        uint32_t bk[4], bv[4];
        ldb_frag<D>(tK, np * 16, kk, bk);
        ldb_frag<D>(tV, np * 16, kk, bv);
        mma16816(s[2 * np], qa, bk[0], bk[1]);
        mma16816(s[2 * np + 1], qa, bk[2], bk[3]);
        mma16816(dp[2 * np], oa, bv[0], bv[1]);
        mma16816(dp[2 * np + 1], oa, bv[2], bv[3]);
      }
    }
    const bool need_mask = k0 + C::BKV - 1 > q0 + r0;
#pragma unroll
    for (int nt = 0; nt < C::BKV / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = (e < 2) ? row_a : row_b;
        float p = exp2f(s[nt][e] * scale_log2 - ((e < 2) ? lse_a : lse_b));
        if (need_mask) {
          const int col = k0 + nt * 8 + 2 * tq + (e & 1);
          if (col > row) p = 0.f;
        }
        s[nt][e] = p * (dp[nt][e] - ((e < 2) ? dl_a : dl_b));  // dS
      }
    }
#pragma unroll
    for (int kk = 0; kk < C::BKV / 16; ++kk) {
      uint32_t da[4];
      da[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      da[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      da[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      da[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dpi = 0; dpi < D / 16; ++dpi) {
        uint32_t bb[4];
        ldb_frag_t<D>(tK, kk * 16, dpi * 16, bb);
        mma16816(dq[2 * dpi], da, bb[0], bb[1]);
        mma16816(dq[2 * dpi + 1], da, bb[2], bb[3]);
      }
    }
    __syncthreads();
  }
  if (row_a < T) {
    __nv_bfloat16* p = dqkv + (seq + row_a) * ld + h * D;
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt)
      *reinterpret_cast<uint32_t*>(p + dt * 8 + 2 * tq) = pack_bf16(dq[dt][0] * scale, dq[dt][1] * scale);
  }
  if (row_b < T) {
    __nv_bfloat16* p = dqkv + (seq + row_b) * ld + h * D;
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt)
      *reinterpret_cast<uint32_t*>(p + dt * 8 + 2 * tq) = pack_bf16(dq[dt][2] * scale, dq[dt][3] * scale);
  }
}

// dK and dV for one key block of one key/value head: loops over the query
// heads of the group (in order) and the query blocks from the diagonal on.
template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::NT, 1)
    attn_bwd_dkv_kernel(const __nv_bfloat16* __restrict__ qkv, int64_t ld, const __nv_bfloat16* __restrict__ d_o,
                        int64_t ld_o, const float* __restrict__ lse, const float* __restrict__ delta,
                        __nv_bfloat16* __restrict__ dqkv, int T, int nq, int nkv, float scale_log2, float scale) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::TILE;
  uint8_t* sQ = smem + 2 * C::TILE;  // 2 buffers
  uint8_t* sO = smem + 4 * C::TILE;  // 2 buffers
  float* sL = reinterpret_cast<float*>(smem + 6 * C::TILE);  // [2][64] lse (log2 domain)
  float* sD = sL + 2 * 64;                                   // [2][64] delta

  const int kb = blockIdx.x;  // small key blocks have the most query blocks: first
  const int c = blockIdx.y, b = blockIdx.z;
  const int grp = nq / nkv;
  const int k0 = kb * C::BKV;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int r0 = warp * 16;
  const int64_t seq = static_cast<int64_t>(b) * T;
  const __nv_bfloat16* Kb = qkv + seq * ld + static_cast<int64_t>(nq) * D + c * D;
  const __nv_bfloat16* Vb = qkv + seq * ld + static_cast<int64_t>(nq + nkv) * D + c * D;

  const int n_qb = (T + C::BQ - 1) / C::BQ;
  const int qb0 = k0 / C::BQ;
  const int per_head = n_qb - qb0;
  const int n_it = grp * per_head;

  auto issue = [&](int it, int buf) {
    const int h = c * grp + it / per_head;
    const int q0 = (qb0 + it % per_head) * C::BQ;
    load_tile<D, C::NT>(sQ + buf * C::TILE, qkv + seq * ld + h * D, ld, q0, T, C::BQ);
    load_tile<D, C::NT>(sO + buf * C::TILE, d_o + seq * ld_o + h * D, ld_o, q0, T, C::BQ);
    const int64_t sb = (static_cast<int64_t>(b) * nq + h) * T;
    for (int i = threadIdx.x; i < C::BQ; i += C::NT) {
      const int t = q0 + i;
      sL[buf * 64 + i] = t < T ? lse[sb + t] * LOG2E : INFINITY;
      sD[buf * 64 + i] = t < T ? delta[sb + t] : 0.f;
    }
  };

  load_tile<D, C::NT>(sK, Kb, ld, k0, T, C::BKV);
  load_tile<D, C::NT>(sV, Vb, ld, k0, T, C::BKV);
  if (n_it > 0) issue(0, 0);
  cp_commit();

  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;

  const int kv_a = k0 + r0 + g, kv_b = kv_a + 8;

  for (int it = 0; it < n_it; ++it) {
    if (it + 1 < n_it) {
      issue(it + 1, (it + 1) & 1);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const int buf = it & 1;
    const uint8_t* tQ = sQ + buf * C::TILE;
    const uint8_t* tO = sO + buf * C::TILE;
    const float* L = sL + buf * 64;
    const float* Dl = sD + buf * 64;
    const int q0 = (qb0 + it % per_head) * C::BQ;

    float s[C::BQ / 8][4], dp[C::BQ / 8][4];
#pragma unroll
    for (int i = 0; i < C::BQ / 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[i][e] = dp[i][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ka[4], va[4];
      lda_frag<D>(sK, r0, kk, ka);
      lda_frag<D>(sV, r0, kk, va);
#pragma unroll
      for (int np = 0; np < C::BQ / 16; ++np) {
        uint32_t bq[4], bo[4];
        ldb_frag<D>(tQ, np * 16, kk, bq);
        ldb_frag<D>(tO, np * 16, kk, bo);
        mma16816(s[2 * np], ka, bq[0], bq[1]);
        mma16816(s[2 * np + 1], ka, bq[2], bq[3]);
        mma16816(dp[2 * np], va, bo[0], bo[1]);
        mma16816(dp[2 * np + 1], va, bo[2], bo[3]);
      }
    }
    // s = S^T (rows kv, cols q) -> P^T; dp = dP^T
    const bool need_mask = q0 < k0 + r0 + 15;
    uint32_t pa[C::BQ / 16][4];
#pragma unroll
    for (int nt = 0; nt < C::BQ / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qi = nt * 8 + 2 * tq + (e & 1);
        float p = exp2f(s[nt][e] * scale_log2 - L[qi]);
        if (need_mask) {
          const int kvr = (e < 2) ? kv_a : kv_b;
          if (kvr > q0 + qi) p = 0.f;
        }
        s[nt][e] = p;
        dp[nt][e] = p * (dp[nt][e] - Dl[qi]);  // dS^T
      }
    }
#pragma unroll
    for (int kk = 0; kk < C::BQ / 16; ++kk) {
      pa[kk][0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[kk][1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[kk][2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[kk][3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
    }
    // dV += P^T dO
#pragma unroll
    for (int kk = 0; kk < C::BQ / 16; ++kk) {
#pragma unroll
      for (int dpi = 0; dpi < D / 16; ++dpi) {
        uint32_t bb[4];
        ldb_frag_t<D>(tO, kk * 16, dpi * 16, bb);
        mma16816(dv[2 * dpi], pa[kk], bb[0], bb[1]);
        mma16816(dv[2 * dpi + 1], pa[kk], bb[2], bb[3]);
      }
    }
    // dK += dS^T Q
#pragma unroll
    for (int kk = 0; kk < C::BQ / 16; ++kk) {
      uint32_t da[4];
      da[0] = pack_bf16(dp[2 * kk][0], dp[2 * kk][1]);
      da[1] = pack_bf16(dp[2 * kk][2], dp[2 * kk][3]);
      da[2] = pack_bf16(dp[2 * kk + 1][0], dp[2 * kk + 1][1]);
      da[3] = pack_bf16(dp[2 * kk + 1][2], dp[2 * kk + 1][3]);
#pragma unroll
      for (int dpi = 0; dpi < D / 16; ++dpi) {
        uint32_t bb[4];
        ldb_frag_t<D>(tQ, kk * 16, dpi * 16, bb);
        mma16816(dk[2 * dpi], da, bb[0], bb[1]);
        mma16816(dk[2 * dpi + 1], da, bb[2], bb[3]);
      }
    }
    __syncthreads();
  }
  const int64_t koff = static_cast<int64_t>(nq) * D + c * D;
  const int64_t voff = static_cast<int64_t>(nq + nkv) * D + c * D;
  if (kv_a < T) {
    __nv_bfloat16* p = dqkv + (seq + kv_a) * ld;
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) {
      *reinterpret_cast<uint32_t*>(p + koff + dt * 8 + 2 * tq) = pack_bf16(dk[dt][0] * scale, dk[dt][1] * scale);
      *reinterpret_cast<uint32_t*>(p + voff + dt * 8 + 2 * tq) = pack_bf16(dv[dt][0], dv[dt][1]);
    }
  }
  if (kv_b < T) {
    __nv_bfloat16* p = dqkv + (seq + kv_b) * ld;
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) {
      *reinterpret_cast<uint32_t*>(p + koff + dt * 8 + 2 * tq) = pack_bf16(dk[dt][2] * scale, dk[dt][3] * scale);
      *reinterpret_cast<uint32_t*>(p + voff + dt * 8 + 2 * tq) = pack_bf16(dv[dt][2], dv[dt][3]);
    }
  }
}

template <class K>
mt_status set_smem(K kernel, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return fail(MT_ERR_CUDA, "attention smem attribute: %s", cudaGetErrorString(e));
  return MT_OK;
}

template <int D>
mt_status fwd_t(const mt_bf16* qkv, int64_t ld, mt_bf16* o, int64_t ld_o, float* lse, int B, int T, int nq, int nkv,
                cudaStream_t st) {
  using C = FwdCfg<D>;
  static std::once_flag once;
  static mt_status attr = MT_OK;
  std::call_once(once, [] { attr = set_smem(attn_fwd_kernel<D>, C::SMEM); });
  MT_TRY(attr);
  dim3 grid((T + C::BQ - 1) / C::BQ, nq, B);
  const float scale_log2 = LOG2E / sqrtf(static_cast<float>(D));
  attn_fwd_kernel<D><<<grid, C::NT, C::SMEM, st>>>(reinterpret_cast<const __nv_bfloat16*>(qkv), ld,
                                                   reinterpret_cast<__nv_bfloat16*>(o), ld_o, lse, T, nq, nkv,
                                                   scale_log2);
  MT_TRY(launch_check("attn_fwd_kernel"));
  // QK^T and PV over the causal half (diagonal blocks counted in full)
  add_exec_flops(4.0 * B * nq * D * (0.5 * double(T) * double(T)));
  return MT_OK;
}

// delta = rowsum(dO * O) per (row, head) into `delta` unless the caller already
// formed it (have_delta), then dQ, dK, dV.
template <int D>
mt_status bwd_t(const mt_bf16* qkv, int64_t ld, const mt_bf16* o, const mt_bf16* d_o, int64_t ld_o, const float* lse,
                mt_bf16* dqkv, int B, int T, int nq, int nkv, float* delta, bool have_delta, const float* rope_tab,
                cudaStream_t st) {
  if (!have_delta) {
    const int64_t rows = static_cast<int64_t>(B) * T;
    const int64_t n = rows * nq;
    attn_delta_kernel<D><<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(o), reinterpret_cast<const __nv_bfloat16*>(d_o), ld_o, delta, rows, T,
        nq);
    MT_TRY(launch_check("attn_delta_kernel"));
  }
  if constexpr (D == 128) {
    return attn_bwd_tc_launch(qkv, ld, d_o, ld_o, lse, delta, dqkv, B, T, nq, nkv, rope_tab, st);
  } else {
    using C = BwdCfg<D>;
    static std::once_flag once;
    static mt_status attr = MT_OK;
    std::call_once(once, [] {
      attr = set_smem(attn_bwd_dq_kernel<D>, C::SMEM);
      if (attr == MT_OK) attr = set_smem(attn_bwd_dkv_kernel<D>, C::SMEM);
    });
    MT_TRY(attr);
    const float scale = 1.0f / sqrtf(static_cast<float>(D));
    const float scale_log2 = LOG2E * scale;
    dim3 gq((T + C::BQ - 1) / C::BQ, nq, B);
    attn_bwd_dq_kernel<D><<<gq, C::NT, C::SMEM, st>>>(reinterpret_cast<const __nv_bfloat16*>(qkv), ld,
                                                      reinterpret_cast<const __nv_bfloat16*>(d_o), ld_o, lse, delta,
                                                      reinterpret_cast<__nv_bfloat16*>(dqkv), T, nq, nkv, scale_log2,
                                                      scale);
    MT_TRY(launch_check("attn_bwd_dq_kernel"));
    dim3 gk((T + C::BKV - 1) / C::BKV, nkv, B);
    attn_bwd_dkv_kernel<D><<<gk, C::NT, C::SMEM, st>>>(reinterpret_cast<const __nv_bfloat16*>(qkv), ld,
                                                       reinterpret_cast<const __nv_bfloat16*>(d_o), ld_o, lse, delta,
                                                       reinterpret_cast<__nv_bfloat16*>(dqkv), T, nq, nkv, scale_log2,
                                                       scale);
    MT_TRY(launch_check("attn_bwd_dkv_kernel"));
    // dq: QK^T, dO V^T, dS K; dkv: QK^T, dO V^T, P^T dO, dS^T Q (causal half)
    add_exec_flops(14.0 * B * nq * D * (0.5 * double(T) * double(T)));
    return MT_OK;
  }
}

}  // namespace

uint64_t attn_bwd_ws_bytes(int B, int T, int nq) {
  return static_cast<uint64_t>(align_up(static_cast<int64_t>(B) * nq * T * 4, 256));
}

mt_status attn_fwd_tc_launch(const mt_bf16* qkv, int64_t ld, mt_bf16* o, int64_t ld_o, float* lse, int B, int T,
                             int nq, int nkv, cudaStream_t st);

// head_dim 128 runs the tcgen05 forward, head_dim 64 the mma.sync one.
mt_status attn_fwd_launch(const mt_bf16* qkv, int64_t ld, mt_bf16* o, int64_t ld_o, float* lse, int B, int T, int nq,
                          int nkv, int d, cudaStream_t st) {
  if (B == 0 || T == 0) return MT_OK;
  if (d == 128) return attn_fwd_tc_launch(qkv, ld, o, ld_o, lse, B, T, nq, nkv, st);
  if (d == 64) return fwd_t<64>(qkv, ld, o, ld_o, lse, B, T, nq, nkv, st);
  return fail(MT_ERR_UNSUPPORTED, "attention supports head_dim 64 and 128, not %d", d);
}

mt_status attn_bwd_launch(const mt_bf16* qkv, int64_t ld, const mt_bf16* o, const mt_bf16* d_o, int64_t ld_o,
                          const float* lse, mt_bf16* dqkv, int B, int T, int nq, int nkv, int d, void* ws,
                          cudaStream_t st) {
  if (B == 0 || T == 0) return MT_OK;
  float* delta = static_cast<float*>(ws);
  if (d == 128) return bwd_t<128>(qkv, ld, o, d_o, ld_o, lse, dqkv, B, T, nq, nkv, delta, false, nullptr, st);
  if (d == 64) return bwd_t<64>(qkv, ld, o, d_o, ld_o, lse, dqkv, B, T, nq, nkv, delta, false, nullptr, st);
  return fail(MT_ERR_UNSUPPORTED, "attention supports head_dim 64 and 128, not %d", d);
}

// The attention backward of the layer: delta already formed (the dO GEMM's epilogue). For
// head_dim 128, a non-NULL rope_tab makes dq and dk come out un-rotated; head_dim 64 takes
// no table (its caller un-rotates with rope_launch).
mt_status attn_bwd_delta_launch(const mt_bf16* qkv, int64_t ld, const mt_bf16* d_o, int64_t ld_o, const float* lse,
                                const float* delta, mt_bf16* dqkv, int B, int T, int nq, int nkv, int d,
                                const float* rope_tab, cudaStream_t st) {
  if (B == 0 || T == 0) return MT_OK;
  float* dl = const_cast<float*>(delta);
  if (d == 128) return bwd_t<128>(qkv, ld, nullptr, d_o, ld_o, lse, dqkv, B, T, nq, nkv, dl, true, rope_tab, st);
  if (d == 64 && rope_tab) return fail(MT_ERR_UNSUPPORTED, "attention backward: un-rotation needs head_dim 128");
  if (d == 64) return bwd_t<64>(qkv, ld, nullptr, d_o, ld_o, lse, dqkv, B, T, nq, nkv, dl, true, nullptr, st);
  return fail(MT_ERR_UNSUPPORTED, "attention supports head_dim 64 and 128, not %d", d);
}

}  // namespace mt

using namespace mt;

static mt_status attn_checks(const void* qkv, int64_t ld_qkv, const void* o, int64_t ld_o, int B, int T, int nq,
                             int nkv, int d) {
  if (!qkv || !o) return fail(MT_ERR_INVALID_ARG, "attention: NULL pointer");
  if (B < 0 || T < 0 || nq <= 0 || nkv <= 0 || nq % nkv) return fail(MT_ERR_INVALID_ARG, "attention: bad head counts");
  if (d != 64 && d != 128) return fail(MT_ERR_UNSUPPORTED, "attention supports head_dim 64 and 128, not %d", d);
  if (ld_qkv < static_cast<int64_t>(nq + 2 * nkv) * d || ld_o < static_cast<int64_t>(nq) * d)
    return fail(MT_ERR_INVALID_ARG, "attention: leading dimension too small");
  if (!aligned16(qkv) || !aligned16(o) || ld_qkv % 8 || ld_o % 8)
    return fail(MT_ERR_ALIGNMENT, "attention: 16-byte alignment of pointers and rows");
  return MT_OK;
}

extern "C" {

mt_status mt_attention_fwd(const mt_bf16* qkv, int64_t ld_qkv, mt_bf16* o, int64_t ld_o, float* lse, int32_t B,
                           int32_t T, int32_t nq, int32_t nkv, int32_t d, void* stream) {
  MT_TRY(attn_checks(qkv, ld_qkv, o, ld_o, B, T, nq, nkv, d));
  if (!lse) return fail(MT_ERR_INVALID_ARG, "attention: NULL lse");
  return attn_fwd_launch(qkv, ld_qkv, o, ld_o, lse, B, T, nq, nkv, d, as_stream(stream));
}

uint64_t mt_attention_bwd_workspace_bytes(int32_t B, int32_t T, int32_t nq) { return attn_bwd_ws_bytes(B, T, nq); }

mt_status mt_attention_bwd(const mt_bf16* qkv, int64_t ld_qkv, const mt_bf16* o, const mt_bf16* d_o, int64_t ld_o,
                           const float* lse, mt_bf16* dqkv, int32_t B, int32_t T, int32_t nq, int32_t nkv, int32_t d,
                           void* ws, uint64_t ws_bytes, void* stream) {
  MT_TRY(attn_checks(qkv, ld_qkv, o, ld_o, B, T, nq, nkv, d));
  if (!d_o || !lse || !dqkv || !ws) return fail(MT_ERR_INVALID_ARG, "attention_bwd: NULL pointer");
  if (!aligned16(d_o) || !aligned16(dqkv)) return fail(MT_ERR_ALIGNMENT, "attention_bwd: 16-byte alignment");
  if (ws_bytes < attn_bwd_ws_bytes(B, T, nq)) return fail(MT_ERR_WORKSPACE, "attention_bwd: workspace too small");
  return attn_bwd_launch(qkv, ld_qkv, o, d_o, ld_o, lse, dqkv, B, T, nq, nkv, d, ws, as_stream(stream));
}

}  // extern "C"
