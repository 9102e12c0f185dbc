// C = A * B^T on the sm_100a tensor cores: TMA-fed, tcgen05.mma with the
// accumulator in tensor memory, persistent and warp-specialised.
//
// This is the dense contraction of every projection of the decoder layer
// (QKV, O, gate/up, down) in its three uses: the forward Y = X W^T (both
// operands K-major), the input gradient dX = dY W (B is MN-major) and the
// weight gradient dW = dY^T X (both MN-major), which the layer template of
// the MegaTrain pages ("stateless layer templates", abstract) runs for every
// streamed layer.
//
// Design (details at the 2-SM kernel below)
// - A cluster of two CTAs on two SMs computes a 256 x 256 output tile with
//   tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16), persistent over the
//   output tiles; the weight-gradient layout at K >= 8192 uses a 256 x 512 tile.
// - Per CTA: warp 0 is the TMA producer, warp 1 allocates TMEM and (in the
//   even CTA) issues the MMAs for the pair, the remaining warps run the
//   epilogue (tcgen05.ld of the fp32 accumulator; bias, residual, fp32
//   accumulate, SwiGLU forward or backward; bf16 or fp32 stores).
// - Two 256-column accumulators in TMEM: the epilogue of one tile overlaps
//   the main loop of the next.
// - Operands are staged with 128-byte swizzle. K-major tiles are boxes of
//   64 (K) x 128 rows; MN-major tiles are boxes of 64 (M or N) x 64 (K) placed
//   one atom apart, which is the descriptor's leading-byte offset.
// - Every mbarrier wait is bounded (4 s); when one runs out the kernel sets
//   the device error word and all roles leave their loops, free TMEM and exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <mutex>
#include <string>

#include "mt_internal.h"
#include "tcgen05.cuh"

namespace mt {
GemmTimer* current_gemm_timer();

namespace {

using namespace tc;

constexpr int MN_BOX = 64 * 64 * 2;  // one 64 x 64 MN-major box: 8 KiB
constexpr uint32_t TMEM_COLS = 512;

struct EpiArgs {
  void* C;
  const __nv_bfloat16* bias;
  const __nv_bfloat16* res;
  int64_t ldc, ldr;
  int M, N, K;
  int c_f32, accumulate;
  int raster;
  // swiglu == 1, SwiGLU epilogue (2-SM kernel, both operands K-major): B holds
  // [Wg; Wu] (N = 2F rows); a pair tile covers 128 features j, C[m, j] =
  // silu(g) * u in bf16, and when gu is set g and u are also stored to gu[m, j]
  // and gu[m, F + j].
  // swiglu == 2, SwiGLU backward epilogue (any layout, N = F): the accumulator
  // is dm[m, j]; g = gu[m, j] and u = gu[m, F + j] are read and replaced by
  // dg = dm u silu'(g) and du = dm silu(g). C is not written.
  int swiglu, F;
  __nv_bfloat16* gu;
  int64_t ld_gu;
  // rope_tab != NULL, RoPE epilogue (bf16 C, no residual): the first rope_cols
  // columns are heads of rope_hd columns; after the bias, the pair (i, i + rope_hd/2)
  // of each such head is rotated by the angle of position t = row % rope_T,
  // (a, b) -> (a cos - b sin, b cos + a sin) with (cos, sin) = rope_tab[t * rope_hd/2 + i],
  // and rounded to bf16 once.
  const float2* rope_tab;
  int rope_cols, rope_hd, rope_T;
  // dot_with != NULL (bf16 C): per row r and head h of dot_hd columns, also
  // dot_out[((r / dot_T) * dot_heads + h) * dot_T + r % dot_T] = sum_j C[r, j] * dot_with[r * ld_dot + j]
  // over the head's columns, with C as stored (rounded to bf16), in fp32.
  const __nv_bfloat16* dot_with;
  int64_t ld_dot;
  float* dot_out;
  int dot_hd, dot_T, dot_heads;
  // 32-byte row chunks (base and row stride multiples of 32 bytes): the epilogue
  // moves C, the residual and g / u with 256-bit accesses, one whole sector each
  int c_v8, res_v8, gu_v8;
};

// Output-tile order. raster 0: groups of 16 row-blocks, columns within a
// group; raster 1: row-major over all column blocks (the B operand stays in
// L2); raster 2: column-major over all row blocks (the A operand stays in L2).
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int raster, int& mb, int& nb) {
  if (raster == 1) {
    mb = t / num_n;
    nb = t - mb * num_n;
    return;
  }
  if (raster == 2) {
    nb = t / num_m;
    mb = t - nb * num_m;
    return;
  }
  constexpr int G = 16;
  const int group_tiles = G * num_n;
  const int g = t / group_tiles;
  const int first_m = g * G;
  const int gm = min(num_m - first_m, G);
  const int r = t - g * group_tiles;
  mb = first_m + r % gm;
  nb = r / gm;
}

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ uint32_t pack_bf16_pair(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// sigmoid(z) = 1 / (1 + 2^(-z log2 e)) with the MUFU ex2 and a fast divide
// (relative error well below bf16 rounding; 2^x saturates to 0 / inf, giving
// sigmoid 1 / 0 at the extremes).
__device__ __forceinline__ float sigmoid_fast(float z) {
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-1.4426950408889634f * z));
  return __fdividef(1.0f, 1.0f + e);
}

// 256-bit global accesses (32 bytes, one L2 sector; p 32-byte aligned). A row
// per thread reads and writes 64 or 128 bytes per 32-column chunk: 16-byte
// accesses would touch each sector twice.
__device__ __forceinline__ void ld_v8(const void* p, uint32_t (&r)[8]) {
  asm volatile("ld.global.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "l"(p)
               : "memory");
}
__device__ __forceinline__ void ld_v8_cs(const void* p, uint32_t (&r)[8]) {
  asm volatile("ld.global.cs.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "l"(p)
               : "memory");
}
__device__ __forceinline__ void st_v8(void* p, const uint32_t (&r)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]),
               "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void st_v8_cs(void* p, const uint32_t (&r)[8]) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]),
               "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// Epilogue of one 32-column chunk of one output row.
__device__ __forceinline__ void store_chunk(const EpiArgs& ep, int row, int col0, const uint32_t (&r)[32]) {
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  const bool full = col0 + 32 <= ep.N;
  if (full) {
    if (ep.bias) {
      const uint4* bp = reinterpret_cast<const uint4*>(ep.bias + col0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 u = __ldg(bp + q);
        const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[q * 8 + j] += bf2f(h[j]);
      }
    }
    if (ep.res) {
      const __nv_bfloat16* rrow = ep.res + static_cast<int64_t>(row) * ep.ldr + col0;
      if (ep.res_v8) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t w[8];
          ld_v8(rrow + hh * 16, w);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
            v[hh * 16 + 2 * j] += f.x;
            v[hh * 16 + 2 * j + 1] += f.y;
          }
        }
      } else {
        const uint4* rp = reinterpret_cast<const uint4*>(rrow);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 u = rp[q];
          const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
          for (int j = 0; j < 8; ++j) v[q * 8 + j] += bf2f(h[j]);
        }
      }
    }
    if (ep.c_f32 && ep.c_v8) {
      float* cp = static_cast<float*>(ep.C) + static_cast<int64_t>(row) * ep.ldc + col0;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        uint32_t w[8];
        if (ep.accumulate) {
          ld_v8(cp + hh * 8, w);
#pragma unroll
          for (int j = 0; j < 8; ++j) w[j] = __float_as_uint(__uint_as_float(w[j]) + v[hh * 8 + j]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) w[j] = __float_as_uint(v[hh * 8 + j]);
        }
        st_v8(cp + hh * 8, w);
      }
    } else if (!ep.c_f32 && ep.c_v8) {
      __nv_bfloat16* cp = static_cast<__nv_bfloat16*>(ep.C) + static_cast<int64_t>(row) * ep.ldc + col0;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = pack_bf16_pair(v[hh * 16 + 2 * j], v[hh * 16 + 2 * j + 1]);
        st_v8(cp + hh * 16, w);
      }
    } else if (ep.c_f32) {
      float4* cp = reinterpret_cast<float4*>(static_cast<float*>(ep.C) + static_cast<int64_t>(row) * ep.ldc + col0);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float4 o = make_float4(v[q * 4], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
        if (ep.accumulate) {
          float4 p = cp[q];
          o.x += p.x;
          o.y += p.y;
          o.z += p.z;
          o.w += p.w;
        }
        cp[q] = o;
      }
    } else {
      uint4* cp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(ep.C) + static_cast<int64_t>(row) * ep.ldc +
                                           col0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) h[j] = __floats2bfloat162_rn(v[q * 8 + 2 * j], v[q * 8 + 2 * j + 1]);
        cp[q] = u;
      }
    }
  } else {
    for (int j = 0; j < 32; ++j) {
      const int col = col0 + j;
      if (col >= ep.N) break;
      float x = v[j];
      if (ep.bias) x += bf2f(ep.bias[col]);
      if (ep.res) x += bf2f(ep.res[static_cast<int64_t>(row) * ep.ldr + col]);
      if (ep.c_f32) {
        float* cp = static_cast<float*>(ep.C) + static_cast<int64_t>(row) * ep.ldc + col;
        *cp = ep.accumulate ? *cp + x : x;
      } else {
        static_cast<__nv_bfloat16*>(ep.C)[static_cast<int64_t>(row) * ep.ldc + col] = __float2bfloat16_rn(x);
      }
    }
  }
}

// RoPE epilogue of one row: 32 columns of the first half of a head (clo, features
// i0 .. i0 + 31 of the rotation) and their 32 partners of the second half (chi).
__device__ __forceinline__ void store_rope_pair(const EpiArgs& ep, int row, int clo, int chi, int i0,
                                                const uint32_t (&rl)[32], const uint32_t (&rh)[32]) {
  float lo[32], hi[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    lo[j] = __uint_as_float(rl[j]);
    hi[j] = __uint_as_float(rh[j]);
  }
  if (ep.bias) {
    const uint4* bl = reinterpret_cast<const uint4*>(ep.bias + clo);
    const uint4* bh = reinterpret_cast<const uint4*>(ep.bias + chi);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 ul = __ldg(bl + q), uh = __ldg(bh + q);
      const __nv_bfloat16* hl = reinterpret_cast<const __nv_bfloat16*>(&ul);
      const __nv_bfloat16* hh = reinterpret_cast<const __nv_bfloat16*>(&uh);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        lo[q * 8 + j] += bf2f(hl[j]);
        hi[q * 8 + j] += bf2f(hh[j]);
      }
    }
  }
  const int t = row % ep.rope_T;
  const float4* tab = reinterpret_cast<const float4*>(ep.rope_tab + static_cast<int64_t>(t) * (ep.rope_hd / 2) + i0);
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const float4 cs = __ldg(tab + q);  // (cos, sin) of features i0 + 2q and i0 + 2q + 1
    const float a0 = lo[2 * q], b0 = hi[2 * q], a1 = lo[2 * q + 1], b1 = hi[2 * q + 1];
    lo[2 * q] = a0 * cs.x - b0 * cs.y;
    hi[2 * q] = b0 * cs.x + a0 * cs.y;
    lo[2 * q + 1] = a1 * cs.z - b1 * cs.w;
    hi[2 * q + 1] = b1 * cs.z + a1 * cs.w;
  }
  __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(ep.C) + static_cast<int64_t>(row) * ep.ldc;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 ul, uh;
    __nv_bfloat162* pl = reinterpret_cast<__nv_bfloat162*>(&ul);
    __nv_bfloat162* ph = reinterpret_cast<__nv_bfloat162*>(&uh);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      pl[j] = __floats2bfloat162_rn(lo[q * 8 + 2 * j], lo[q * 8 + 2 * j + 1]);
      ph[j] = __floats2bfloat162_rn(hi[q * 8 + 2 * j], hi[q * 8 + 2 * j + 1]);
    }
    reinterpret_cast<uint4*>(crow + clo)[q] = ul;
    reinterpret_cast<uint4*>(crow + chi)[q] = uh;
  }
}

// bf16 store of one 32-column chunk (no bias or residual) that also returns
// sum_j bf16(v_j) * dot_with[row, col0 + j] in fp32 (the dot epilogue).
__device__ __forceinline__ float store_chunk_dot(const EpiArgs& ep, int row, int col0, const uint32_t (&r)[32]) {
  uint4* cp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(ep.C) + static_cast<int64_t>(row) * ep.ldc + col0);
  const uint4* op = reinterpret_cast<const uint4*>(ep.dot_with + static_cast<int64_t>(row) * ep.ld_dot + col0);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 ov = op[q];
    const __nv_bfloat162* ho = reinterpret_cast<const __nv_bfloat162*>(&ov);
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      h[j] = __floats2bfloat162_rn(__uint_as_float(r[q * 8 + 2 * j]), __uint_as_float(r[q * 8 + 2 * j + 1]));
      const float2 c = __bfloat1622float2(h[j]), o = __bfloat1622float2(ho[j]);
      acc[q] = fmaf(c.x, o.x, acc[q]);
      acc[q] = fmaf(c.y, o.y, acc[q]);
    }
    cp[q] = u;
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// SwiGLU backward of 32 features of one row from the fp32 dm accumulators:
// with s = sigmoid(g), dg = dm u s (1 + g (1 - s)) and du = dm g s, written over
// g and u in place (each element is read and written by the same thread).
__device__ __forceinline__ void store_swiglu_bwd(const EpiArgs& ep, int row, int f0, const uint32_t (&r)[32]) {
  __nv_bfloat16* grow = ep.gu + static_cast<int64_t>(row) * ep.ld_gu;
  if (f0 + 32 <= ep.F && ep.gu_v8) {
    uint32_t gw[2][8], uw[2][8];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      ld_v8_cs(grow + f0 + hh * 16, gw[hh]);
      ld_v8_cs(grow + ep.F + f0 + hh * 16, uw[hh]);
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[hh][j]));
        const float2 u = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uw[hh][j]));
        const float d0 = __uint_as_float(r[hh * 16 + 2 * j]), d1 = __uint_as_float(r[hh * 16 + 2 * j + 1]);
        const float s0 = sigmoid_fast(g.x), s1 = sigmoid_fast(g.y);
        gw[hh][j] = pack_bf16_pair(d0 * u.x * s0 * (1.0f + g.x * (1.0f - s0)), d1 * u.y * s1 * (1.0f + g.y * (1.0f - s1)));
        uw[hh][j] = pack_bf16_pair(d0 * g.x * s0, d1 * g.y * s1);
      }
      st_v8_cs(grow + f0 + hh * 16, gw[hh]);
      st_v8_cs(grow + ep.F + f0 + hh * 16, uw[hh]);
    }
  } else if (f0 + 32 <= ep.F) {
    uint4* gp = reinterpret_cast<uint4*>(grow + f0);
    uint4* up = reinterpret_cast<uint4*>(grow + ep.F + f0);
    // g and u are read once and written once: streaming loads / stores keep them from
    // evicting the GEMM's operand tiles from L2; all eight loads are in flight together
    uint4 ug[4], uu[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      ug[q] = __ldcs(gp + q);
      uu[q] = __ldcs(up + q);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 og, ou;
      const __nv_bfloat162* hg = reinterpret_cast<const __nv_bfloat162*>(&ug[q]);
      const __nv_bfloat162* hu = reinterpret_cast<const __nv_bfloat162*>(&uu[q]);
      __nv_bfloat162* dg = reinterpret_cast<__nv_bfloat162*>(&og);
      __nv_bfloat162* du = reinterpret_cast<__nv_bfloat162*>(&ou);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 g = __bfloat1622float2(hg[j]), u = __bfloat1622float2(hu[j]);
        const float d0 = __uint_as_float(r[q * 8 + 2 * j]), d1 = __uint_as_float(r[q * 8 + 2 * j + 1]);
        const float s0 = sigmoid_fast(g.x), s1 = sigmoid_fast(g.y);
        dg[j] = __floats2bfloat162_rn(d0 * u.x * s0 * (1.0f + g.x * (1.0f - s0)),
                                      d1 * u.y * s1 * (1.0f + g.y * (1.0f - s1)));
        du[j] = __floats2bfloat162_rn(d0 * g.x * s0, d1 * g.y * s1);
      }
      __stcs(gp + q, og);
      __stcs(up + q, ou);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (f0 + j < ep.F) {
        const float g = bf2f(grow[f0 + j]), u = bf2f(grow[ep.F + f0 + j]), d = __uint_as_float(r[j]);
        const float sg = sigmoid_fast(g);
        grow[f0 + j] = __float2bfloat16_rn(d * u * sg * (1.0f + g * (1.0f - sg)));
        grow[ep.F + f0 + j] = __float2bfloat16_rn(d * g * sg);
      }
    }
  }
}

// SwiGLU epilogue of 32 features of one row: m = silu(g) * u from the fp32
// accumulators (g, u optionally stored too).
__device__ __forceinline__ void store_swiglu(const EpiArgs& ep, int row, int f0, const uint32_t (&rg)[32],
                                             const uint32_t (&ru)[32]) {
  float m[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float g = __uint_as_float(rg[j]), u = __uint_as_float(ru[j]);
    m[j] = g * sigmoid_fast(g) * u;
  }
  __nv_bfloat16* mrow = static_cast<__nv_bfloat16*>(ep.C) + static_cast<int64_t>(row) * ep.ldc;
  __nv_bfloat16* grow = ep.gu ? ep.gu + static_cast<int64_t>(row) * ep.ld_gu : nullptr;
  if (f0 + 32 <= ep.F && ep.c_v8 && (!grow || ep.gu_v8)) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t wm[8], wg[8], wu[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = hh * 16 + 2 * j;
        wm[j] = pack_bf16_pair(m[e], m[e + 1]);
        wg[j] = pack_bf16_pair(__uint_as_float(rg[e]), __uint_as_float(rg[e + 1]));
        wu[j] = pack_bf16_pair(__uint_as_float(ru[e]), __uint_as_float(ru[e + 1]));
      }
      st_v8(mrow + f0 + hh * 16, wm);
      if (grow) {
        st_v8(grow + f0 + hh * 16, wg);
        st_v8(grow + ep.F + f0 + hh * 16, wu);
      }
    }
  } else if (f0 + 32 <= ep.F) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 um, ug, uu;
      __nv_bfloat162* hm = reinterpret_cast<__nv_bfloat162*>(&um);
      __nv_bfloat162* hg = reinterpret_cast<__nv_bfloat162*>(&ug);
      __nv_bfloat162* hu = reinterpret_cast<__nv_bfloat162*>(&uu);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = q * 8 + 2 * j;
        hm[j] = __floats2bfloat162_rn(m[e], m[e + 1]);
        hg[j] = __floats2bfloat162_rn(__uint_as_float(rg[e]), __uint_as_float(rg[e + 1]));
        hu[j] = __floats2bfloat162_rn(__uint_as_float(ru[e]), __uint_as_float(ru[e + 1]));
      }
      reinterpret_cast<uint4*>(mrow + f0)[q] = um;
      if (grow) {
        reinterpret_cast<uint4*>(grow + f0)[q] = ug;
        reinterpret_cast<uint4*>(grow + ep.F + f0)[q] = uu;
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (f0 + j < ep.F) {
        mrow[f0 + j] = __float2bfloat16_rn(m[j]);
        if (grow) {
          grow[f0 + j] = __float2bfloat16_rn(__uint_as_float(rg[j]));
          grow[ep.F + f0 + j] = __float2bfloat16_rn(__uint_as_float(ru[j]));
        }
      }
    }
  }
}

// ============================================================== 2-SM kernel
// tcgen05.mma.cta_group::2: a cluster of two CTAs on two SMs computes a
// 256 x 256 output tile. Each CTA stages its own 128 rows of A and its own 128
// columns' worth of B (3 stages of 64 KiB), so per FLOP each SM moves a third
// less operand data through shared memory than a one-SM 128 x 256 tile. The even CTA issues the MMAs for the pair; its full
// barriers count both CTAs' TMA bytes, each MMA commit signals both CTAs'
// empty / accumulator-full barriers, and both CTAs' epilogue warps arrive on
// the even CTA's accumulator-empty barrier. Every CTA loads its own operands
// with plain per-CTA tensor copies; no copy is shared between CTAs.
// NH = 2 widens the pair tile to 256 x 512 (two N = 256 MMAs per K step into
// one 512-column accumulator, four stages of 64-wide K, eight epilogue
// warps): a quarter fewer operand bytes per FLOP and a deeper ring, at the
// price of a single accumulator, whose epilogue the next tile's MMAs wait for.
namespace c2 {
constexpr int BM = 256, BN = 256;
constexpr int HALF = 128 * 64 * 2;  // 16 KiB: one CTA's 128 rows of A (or B) for one 64-wide K atom
constexpr int SMEM_TILES = 6 * 2 * HALF;  // 6 atoms of A and B per CTA: 192 KiB
constexpr int SMEM_BYTES = SMEM_TILES + 256 + 1024;
}  // namespace c2

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA load into this CTA's shared memory that completes its bytes on the
// pair's barrier (which lives in the even CTA).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t cluster_bar, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void umma2_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrives on the barrier at this shared offset in both CTAs of the pair once
// the MMAs issued so far have completed.
__device__ __forceinline__ void umma2_commit_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

__host__ __device__ constexpr uint32_t make_idesc2(bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(c2::BN >> 3) << 17) | (static_cast<uint32_t>(c2::BM >> 4) << 24);
}

// Bytes one CTA loads for 128 rows of one operand and one 64-wide K atom
// (boxes wholly past the operand's rows are skipped).
__device__ __forceinline__ uint32_t rows_bytes(bool mn, int r0, int R) {
  uint32_t b = 0;
  if (!mn) {
    if (r0 < R) b += c2::HALF;
  } else {
    for (int j = 0; j < 2; ++j)
      if (r0 + 64 * j < R) b += MN_BOX;
  }
  return b;
}

// TMA warp, MMA warp and four epilogue warps per 256 accumulator columns, one
// per TMEM lane quarter. Measured and not kept: eight epilogue warps on the
// 256 x 256 tile (5-12% slower on every shape of the layer), an L2 prefetch of
// the next tile's epilogue operands and register double-buffering of the
// SwiGLU backward's g / u loads (no gain; 15% slower).
constexpr int threads2(int nh) { return 64 + 128 * nh; }

// KA: 64-wide K atoms per pipeline stage (NH = 1: 1 -> 6 stages of 64, 2 -> 3
// stages of 128; NH = 2: 1 -> 4 stages of 64). NH: N = 256 halves of the tile.
template <bool A_MN, bool B_MN, int KA, int NH>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(threads2(NH), 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, EpiArgs ep,
                 int32_t* err) {
  constexpr int BM = c2::BM, BN = 256 * NH, BK = 64 * KA, HALF = c2::HALF;
  constexpr int STAGES = (NH == 1 ? 6 : 4) / KA;
  constexpr int A_STAGE = HALF * KA, B_STAGE = HALF * KA * NH;  // one CTA's A / B bytes per stage
  constexpr int NACC = NH == 1 ? 2 : 1;                           // accumulators in TMEM
  constexpr int EPI_WARPS = 4 * NH;
  constexpr int SMEM_TILES = STAGES * (A_STAGE + B_STAGE);
  static_assert(SMEM_TILES == c2::SMEM_TILES, "every variant stages 192 KiB");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_TILES);
  uint64_t* full = bars;                // TMA (both CTAs) -> MMA; used in the even CTA
  uint64_t* empty = bars + STAGES;      // MMA -> TMA, in each CTA
  uint64_t* tfull = bars + 2 * STAGES;  // MMA -> epilogue, in each CTA
  uint64_t* tempty = tfull + NACC;      // epilogue warps of both CTAs -> MMA; used in the even CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + NACC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int num_m = (ep.M + BM - 1) / BM;
  const int num_n = ep.swiglu == 1 ? (ep.F + 128 * NH - 1) / (128 * NH) : (ep.N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (ep.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 2 * EPI_WARPS);  // one arrival per epilogue warp of each CTA
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
  }
  cluster_sync();  // barriers of both CTAs are initialised before any remote use
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    uint32_t it = 0;
    bool ok = true;
    for (int t = cluster; t < num_tiles && ok; t += n_clusters) {
      int mb, nb;
      tile_coords(t, num_m, num_n, ep.raster, mb, nb);
      const int m_own = mb * BM + static_cast<int>(rank) * 128;  // this CTA's A rows
      // this CTA's B rows of N-half h (SwiGLU: the gate rows in the even CTA, the up rows in the odd one)
      auto n_base = [&](int h, int rk) {
        if (ep.swiglu == 1) return (rk == 0 ? 0 : ep.F) + nb * 128 * NH + h * 128;
        return nb * BN + h * 256 + rk * 128;
      };
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        if (!warp_wait(smem_u32(&empty[s]), ph ^ 1u, abort_flag, err, DEV_ERR_TIMEOUT_PRODUCER)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const uint32_t fb = map_to_rank(smem_u32(&full[s]), 0);
          const int k0 = kb * BK;
          const int atoms = min(KA, (ep.K - k0 + 63) / 64);  // atoms wholly past K are not loaded
          if (rank == 0) {
            uint32_t bytes = rows_bytes(A_MN, mb * BM, ep.M) + rows_bytes(A_MN, mb * BM + 128, ep.M);
            for (int h = 0; h < NH; ++h) bytes += rows_bytes(B_MN, n_base(h, 0), ep.N) + rows_bytes(B_MN, n_base(h, 1), ep.N);
            mbar_expect_tx(smem_u32(&full[s]), bytes * static_cast<uint32_t>(atoms));
          }
          const uint32_t a_dst = smem_u32(sA + s * A_STAGE), b_dst0 = smem_u32(sB + s * B_STAGE);
          for (int at = 0; at < atoms; ++at) {
            const int ka = k0 + 64 * at;
            if (!A_MN) {
              if (m_own < ep.M) tma_load_2d_pair(a_dst + at * HALF, &tmA, fb, ka, m_own);
            } else {
              for (int j = 0; j < 2; ++j)
                if (m_own + 64 * j < ep.M)
                  tma_load_2d_pair(a_dst + j * KA * MN_BOX + at * MN_BOX, &tmA, fb, m_own + 64 * j, ka);
            }
            for (int h = 0; h < NH; ++h) {
              const int n_own = n_base(h, static_cast<int>(rank));
              const uint32_t b_dst = b_dst0 + h * HALF * KA;  // sub-tile of N-half h
              if (!B_MN) {
                if (n_own < ep.N) tma_load_2d_pair(b_dst + at * HALF, &tmB, fb, ka, n_own);
              } else {
                for (int j = 0; j < 2; ++j)
                  if (n_own + 64 * j < ep.N)
                    tma_load_2d_pair(b_dst + j * KA * MN_BOX + at * MN_BOX, &tmB, fb, n_own + 64 * j, ka);
              }
            }
          }
        }
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (even CTA)
    if (rank == 0) {
      constexpr uint32_t idesc = make_idesc2(A_MN, B_MN);
      uint32_t it = 0;
      int tl = 0;
      bool ok = true;
      for (int t = cluster; t < num_tiles && ok; t += n_clusters, ++tl) {
        const int ab = NACC == 2 ? (tl & 1) : 0;
        const uint32_t aph = static_cast<uint32_t>(NACC == 2 ? (tl >> 1) : tl) & 1u;
        if (!warp_wait(smem_u32(&tempty[ab]), aph ^ 1u, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) break;
        fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(ab * BN);
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!warp_wait(smem_u32(&full[s]), ph, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          fence_after();
          if (lane == 0) {
            const uint32_t a_base = smem_u32(sA + s * A_STAGE), b_base = smem_u32(sB + s * B_STAGE);
            const int ksteps = 4 * min(KA, (ep.K - kb * BK + 63) / 64);
            for (int kk = 0; kk < ksteps; ++kk) {
              // K-major: atom kk/4, then 16 elements (32 bytes) per step inside the swizzled row.
              // MN-major: 16 K-rows (two 8-row groups of 1 KiB) per step; MN atoms KA*8 KiB apart.
              const uint32_t koff_k = static_cast<uint32_t>((kk >> 2) * HALF + (kk & 3) * 32);
              const uint32_t koff_mn = static_cast<uint32_t>(kk * 2048);
              const uint64_t ad = A_MN ? smem_desc(a_base + koff_mn, KA * MN_BOX, 1024) : smem_desc(a_base + koff_k, 16, 1024);
#pragma unroll
              for (int h = 0; h < NH; ++h) {
                const uint32_t bh = b_base + h * HALF * KA;
                const uint64_t bd = B_MN ? smem_desc(bh + koff_mn, KA * MN_BOX, 1024) : smem_desc(bh + koff_k, 16, 1024);
                umma2_bf16(d_tmem + h * 256, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
              }
            }
            umma2_commit_both(smem_u32(&empty[s]));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) umma2_commit_both(smem_u32(&tfull[ab]));
        __syncwarp();
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;          // TMEM lanes [32 q, 32 q + 32)
    const int hc = (warp - 2) >> 2;  // N-half of the accumulator this warp drains
    int tl = 0;
    for (int t = cluster; t < num_tiles; t += n_clusters, ++tl) {
      const int ab = NACC == 2 ? (tl & 1) : 0;
      const uint32_t aph = static_cast<uint32_t>(NACC == 2 ? (tl >> 1) : tl) & 1u;
      int mb, nb;
      tile_coords(t, num_m, num_n, ep.raster, mb, nb);
      if (!warp_wait(smem_u32(&tfull[ab]), aph, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) break;
      fence_after();
      const int row = mb * BM + static_cast<int>(rank) * 128 + q * 32 + lane;
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(ab * BN + hc * 256);
      if (ep.swiglu == 1) {
        for (int c = 0; c < 4; ++c) {
          const int f0 = nb * 128 * NH + hc * 128 + c * 32;
          if (f0 >= ep.F) break;
          uint32_t rg[32], ru[32];
          tmem_ld32(tbase + static_cast<uint32_t>(c * 32), rg);
          tmem_ld32(tbase + static_cast<uint32_t>(128 + c * 32), ru);
          if (row < ep.M) store_swiglu(ep, row, f0, rg, ru);
        }
      } else if (ep.rope_tab) {
        // a head holds hcn chunks of 32 columns; chunk c pairs with chunk c + hcn / 2
        // (tiles start on head boundaries: 256 columns are whole heads of 64 or 128)
        const int hcn = ep.rope_hd / 32, half = hcn / 2;
        for (int c = 0; c < 8; ++c) {
          const int col0 = nb * BN + hc * 256 + c * 32;
          if (col0 >= ep.N) break;
          const int within = c % hcn;
          if (col0 < ep.rope_cols) {
            if (within >= half) continue;  // done with its partner
            uint32_t rl[32], rh[32];
            tmem_ld32(tbase + static_cast<uint32_t>(c * 32), rl);
            tmem_ld32(tbase + static_cast<uint32_t>((c + half) * 32), rh);
            if (row < ep.M) store_rope_pair(ep, row, col0, col0 + half * 32, within * 32, rl, rh);
          } else {
            uint32_t r[32];
            tmem_ld32(tbase + static_cast<uint32_t>(c * 32), r);
            if (row < ep.M) store_chunk(ep, row, col0, r);
          }
        }
      } else if (ep.dot_with) {
        const int hcn = ep.dot_hd / 32;
        float acc = 0.f;
        for (int c = 0; c < 8; ++c) {
          const int col0 = nb * BN + hc * 256 + c * 32;
          if (col0 >= ep.N) break;
          uint32_t r[32];
          tmem_ld32(tbase + static_cast<uint32_t>(c * 32), r);
          if (row < ep.M) {
            acc += store_chunk_dot(ep, row, col0, r);
            if (c % hcn == hcn - 1) {  // the head's last chunk
              const int h = col0 / ep.dot_hd;
              const int sq = row / ep.dot_T, t = row - sq * ep.dot_T;
              ep.dot_out[(static_cast<int64_t>(sq) * ep.dot_heads + h) * ep.dot_T + t] = acc;
              acc = 0.f;
            }
          }
        }
      } else {
        for (int c = 0; c < 8; ++c) {
          const int col0 = nb * BN + hc * 256 + c * 32;
          if (col0 >= ep.N) break;
          uint32_t r[32];
          tmem_ld32(tbase + static_cast<uint32_t>(c * 32), r);
          if (row < ep.M) {
            if (ep.swiglu == 2)
              store_swiglu_bwd(ep, row, col0, r);
            else
              store_chunk(ep, row, col0, r);
          }
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_rank(smem_u32(&tempty[ab]), 0));
    }
  }

  fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while its peer may still signal it
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

// ------------------------------------------------------------------ host side
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

mt_status make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                   uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return fail(MT_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld_elems * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for a %llu x %llu tensor, ld %llu", int(r),
                (unsigned long long)inner, (unsigned long long)outer, (unsigned long long)ld_elems);
  return MT_OK;
}

// Largest number of 2-CTA clusters of gemm2_kernel that fit on the device at once.
template <bool A_MN, bool B_MN, int KA, int NH>
int max_pair_clusters() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
    cfg.blockDim = dim3(threads2(NH), 1, 1);
    cfg.dynamicSmemBytes = c2::SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm2_kernel<A_MN, B_MN, KA, NH>, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms() / 2;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

template <bool A_MN, bool B_MN, int KA, int NH>
mt_status launch_2sm_ka(const CUtensorMap& ta, const CUtensorMap& tb, const EpiArgs& ep, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm2_kernel<A_MN, B_MN, KA, NH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    c2::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return fail(MT_ERR_CUDA, "gemm2 smem attribute: %s", cudaGetErrorString(attr_err));
  const int num_n = ep.swiglu == 1 ? (ep.F + 128 * NH - 1) / (128 * NH) : (ep.N + 256 * NH - 1) / (256 * NH);
  const int num_tiles = ((ep.M + c2::BM - 1) / c2::BM) * num_n;
  const int clusters = std::min(num_tiles, max_pair_clusters<A_MN, B_MN, KA, NH>());
  int32_t* err = device_error_word();
  if (!err) return fail(MT_ERR_CUDA, "device error word unavailable");
  gemm2_kernel<A_MN, B_MN, KA, NH><<<2 * clusters, threads2(NH), c2::SMEM_BYTES, st>>>(ta, tb, ep, err);
  return launch_check("gemm2_kernel");
}

// Pair-tile width. The 256 x 512 tile (NH = 2) measured 4-7% faster on the
// weight-gradient layout (both operands MN-major, K = tokens >= 16384, fp32 out),
// where a tile's main loop is long enough to hide its unbuffered epilogue, and
// 2-5% slower on the forward and input-gradient shapes of the layer with K = 3584.
// On the long-K forward / input-gradient launches (the down projection, K = F,
// and dh2 = dgu Wgu, K = 2F) it measured 10-13% faster at 98304 rows but 4%
// slower at 8192 (fewer tiles than two waves of clusters). So: the weight-gradient
// layout with K >= 8192, and any plain epilogue with K >= 8192 and M >= 65536.
// Every other launch runs the 256 x 256 tile with three stages of 128-wide K
// (eight MMAs per barrier round trip measured 7-16% faster than four).
// A launch whose wide tiles leave a last wave of clusters mostly idle (the
// 3584 x 3584 weight gradient: 98 tiles of 256 x 512 on 74 clusters, two waves,
// against 196 of 256 x 256 in three) runs the 256 x 256 tile: the wide tile is
// taken only while its waves of clusters, each costing about 1.8 narrow waves
// (it is 4-13% faster per FLOP), are not more than the narrow tile's.
template <bool A_MN, bool B_MN>
mt_status launch_2sm(const CUtensorMap& ta, const CUtensorMap& tb, EpiArgs ep, cudaStream_t st) {
  // 256-bit epilogue accesses where every 32-column row chunk is 32-byte aligned: the base pointer and
  // the row stride in bytes are multiples of 32 (chunks start every 32 columns)
  auto a32 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; };
  ep.c_v8 = ep.C && a32(ep.C) && (ep.ldc * (ep.c_f32 ? 4 : 2)) % 32 == 0;
  ep.res_v8 = ep.res && a32(ep.res) && (ep.ldr * 2) % 32 == 0;
  ep.gu_v8 = ep.gu && a32(ep.gu) && (ep.ld_gu * 2) % 32 == 0 && (static_cast<int64_t>(ep.F) * 2) % 32 == 0;
  const bool plain = ep.swiglu == 0 && !ep.rope_tab && !ep.dot_with;
  bool wide = plain && ep.K >= 8192 && ((A_MN && B_MN) || ep.M >= 65536);
  if (wide) {
    const int64_t num_m = (ep.M + c2::BM - 1) / c2::BM;
    const int64_t clusters = std::max(1, max_pair_clusters<A_MN, B_MN, 1, 2>());
    const int64_t waves_wide = (num_m * ((ep.N + 511) / 512) + clusters - 1) / clusters;
    const int64_t waves_narrow = (num_m * ((ep.N + 255) / 256) + clusters - 1) / clusters;
    wide = 18 * waves_wide <= 10 * waves_narrow;
  }
  if (wide) return launch_2sm_ka<A_MN, B_MN, 1, 2>(ta, tb, ep, st);
  return launch_2sm_ka<A_MN, B_MN, 2, 1>(ta, tb, ep, st);
}

// Tile order that keeps the smaller operand resident in L2 when it fits.
int pick_raster(int64_t M, int64_t N, int64_t K) {
  const int64_t l2_budget = 40ll << 20;
  if (N * K * 2 <= l2_budget) return 1;
  if (M * K * 2 <= l2_budget) return 2;
  return 0;
}

}  // namespace

namespace {

// Tensor maps for the operands, then the kernel chosen by layout, timed by the
// engine's observer. `ep` carries the epilogue; M, N, K come from it.
mt_status gemm_dispatch(const mt_bf16* A, int64_t lda, bool a_mn, const mt_bf16* B, int64_t ldb, bool b_mn,
                        EpiArgs ep, cudaStream_t st) {
  const int64_t M = ep.M, N = ep.N, K = ep.K;
  if (M == 0 || N == 0) return MT_OK;
  CUtensorMap ta, tb;
  if (!a_mn)
    MT_TRY(make_map(&ta, A, K, M, lda, 64, 128));
  else
    MT_TRY(make_map(&ta, A, M, K, lda, 64, 64));
  if (!b_mn)
    MT_TRY(make_map(&tb, B, K, N, ldb, 64, 128));
  else
    MT_TRY(make_map(&tb, B, N, K, ldb, 64, 64));
  ep.raster = pick_raster(M, N, K);
  const double flops = 2.0 * double(M) * double(N) * double(K);
  GemmTimer* tm = current_gemm_timer();
  if (tm) tm->before(st);
  mt_status s;
  if (!a_mn && !b_mn)
    s = launch_2sm<false, false>(ta, tb, ep, st);
  else if (!a_mn && b_mn)
    s = launch_2sm<false, true>(ta, tb, ep, st);
  else if (a_mn && !b_mn)
    s = launch_2sm<true, false>(ta, tb, ep, st);
  else
    s = launch_2sm<true, true>(ta, tb, ep, st);
  if (tm) tm->after(st, flops);
  add_exec_flops(flops);
  return s;
}

EpiArgs plain_epilogue(int64_t M, int64_t N, int64_t K) {
  EpiArgs ep;
  ep.C = nullptr;
  ep.bias = nullptr;
  ep.res = nullptr;
  ep.ldc = 0;
  ep.ldr = 0;
  ep.M = static_cast<int>(M);
  ep.N = static_cast<int>(N);
  ep.K = static_cast<int>(K);
  ep.c_f32 = 0;
  ep.accumulate = 0;
  ep.raster = 0;
  ep.swiglu = 0;
  ep.F = 0;
  ep.gu = nullptr;
  ep.ld_gu = 0;
  ep.c_v8 = ep.res_v8 = ep.gu_v8 = 0;
  ep.rope_tab = nullptr;
  ep.rope_cols = ep.rope_hd = ep.rope_T = 0;
  ep.dot_with = nullptr;
  ep.ld_dot = 0;
  ep.dot_out = nullptr;
  ep.dot_hd = ep.dot_T = ep.dot_heads = 0;
  return ep;
}

}  // namespace

mt_status gemm_launch(const mt_bf16* A, int64_t lda, bool a_mn, const mt_bf16* B, int64_t ldb, bool b_mn, void* C,
                      int64_t ldc, bool c_f32, bool accumulate, int64_t M, int64_t N, int64_t K,
                      const mt_bf16* bias, const mt_bf16* residual, int64_t ldr, cudaStream_t st) {
  EpiArgs ep = plain_epilogue(M, N, K);
  ep.C = C;
  ep.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
  ep.res = reinterpret_cast<const __nv_bfloat16*>(residual);
  ep.ldc = ldc;
  ep.ldr = ldr;
  ep.c_f32 = c_f32 ? 1 : 0;
  ep.accumulate = accumulate ? 1 : 0;
  return gemm_dispatch(A, lda, a_mn, B, ldb, b_mn, ep, st);
}

mt_status gemm_swiglu_bwd_launch(const mt_bf16* A, int64_t lda, bool a_mn, const mt_bf16* B, int64_t ldb, bool b_mn,
                                 mt_bf16* gu, int64_t ld_gu, int64_t M, int64_t F, int64_t K, cudaStream_t st) {
  EpiArgs ep = plain_epilogue(M, F, K);
  ep.swiglu = 2;
  ep.F = static_cast<int>(F);
  ep.gu = reinterpret_cast<__nv_bfloat16*>(gu);
  ep.ld_gu = ld_gu;
  return gemm_dispatch(A, lda, a_mn, B, ldb, b_mn, ep, st);
}

mt_status gemm_rope_launch(const mt_bf16* A, int64_t lda, const mt_bf16* B, int64_t ldb, mt_bf16* C, int64_t ldc,
                           int64_t M, int64_t N, int64_t K, const mt_bf16* bias, const float* rope_tab, int rope_cols,
                           int head_dim, int T, cudaStream_t st) {
  if (N % head_dim || rope_cols % head_dim || rope_cols > N || (head_dim != 64 && head_dim != 128) || T <= 0)
    return fail(MT_ERR_UNSUPPORTED, "RoPE epilogue: whole heads of 64 or 128 columns");
  EpiArgs ep = plain_epilogue(M, N, K);
  ep.C = C;
  ep.ldc = ldc;
  ep.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
  ep.rope_tab = reinterpret_cast<const float2*>(rope_tab);
  ep.rope_cols = rope_cols;
  ep.rope_hd = head_dim;
  ep.rope_T = T;
  return gemm_dispatch(A, lda, false, B, ldb, false, ep, st);
}

mt_status gemm_dot_launch(const mt_bf16* A, int64_t lda, bool a_mn, const mt_bf16* B, int64_t ldb, bool b_mn,
                          mt_bf16* C, int64_t ldc, int64_t M, int64_t N, int64_t K, const mt_bf16* dot_with,
                          int64_t ld_dot, float* dot_out, int head_dim, int T, cudaStream_t st) {
  if (N % head_dim || (head_dim != 64 && head_dim != 128) || T <= 0 || M % T)
    return fail(MT_ERR_UNSUPPORTED, "dot epilogue: whole heads of 64 or 128 and whole sequences");
  EpiArgs ep = plain_epilogue(M, N, K);
  ep.C = C;
  ep.ldc = ldc;
  ep.dot_with = reinterpret_cast<const __nv_bfloat16*>(dot_with);
  ep.ld_dot = ld_dot;
  ep.dot_out = dot_out;
  ep.dot_hd = head_dim;
  ep.dot_T = T;
  ep.dot_heads = static_cast<int>(N / head_dim);
  return gemm_dispatch(A, lda, a_mn, B, ldb, b_mn, ep, st);
}

mt_status tma_map_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                     uint32_t box_inner, uint32_t box_outer) {
  return make_map(m, ptr, inner, outer, ld_elems, box_inner, box_outer);
}

mt_status gemm_swiglu_launch(const mt_bf16* A, int64_t lda, const mt_bf16* Wgu, int64_t ldw, mt_bf16* m, int64_t ldm,
                             mt_bf16* gu, int64_t ld_gu, int64_t M, int64_t F, int64_t K, cudaStream_t st) {
  if (M == 0 || F == 0) return MT_OK;
  CUtensorMap ta, tb;
  MT_TRY(make_map(&ta, A, K, M, lda, 64, 128));
  MT_TRY(make_map(&tb, Wgu, K, 2 * F, ldw, 64, 128));
  EpiArgs ep = plain_epilogue(M, 2 * F, K);
  ep.C = m;
  ep.ldc = ldm;
  ep.raster = pick_raster(M, 2 * F, K);
  ep.swiglu = 1;
  ep.F = static_cast<int>(F);
  ep.gu = reinterpret_cast<__nv_bfloat16*>(gu);
  ep.ld_gu = ld_gu;
  const double flops = 2.0 * double(M) * double(2 * F) * double(K);
  GemmTimer* tm = current_gemm_timer();
  if (tm) tm->before(st);
  mt_status s = launch_2sm<false, false>(ta, tb, ep, st);
  if (tm) tm->after(st, flops);
  add_exec_flops(flops);
  return s;
}

}  // namespace mt

using namespace mt;

extern "C" mt_status mt_gemm_bf16(const mt_bf16* A, int64_t lda, int32_t a_mn_major, const mt_bf16* Bm, int64_t ldb,
                                  int32_t b_mn_major, void* C, int64_t ldc, int32_t c_f32, int32_t accumulate,
                                  int64_t M, int64_t N, int64_t K, const mt_bf16* bias, const mt_bf16* residual,
                                  int64_t ldr, void* stream) {
  if (!A || !Bm || !C) return fail(MT_ERR_INVALID_ARG, "A, B and C must not be NULL");
  if (M < 0 || N < 0 || K <= 0) return fail(MT_ERR_INVALID_ARG, "need M, N >= 0 and K > 0");
  if (M >= (1ll << 31) || N >= (1ll << 31) || K >= (1ll << 31)) return fail(MT_ERR_INVALID_ARG, "dimension too large");
  if (accumulate && !c_f32) return fail(MT_ERR_INVALID_ARG, "accumulate needs an fp32 C");
  const int64_t a_inner = a_mn_major ? M : K, b_inner = b_mn_major ? N : K;
  if (lda < a_inner || ldb < b_inner || ldc < N || (residual && ldr < N))
    return fail(MT_ERR_INVALID_ARG, "leading dimension smaller than the row it holds");
  if (!aligned16(A) || !aligned16(Bm) || !aligned16(C) || (bias && !aligned16(bias)) ||
      (residual && !aligned16(residual)))
    return fail(MT_ERR_ALIGNMENT, "gemm pointers must be 16-byte aligned");
  if (lda % 8 || ldb % 8 || ldc % 8 || (residual && ldr % 8))
    return fail(MT_ERR_ALIGNMENT, "leading dimensions must be multiples of 8 elements");
  return gemm_launch(A, lda, a_mn_major != 0, Bm, ldb, b_mn_major != 0, C, ldc, c_f32 != 0, accumulate != 0, M, N, K,
                     bias, residual, ldr, as_stream(stream));
}

extern "C" mt_status mt_gemm_swiglu_bf16(const mt_bf16* A, int64_t lda, const mt_bf16* Wgu, int64_t ldw, mt_bf16* m,
                                         int64_t ldm, mt_bf16* gu, int64_t ld_gu, int64_t M, int64_t F, int64_t K,
                                         void* stream) {
  if (!A || !Wgu || !m) return fail(MT_ERR_INVALID_ARG, "gemm_swiglu: A, Wgu and m must not be NULL");
  if (M < 0 || F < 0 || K <= 0 || M >= (1ll << 31) || 2 * F >= (1ll << 31) || K >= (1ll << 31))
    return fail(MT_ERR_INVALID_ARG, "gemm_swiglu: bad sizes");
  if (lda < K || ldw < K || ldm < F || (gu && ld_gu < 2 * F))
    return fail(MT_ERR_INVALID_ARG, "gemm_swiglu: leading dimension smaller than the row it holds");
  if (!aligned16(A) || !aligned16(Wgu) || !aligned16(m) || (gu && !aligned16(gu)) || lda % 8 || ldw % 8 || ldm % 8 ||
      F % 8 || (gu && ld_gu % 8))
    return fail(MT_ERR_ALIGNMENT, "gemm_swiglu: 16-byte alignment of pointers, rows and F");
  return gemm_swiglu_launch(A, lda, Wgu, ldw, m, ldm, gu, ld_gu, M, F, K, as_stream(stream));
}

extern "C" mt_status mt_gemm_swiglu_bwd_bf16(const mt_bf16* dY, int64_t ld_dy, const mt_bf16* Wd, int64_t ldw,
                                             mt_bf16* gu, int64_t ld_gu, int64_t M, int64_t F, int64_t K,
                                             void* stream) {
  if (!dY || !Wd || !gu) return fail(MT_ERR_INVALID_ARG, "gemm_swiglu_bwd: dY, Wd and gu must not be NULL");
  if (M < 0 || F <= 0 || K <= 0 || M >= (1ll << 31) || F >= (1ll << 30) || K >= (1ll << 31))
    return fail(MT_ERR_INVALID_ARG, "gemm_swiglu_bwd: bad sizes");
  if (ld_dy < K || ldw < F || ld_gu < 2 * F)
    return fail(MT_ERR_INVALID_ARG, "gemm_swiglu_bwd: leading dimension smaller than the row it holds");
  if (!aligned16(dY) || !aligned16(Wd) || !aligned16(gu) || ld_dy % 8 || ldw % 8 || ld_gu % 8 || F % 8)
    return fail(MT_ERR_ALIGNMENT, "gemm_swiglu_bwd: 16-byte alignment of pointers, rows and F");
  return gemm_swiglu_bwd_launch(dY, ld_dy, false, Wd, ldw, true, gu, ld_gu, M, F, K, as_stream(stream));
}
