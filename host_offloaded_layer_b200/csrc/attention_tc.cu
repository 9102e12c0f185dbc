// Causal grouped-query flash attention forward on the sm_100a tensor cores
// (head_dim 128): S = Q K^T and O += P V are tcgen05.mma with both
// accumulators in tensor memory, the operands staged by TMA.
//
// One CTA per (128 query rows, query head, sequence):
//   warp 0     TMA: Q once, then K_j and V_j (128 key rows each) into a
//              two-stage ring;
//   warp 1     TMEM allocation and the MMA issuer: S_{j+1} = Q K_{j+1}^T is
//              issued before O += P_j V_j so the tensor cores work while the
//              softmax of block j runs;
//   warps 2-5  softmax, one thread per query row: S row from TMEM, online
//              softmax in the log2 domain, P (bf16) written to shared memory
//              in the 128-byte-swizzled K-major layout the next MMA reads,
//              then the final O / l and the log-sum-exp.
// TMEM: two S buffers (128 columns each) and O (128 columns). O is rescaled
// only when a row's running maximum grows by more than 8 (a factor 256 in
// the exponent); otherwise the stale maximum stays, which keeps P <= 256 and
// the result exact up to rounding (the final division uses the same
// maximum as every P). Every mbarrier wait is bounded.
#include <mutex>

#include "mt_internal.h"
#include "tcgen05.cuh"

namespace mt {
namespace {

using namespace tc;

constexpr int D = 128, BQ = 128, BKV = 128;
constexpr int TILE = BQ * D * 2;  // 32 KiB: a 128 x 128 bf16 tile (two 64-column swizzle atoms)
constexpr int ATOM = 128 * 64 * 2;  // 16 KiB
// shared memory: Q | K0 V0 | K1 V1 | P0 | P1
constexpr int OFF_Q = 0, OFF_KV = TILE, OFF_P = 5 * TILE;
constexpr int SMEM_TILES = 7 * TILE;
constexpr int SMEM_BYTES = SMEM_TILES + 256 + 1024;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S0 = 0, COL_O = 256;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, __nv_bfloat16* __restrict__ o, int64_t ld_o,
                       float* __restrict__ lse, int T, int nq, int nkv, float scale_log2, int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_TILES);
  uint64_t* q_full = bars;          // 1
  uint64_t* kv_full = bars + 1;     // 2
  uint64_t* kv_empty = bars + 3;    // 2
  uint64_t* s_full = bars + 5;      // 2
  uint64_t* p_full = bars + 7;      // 2
  uint64_t* o_done = bars + 9;      // 2
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int qb = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int c = (h * nkv) / nq;
  const int q0 = qb * BQ;
  const int n_kv = min((T + BKV - 1) / BKV, qb + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = b * T;  // first row of this sequence in the [B*T, ld] qkv array
  const int col_q = h * D, col_k = (nq + c) * D, col_v = (nq + nkv + c) * D;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&kv_full[i]), 1);
      mbar_init(smem_u32(&kv_empty[i]), 1);
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&p_full[i]), 128);
      mbar_init(smem_u32(&o_done[i]), 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_qkv)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t qb_bar = smem_u32(q_full);
      mbar_expect_tx(qb_bar, TILE);
      tma_load_2d(smem_u32(smem + OFF_Q), &tm_qkv, qb_bar, col_q, row0 + q0);
      tma_load_2d(smem_u32(smem + OFF_Q + ATOM), &tm_qkv, qb_bar, col_q + 64, row0 + q0);
    }
    __syncwarp();
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      if (!warp_wait(smem_u32(&kv_empty[s]), ((j >> 1) & 1) ^ 1, abort_flag, err, DEV_ERR_TIMEOUT_PRODUCER)) break;
      if (lane == 0) {
        const uint32_t fb = smem_u32(&kv_full[s]);
        uint8_t* kt = smem + OFF_KV + s * 2 * TILE;
        uint8_t* vt = kt + TILE;
        const int r = row0 + j * BKV;
        mbar_expect_tx(fb, 2 * TILE);
        tma_load_2d(smem_u32(kt), &tm_qkv, fb, col_k, r);
        tma_load_2d(smem_u32(kt + ATOM), &tm_qkv, fb, col_k + 64, r);
        tma_load_2d(smem_u32(vt), &tm_qkv, fb, col_v, r);
        tma_load_2d(smem_u32(vt + ATOM), &tm_qkv, fb, col_v + 64, r);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, BKV, false, false);  // S = Q K^T: both K-major
    constexpr uint32_t idesc_o = idesc_bf16(128, D, false, true);     // O += P V: V is MN-major (d contiguous)
    const uint32_t q_base = smem_u32(smem + OFF_Q);
    bool ok = warp_wait(smem_u32(q_full), 0, abort_flag, err, DEV_ERR_TIMEOUT_MMA);
    auto issue_s = [&](int j) -> bool {
      const int s = j & 1;
      if (!warp_wait(smem_u32(&kv_full[s]), (j >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) return false;
      fence_after();
      if (lane == 0) {
        const uint32_t k_base = smem_u32(smem + OFF_KV + s * 2 * TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk >> 2) * ATOM + (kk & 3) * 32);
          umma_bf16(tmem + COL_S0 + s * BKV, smem_desc(q_base + off, 16, 1024), smem_desc(k_base + off, 16, 1024),
                    idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(smem_u32(&s_full[s]));
      }
      __syncwarp();
      return true;
    };
    if (ok) ok = issue_s(0);
    for (int j = 0; j < n_kv && ok; ++j) {
      const int s = j & 1;
      if (j + 1 < n_kv && !issue_s(j + 1)) break;
      if (!warp_wait(smem_u32(&p_full[s]), (j >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) break;
      fence_after();
      if (lane == 0) {
        const uint32_t p_base = smem_u32(smem + OFF_P + s * TILE);
        const uint32_t v_base = smem_u32(smem + OFF_KV + s * 2 * TILE + TILE);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint32_t poff = static_cast<uint32_t>((kk >> 2) * ATOM + (kk & 3) * 32);
          umma_bf16(tmem + COL_O, smem_desc(p_base + poff, 16, 1024), smem_desc(v_base + kk * 2048, ATOM, 1024),
                    idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&o_done[s]));
        umma_commit(smem_u32(&kv_empty[s]));
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax (one thread per query row)
    const int qw = warp & 3;  // TMEM lanes [32 qw, 32 qw + 32)
    const int r = qw * 32 + lane;
    const int q_row = q0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(qw * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      if (!warp_wait(smem_u32(&s_full[s]), (j >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
        ok = false;
        break;
      }
      fence_after();
      float sv[BKV];
#pragma unroll
      for (int ch = 0; ch < BKV / 32; ++ch) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_base + COL_S0 + s * BKV + ch * 32, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[ch * 32 + e] = __uint_as_float(u[e]);
      }
      const int k0 = j * BKV;
      const bool diag = k0 + BKV - 1 > q0;
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < BKV; ++e) {
        float v = sv[e] * scale_log2;
        if (diag && k0 + e > q_row) v = -INFINITY;
        sv[e] = v;
        mx = fmaxf(mx, v);
      }
      // rescale O only when some row of the warp raised its maximum by more than the threshold
      const bool need = (m_run == -INFINITY) || (mx > m_run + RESCALE_THRESHOLD);
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = fmaxf(m_run, mx);
        const float alpha = exp2f(m_run - m_new);  // 0 for the first block
        if (j > 0) {
          // O must hold P_{j-1} V_{j-1} before it is rescaled
          if (!warp_wait(smem_u32(&o_done[(j - 1) & 1]), ((j - 1) >> 1) & 1, abort_flag, err,
                         DEV_ERR_TIMEOUT_EPILOGUE)) {
            ok = false;
            break;
          }
          fence_after();
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t u[32];
            tmem_ld32(tmem + lane_base + COL_O + ch * 32, u);
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
            tmem_st32(tmem + lane_base + COL_O + ch * 32, u);
          }
        }
        l_run *= alpha;
        m_run = m_new;
      }
      // P_{j-2} V_{j-2} must be done reading P buffer s before it is overwritten
      if (j >= 2) {
        if (!warp_wait(smem_u32(&o_done[s]), ((j - 2) >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
          ok = false;
          break;
        }
      }
      uint8_t* prow = smem + OFF_P + s * TILE + r * 128;
      float lsum = 0.f;
#pragma unroll
      for (int ch = 0; ch < BKV / 8; ++ch) {  // 16-byte chunks of 8 columns
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = exp2f(sv[ch * 8 + e] - m_run);
          lsum += p[e];
        }
        uint4 w;
        w.x = pack_bf16(p[0], p[1]);
        w.y = pack_bf16(p[2], p[3]);
        w.z = pack_bf16(p[4], p[5]);
        w.w = pack_bf16(p[6], p[7]);
        const int atom = ch >> 3, c16 = ch & 7;
        *reinterpret_cast<uint4*>(prow + atom * ATOM + ((c16 ^ (r & 7)) << 4)) = w;
      }
      l_run += lsum;
      fence_proxy_async_smem();
      fence_before();
      mbar_arrive(smem_u32(&p_full[s]));
    }
    if (ok && n_kv > 0) {
      const int jl = n_kv - 1;
      if (warp_wait(smem_u32(&o_done[jl & 1]), (jl >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
        fence_after();
        const float inv = 1.f / l_run;
        __nv_bfloat16* orow = o + (static_cast<int64_t>(row0) + q_row) * ld_o + static_cast<int64_t>(h) * D;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t u[32];
          tmem_ld32(tmem + lane_base + COL_O + ch * 32, u);
          if (q_row < T) {
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(u[qd * 8 + 0]) * inv, __uint_as_float(u[qd * 8 + 1]) * inv);
              w.y = pack_bf16(__uint_as_float(u[qd * 8 + 2]) * inv, __uint_as_float(u[qd * 8 + 3]) * inv);
              w.z = pack_bf16(__uint_as_float(u[qd * 8 + 4]) * inv, __uint_as_float(u[qd * 8 + 5]) * inv);
              w.w = pack_bf16(__uint_as_float(u[qd * 8 + 6]) * inv, __uint_as_float(u[qd * 8 + 7]) * inv);
              *reinterpret_cast<uint4*>(orow + ch * 32 + qd * 8) = w;
            }
          }
        }
        if (q_row < T) lse[(static_cast<int64_t>(b) * nq + h) * T + q_row] = (m_run + log2f(l_run)) * LN2;
      }
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace

// Launches the tcgen05 forward (head_dim 128). qkv must be 16-byte aligned with
// ld_qkv a multiple of 8 (checked by the caller).
mt_status attn_fwd_tc_launch(const mt_bf16* qkv, int64_t ld, mt_bf16* o, int64_t ld_o, float* lse, int B, int T,
                             int nq, int nkv, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  if (attr != cudaSuccess) return fail(MT_ERR_CUDA, "attention smem attribute: %s", cudaGetErrorString(attr));
  CUtensorMap tm;
  MT_TRY(tma_map_2d(&tm, qkv, static_cast<uint64_t>((nq + 2 * nkv) * D), static_cast<uint64_t>(B) * T,
                    static_cast<uint64_t>(ld), 64, 128));
  int32_t* err = device_error_word();
  if (!err) return fail(MT_ERR_CUDA, "device error word unavailable");
  dim3 grid((T + BQ - 1) / BQ, nq, B);
  const float scale_log2 = LOG2E / sqrtf(static_cast<float>(D));
  attn_fwd_tc_kernel<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(tm, reinterpret_cast<__nv_bfloat16*>(o), ld_o, lse, T, nq,
                                                            nkv, scale_log2, err);
  MT_TRY(launch_check("attn_fwd_tc_kernel"));
  add_exec_flops(4.0 * B * nq * D * (0.5 * double(T) * double(T)));
  return MT_OK;
}

}  // namespace mt
