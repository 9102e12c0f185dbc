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
constexpr int SMEM_BYTES = SMEM_TILES + 128 + 1024 + 1024;  // tiles, barriers, row exchange, alignment
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S0 = 0, COL_O = 256;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;

// Bounded barrier among a group of threads built on an mbarrier initialised
// with the group's size: arrive, then wait (bounded) for the phase to flip.
// `phase` counts this thread's uses. Returns false when the wait ran out.
__device__ __forceinline__ bool group_sync(uint32_t bar, uint32_t& phase, volatile int* abort_flag, int32_t* err) {
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase & 1u, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE);
  ++phase;
  return ok;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// NG softmax warpgroups: with NG = 2, warps 2-5 take key columns 0-63 (and O
// columns 0-63) of the 128 rows, warps 6-9 columns 64-127 of the same rows;
// the two halves of each row maximum and row sum meet in shared memory.
template <int NG>
__global__ void __launch_bounds__(64 + 128 * NG, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, __nv_bfloat16* __restrict__ o, int64_t ld_o,
                       float* __restrict__ lse, int T, int nq, int nkv, float scale_log2, int32_t* err) {
  constexpr int SCOLS = BKV / NG, OCOLS = D / NG;  // S and O columns per softmax group
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_TILES);
  uint64_t* q_full = bars;          // 1
  uint64_t* kv_full = bars + 1;     // 2
  uint64_t* kv_empty = bars + 3;    // 2
  uint64_t* s_full = bars + 5;      // 2
  uint64_t* p_full = bars + 7;      // 2
  uint64_t* o_done = bars + 9;      // 2
  uint64_t* x_bar = bars + 11;      // 1: row exchange between the softmax groups
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xch = reinterpret_cast<float*>(smem + SMEM_TILES + 128);  // [NG][128] row halves

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
      mbar_init(smem_u32(&p_full[i]), 128 * NG);
      mbar_init(smem_u32(&o_done[i]), 1);
    }
    mbar_init(smem_u32(x_bar), 128 * NG);
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
    // ------------------------------------------------------------ softmax (one thread per query row and group)
    const int g = (warp - 2) >> 2;  // softmax group: columns [g*SCOLS, (g+1)*SCOLS) of S
    const int qw = warp & 3;        // TMEM lanes [32 qw, 32 qw + 32)
    const int r = qw * 32 + lane;
    const int q_row = q0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(qw * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    uint32_t xph = 0;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      if (!warp_wait(smem_u32(&s_full[s]), (j >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
        ok = false;
        break;
      }
      fence_after();
      float sv[SCOLS];
#pragma unroll
      for (int ch = 0; ch < SCOLS / 32; ++ch) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_base + COL_S0 + s * BKV + g * SCOLS + ch * 32, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[ch * 32 + e] = __uint_as_float(u[e]);
      }
      const int k0 = j * BKV + g * SCOLS;
      const bool diag = k0 + SCOLS - 1 > q0;
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < SCOLS; ++e) {
        float v = sv[e] * scale_log2;
        if (diag && k0 + e > q_row) v = -INFINITY;
        sv[e] = v;
        mx = fmaxf(mx, v);
      }
      if (NG == 2) {  // the other half of the row's maximum
        xch[g * 128 + r] = mx;
        if (!group_sync(smem_u32(x_bar), xph, abort_flag, err)) {
          ok = false;
          break;
        }
        mx = fmaxf(mx, xch[(g ^ 1) * 128 + r]);
        if (!group_sync(smem_u32(x_bar), xph, abort_flag, err)) {  // both halves read before the next write
          ok = false;
          break;
        }
      }
      // rescale O only when some row of the warp raised its maximum by more than the threshold
      // (the decision is the same in both groups: it depends on the row maximum only)
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
          for (int ch = 0; ch < OCOLS / 32; ++ch) {
            uint32_t u[32];
            const uint32_t col = COL_O + g * OCOLS + ch * 32;
            tmem_ld32(tmem + lane_base + col, u);
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
            tmem_st32(tmem + lane_base + col, u);
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
      for (int ch = 0; ch < SCOLS / 8; ++ch) {  // 16-byte chunks of 8 columns
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
        const int cg = g * (SCOLS / 8) + ch;  // chunk index within the row of 128 columns
        const int atom = cg >> 3, c16 = cg & 7;
        *reinterpret_cast<uint4*>(prow + atom * ATOM + ((c16 ^ (r & 7)) << 4)) = w;
      }
      l_run += lsum;
      fence_proxy_async_smem();
      fence_before();
      mbar_arrive(smem_u32(&p_full[s]));
    }
    float l_tot = l_run;
    if (NG == 2 && ok) {
      xch[g * 128 + r] = l_run;
      ok = group_sync(smem_u32(x_bar), xph, abort_flag, err);
      l_tot = l_run + xch[(g ^ 1) * 128 + r];
    }
    if (ok && n_kv > 0) {
      const int jl = n_kv - 1;
      if (warp_wait(smem_u32(&o_done[jl & 1]), (jl >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
        fence_after();
        const float inv = 1.f / l_tot;
        __nv_bfloat16* orow = o + (static_cast<int64_t>(row0) + q_row) * ld_o + static_cast<int64_t>(h) * D;
#pragma unroll
        for (int ch = 0; ch < OCOLS / 32; ++ch) {
          uint32_t u[32];
          const int oc = g * OCOLS + ch * 32;
          tmem_ld32(tmem + lane_base + COL_O + oc, u);
          if (q_row < T) {
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(u[qd * 8 + 0]) * inv, __uint_as_float(u[qd * 8 + 1]) * inv);
              w.y = pack_bf16(__uint_as_float(u[qd * 8 + 2]) * inv, __uint_as_float(u[qd * 8 + 3]) * inv);
              w.z = pack_bf16(__uint_as_float(u[qd * 8 + 4]) * inv, __uint_as_float(u[qd * 8 + 5]) * inv);
              w.w = pack_bf16(__uint_as_float(u[qd * 8 + 6]) * inv, __uint_as_float(u[qd * 8 + 7]) * inv);
              *reinterpret_cast<uint4*>(orow + oc + qd * 8) = w;
            }
          }
        }
        if (q_row < T && g == 0) lse[(static_cast<int64_t>(b) * nq + h) * T + q_row] = (m_run + log2f(l_tot)) * LN2;
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
  constexpr int NG = 2;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(attn_fwd_tc_kernel<NG>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  if (attr != cudaSuccess) return fail(MT_ERR_CUDA, "attention smem attribute: %s", cudaGetErrorString(attr));
  CUtensorMap tm;
  MT_TRY(tma_map_2d(&tm, qkv, static_cast<uint64_t>((nq + 2 * nkv) * D), static_cast<uint64_t>(B) * T,
                    static_cast<uint64_t>(ld), 64, 128));
  int32_t* err = device_error_word();
  if (!err) return fail(MT_ERR_CUDA, "device error word unavailable");
  dim3 grid((T + BQ - 1) / BQ, nq, B);
  const float scale_log2 = LOG2E / sqrtf(static_cast<float>(D));
  attn_fwd_tc_kernel<NG><<<grid, 64 + 128 * NG, SMEM_BYTES, st>>>(tm, reinterpret_cast<__nv_bfloat16*>(o), ld_o, lse,
                                                                  T, nq, nkv, scale_log2, err);
  MT_TRY(launch_check("attn_fwd_tc_kernel"));
  add_exec_flops(4.0 * B * nq * D * (0.5 * double(T) * double(T)));
  return MT_OK;
}

}  // namespace mt

// ============================================================== backward
// Two deterministic kernels on the tensor cores (no atomics): dK/dV per block
// of 128 key rows (looping over the group's query heads in order and over
// 64-row query blocks from the diagonal on) and dQ per block of 128 query
// rows (looping over 64-row key blocks up to the diagonal). Both recompute
// S and dP with tcgen05.mma into double-buffered TMEM, so the MMAs of the
// next block run while one thread per row turns the current block into
// P and dS (bf16, written to shared memory in the swizzled K-major layout
// that the following MMAs read).
namespace mt {
namespace {

constexpr int HALF_TILE = 64 * D * 2;      // 16 KiB: 64 rows x 128 columns
constexpr int HALF_ATOM = 64 * 64 * 2;     // 8 KiB: 64 rows of one 64-column atom

// ------------------------------------------------------------ dK, dV
// smem: K | V | Q0 dO0 | Q1 dO1 | PT0 DST0 | PT1 DST1 | lse/delta [2][2][64]
constexpr int KV_OFF_K = 0, KV_OFF_V = TILE, KV_OFF_QO = 2 * TILE, KV_OFF_PD = 2 * TILE + 4 * HALF_TILE;
constexpr int KV_OFF_LD = KV_OFF_PD + 4 * ATOM;
constexpr int KV_SMEM_TILES = KV_OFF_LD + 4 * 64 * 4;
constexpr int KV_SMEM_BYTES = KV_SMEM_TILES + 256 + 1024;
constexpr uint32_t KV_COL_ST = 0, KV_COL_DPT = 128, KV_COL_DV = 256, KV_COL_DK = 384;
// Both backward kernels run two groups of four compute warps (warps 2-5 and 6-9),
// each on half of a block's 64 columns: no row reduction crosses the halves.
constexpr int BWD_THREADS = 64 + 256;

__global__ void __launch_bounds__(BWD_THREADS, 1)
    attn_bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_kv128, const __grid_constant__ CUtensorMap tm_q64,
                           const __grid_constant__ CUtensorMap tm_do64, const float* __restrict__ lse,
                           const float* __restrict__ delta, __nv_bfloat16* __restrict__ dqkv, int64_t ld, int T,
                           int nq, int nkv, float scale_log2, float scale, int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* lsd = reinterpret_cast<float*>(smem + KV_OFF_LD);  // [stage][lse2 | delta][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + KV_SMEM_TILES);
  uint64_t* kv_full = bars;       // 1
  uint64_t* qo_full = bars + 1;   // 2
  uint64_t* qo_empty = bars + 3;  // 2
  uint64_t* sp_full = bars + 5;   // 2
  uint64_t* pd_full = bars + 7;   // 2
  uint64_t* mma_done = bars + 9;  // 2
  uint64_t* fin = bars + 11;      // 1
  uint64_t* l_bar = bars + 12;    // 1: lse/delta of a block written by the 128 compute threads
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int kb = blockIdx.x;  // small key blocks have the most query blocks: first
  const int c = blockIdx.y, b = blockIdx.z;
  const int grp = nq / nkv;
  const int k0 = kb * 128;
  const int row0 = b * T;
  const int n_qb = (T + 63) / 64;
  const int qb0 = k0 / 64;
  const int per_head = n_qb - qb0;
  const int n_it = grp * per_head;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col_k = (nq + c) * D, col_v = (nq + nkv + c) * D;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(kv_full), 1);
    mbar_init(smem_u32(fin), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&qo_full[i]), 1);
      mbar_init(smem_u32(&qo_empty[i]), 1);
      mbar_init(smem_u32(&sp_full[i]), 1);
      mbar_init(smem_u32(&pd_full[i]), 256);
      mbar_init(smem_u32(&mma_done[i]), 1);
    }
    mbar_init(smem_u32(l_bar), 256);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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
    if (lane == 0 && n_it > 0) {
      const uint32_t fb = smem_u32(kv_full);
      mbar_expect_tx(fb, 2 * TILE);
      tma_load_2d(smem_u32(smem + KV_OFF_K), &tm_kv128, fb, col_k, row0 + k0);
      tma_load_2d(smem_u32(smem + KV_OFF_K + ATOM), &tm_kv128, fb, col_k + 64, row0 + k0);
      tma_load_2d(smem_u32(smem + KV_OFF_V), &tm_kv128, fb, col_v, row0 + k0);
      tma_load_2d(smem_u32(smem + KV_OFF_V + ATOM), &tm_kv128, fb, col_v + 64, row0 + k0);
    }
    __syncwarp();
    for (int it = 0; it < n_it; ++it) {
      const int st = it & 1;
      if (!warp_wait(smem_u32(&qo_empty[st]), ((it >> 1) & 1) ^ 1, abort_flag, err, DEV_ERR_TIMEOUT_PRODUCER)) break;
      if (lane == 0) {
        const int h = c * grp + it / per_head;
        const int q0 = (qb0 + it % per_head) * 64;
        const uint32_t fb = smem_u32(&qo_full[st]);
        uint8_t* qt = smem + KV_OFF_QO + st * 2 * HALF_TILE;
        uint8_t* ot = qt + HALF_TILE;
        mbar_expect_tx(fb, 2 * HALF_TILE);
        tma_load_2d(smem_u32(qt), &tm_q64, fb, h * D, row0 + q0);
        tma_load_2d(smem_u32(qt + HALF_ATOM), &tm_q64, fb, h * D + 64, row0 + q0);
        tma_load_2d(smem_u32(ot), &tm_do64, fb, h * D, row0 + q0);
        tma_load_2d(smem_u32(ot + HALF_ATOM), &tm_do64, fb, h * D + 64, row0 + q0);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_sp = idesc_bf16(128, 64, false, false);  // S^T = K Q^T, dP^T = V dO^T
    constexpr uint32_t idesc_acc = idesc_bf16(128, D, false, true);   // dV += P^T dO, dK += dS^T Q
    const uint32_t k_base = smem_u32(smem + KV_OFF_K), v_base = smem_u32(smem + KV_OFF_V);
    bool ok = n_it == 0 || warp_wait(smem_u32(kv_full), 0, abort_flag, err, DEV_ERR_TIMEOUT_MMA);
    auto issue_sp = [&](int it) -> bool {
      const int st = it & 1;
      if (!warp_wait(smem_u32(&qo_full[st]), (it >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) return false;
      fence_after();
      if (lane == 0) {
        const uint32_t q_base = smem_u32(smem + KV_OFF_QO + st * 2 * HALF_TILE);
        const uint32_t o_base = q_base + HALF_TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off_a = static_cast<uint32_t>((kk >> 2) * ATOM + (kk & 3) * 32);
          const uint32_t off_b = static_cast<uint32_t>((kk >> 2) * HALF_ATOM + (kk & 3) * 32);
          umma_bf16(tmem + KV_COL_ST + st * 64, smem_desc(k_base + off_a, 16, 1024),
                    smem_desc(q_base + off_b, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
          umma_bf16(tmem + KV_COL_DPT + st * 64, smem_desc(v_base + off_a, 16, 1024),
                    smem_desc(o_base + off_b, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
        }
        umma_commit(smem_u32(&sp_full[st]));
      }
      __syncwarp();
      return true;
    };
    if (ok && n_it > 0) ok = issue_sp(0);
    for (int it = 0; it < n_it && ok; ++it) {
      const int st = it & 1;
      if (it + 1 < n_it && !issue_sp(it + 1)) {
        ok = false;
        break;
      }
      if (!warp_wait(smem_u32(&pd_full[st]), (it >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) {
        ok = false;
        break;
      }
      fence_after();
      if (lane == 0) {
        const uint32_t q_base = smem_u32(smem + KV_OFF_QO + st * 2 * HALF_TILE);
        const uint32_t o_base = q_base + HALF_TILE;
        const uint32_t pt = smem_u32(smem + KV_OFF_PD + st * 2 * ATOM);
        const uint32_t dst = pt + ATOM;
#pragma unroll
        for (int kk = 0; kk < 64 / 16; ++kk) {
          const uint32_t off_a = static_cast<uint32_t>(kk * 32);
          umma_bf16(tmem + KV_COL_DV, smem_desc(pt + off_a, 16, 1024), smem_desc(o_base + kk * 2048, HALF_ATOM, 1024),
                    idesc_acc, (it > 0 || kk > 0) ? 1u : 0u);
          umma_bf16(tmem + KV_COL_DK, smem_desc(dst + off_a, 16, 1024), smem_desc(q_base + kk * 2048, HALF_ATOM, 1024),
                    idesc_acc, (it > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&qo_empty[st]));
        umma_commit(smem_u32(&mma_done[st]));
      }
      __syncwarp();
    }
    if (lane == 0) umma_commit(smem_u32(fin));
    __syncwarp();
  } else {
    // ------------------------------------------------------------ P^T / dS^T, one thread per key row and group
    const int g = (warp - 2) >> 2;  // query columns [32 g, 32 g + 32) of each 64-column block
    const int qw = warp & 3;
    const int r = qw * 32 + lane;  // key row within the block
    const int t = threadIdx.x - 64;  // 0..255 among the compute threads
    const int kv_row = k0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(qw * 32) << 16;
    uint32_t lph = 0;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int st = it & 1;
      const int h = c * grp + it / per_head;
      const int q0 = (qb0 + it % per_head) * 64;
      {  // this block's log-sum-exp (log2 domain) and delta, shared by all key rows
        if (t < 128) {
          const int q = q0 + (t & 63);
          const int64_t sb = (static_cast<int64_t>(b) * nq + h) * T;
          if (t < 64)
            lsd[st * 128 + t] = q < T ? lse[sb + q] * LOG2E : INFINITY;
          else
            lsd[st * 128 + t] = q < T ? delta[sb + q] : 0.f;
        }
        if (!group_sync(smem_u32(l_bar), lph, abort_flag, err)) {
          ok = false;
          break;
        }
      }
      if (!warp_wait(smem_u32(&sp_full[st]), (it >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
        ok = false;
        break;
      }
      fence_after();
      float sv[32], dv[32];
      {
        uint32_t u[32];
        tmem_ld32(tmem + lane_base + KV_COL_ST + st * 64 + g * 32, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[e] = __uint_as_float(u[e]);
        tmem_ld32(tmem + lane_base + KV_COL_DPT + st * 64 + g * 32, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) dv[e] = __uint_as_float(u[e]);
      }
      const float* L2 = lsd + st * 128 + g * 32;
      const float* Dl = L2 + 64;
      const int qc0 = q0 + g * 32;
      const bool diag = qc0 < k0 + 127;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        float p = exp2f(sv[e] * scale_log2 - L2[e]);
        if (diag && kv_row > qc0 + e) p = 0.f;
        sv[e] = p;
        dv[e] = p * (dv[e] - Dl[e]);
      }
      if (it >= 2) {  // the dV/dK MMAs of it-2 must be done reading this P^T / dS^T buffer
        if (!warp_wait(smem_u32(&mma_done[st]), ((it - 2) >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
          ok = false;
          break;
        }
      }
      uint8_t* prow = smem + KV_OFF_PD + st * 2 * ATOM + r * 128;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const int c16 = g * 4 + ch;
        uint4 wp, wd;
        wp.x = pack_bf16(sv[ch * 8 + 0], sv[ch * 8 + 1]);
        wp.y = pack_bf16(sv[ch * 8 + 2], sv[ch * 8 + 3]);
        wp.z = pack_bf16(sv[ch * 8 + 4], sv[ch * 8 + 5]);
        wp.w = pack_bf16(sv[ch * 8 + 6], sv[ch * 8 + 7]);
        wd.x = pack_bf16(dv[ch * 8 + 0], dv[ch * 8 + 1]);
        wd.y = pack_bf16(dv[ch * 8 + 2], dv[ch * 8 + 3]);
        wd.z = pack_bf16(dv[ch * 8 + 4], dv[ch * 8 + 5]);
        wd.w = pack_bf16(dv[ch * 8 + 6], dv[ch * 8 + 7]);
        const int sw = (c16 ^ (r & 7)) << 4;
        *reinterpret_cast<uint4*>(prow + sw) = wp;
        *reinterpret_cast<uint4*>(prow + ATOM + sw) = wd;
      }
      fence_proxy_async_smem();
      fence_before();
      mbar_arrive(smem_u32(&pd_full[st]));
    }
    if (ok && n_it > 0 && warp_wait(smem_u32(fin), 0, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
      fence_after();
      __nv_bfloat16* drow = dqkv + (static_cast<int64_t>(row0) + kv_row) * ld;
      {
        const int which = g;  // group 0 writes dK (scaled), group 1 dV
        const uint32_t col = which == 0 ? KV_COL_DK : KV_COL_DV;
        const float f = which == 0 ? scale : 1.f;
        __nv_bfloat16* out = drow + (which == 0 ? col_k : col_v);
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t u[32];
          tmem_ld32(tmem + lane_base + col + ch * 32, u);
          if (kv_row < T) {
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(u[qd * 8 + 0]) * f, __uint_as_float(u[qd * 8 + 1]) * f);
              w.y = pack_bf16(__uint_as_float(u[qd * 8 + 2]) * f, __uint_as_float(u[qd * 8 + 3]) * f);
              w.z = pack_bf16(__uint_as_float(u[qd * 8 + 4]) * f, __uint_as_float(u[qd * 8 + 5]) * f);
              w.w = pack_bf16(__uint_as_float(u[qd * 8 + 6]) * f, __uint_as_float(u[qd * 8 + 7]) * f);
              *reinterpret_cast<uint4*>(out + ch * 32 + qd * 8) = w;
            }
          }
        }
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

// ------------------------------------------------------------ dQ
// smem: Q | dO | K0 V0 | K1 V1 | DS0 | DS1
constexpr int DQ_OFF_Q = 0, DQ_OFF_O = TILE, DQ_OFF_KV = 2 * TILE, DQ_OFF_DS = 2 * TILE + 4 * HALF_TILE;
constexpr int DQ_SMEM_TILES = DQ_OFF_DS + 2 * ATOM;
constexpr int DQ_SMEM_BYTES = DQ_SMEM_TILES + 256 + 1024;
constexpr uint32_t DQ_COL_S = 0, DQ_COL_DP = 128, DQ_COL_DQ = 256;

__global__ void __launch_bounds__(BWD_THREADS, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q128, const __grid_constant__ CUtensorMap tm_do128,
                          const __grid_constant__ CUtensorMap tm_kv64, const float* __restrict__ lse,
                          const float* __restrict__ delta, __nv_bfloat16* __restrict__ dqkv, int64_t ld, int T, int nq,
                          int nkv, float scale_log2, float scale, int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DQ_SMEM_TILES);
  uint64_t* q_full = bars;        // 1
  uint64_t* kv_full = bars + 1;   // 2
  uint64_t* kv_empty = bars + 3;  // 2
  uint64_t* sp_full = bars + 5;   // 2
  uint64_t* ds_full = bars + 7;   // 2
  uint64_t* mma_done = bars + 9;  // 2
  uint64_t* fin = bars + 11;      // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int qb = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int c = (h * nkv) / nq;
  const int q0 = qb * 128;
  const int n_j = min((T + 63) / 64, (q0 + 128) / 64);
  const int row0 = b * T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col_k = (nq + c) * D, col_v = (nq + nkv + c) * D;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    mbar_init(smem_u32(fin), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&kv_full[i]), 1);
      mbar_init(smem_u32(&kv_empty[i]), 1);
      mbar_init(smem_u32(&sp_full[i]), 1);
      mbar_init(smem_u32(&ds_full[i]), 256);
      mbar_init(smem_u32(&mma_done[i]), 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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
    if (lane == 0) {
      const uint32_t fb = smem_u32(q_full);
      mbar_expect_tx(fb, 2 * TILE);
      tma_load_2d(smem_u32(smem + DQ_OFF_Q), &tm_q128, fb, h * D, row0 + q0);
      tma_load_2d(smem_u32(smem + DQ_OFF_Q + ATOM), &tm_q128, fb, h * D + 64, row0 + q0);
      tma_load_2d(smem_u32(smem + DQ_OFF_O), &tm_do128, fb, h * D, row0 + q0);
      tma_load_2d(smem_u32(smem + DQ_OFF_O + ATOM), &tm_do128, fb, h * D + 64, row0 + q0);
    }
    __syncwarp();
    for (int j = 0; j < n_j; ++j) {
      const int st = j & 1;
      if (!warp_wait(smem_u32(&kv_empty[st]), ((j >> 1) & 1) ^ 1, abort_flag, err, DEV_ERR_TIMEOUT_PRODUCER)) break;
      if (lane == 0) {
        const uint32_t fb = smem_u32(&kv_full[st]);
        uint8_t* kt = smem + DQ_OFF_KV + st * 2 * HALF_TILE;
        uint8_t* vt = kt + HALF_TILE;
        const int r = row0 + j * 64;
        mbar_expect_tx(fb, 2 * HALF_TILE);
        tma_load_2d(smem_u32(kt), &tm_kv64, fb, col_k, r);
        tma_load_2d(smem_u32(kt + HALF_ATOM), &tm_kv64, fb, col_k + 64, r);
        tma_load_2d(smem_u32(vt), &tm_kv64, fb, col_v, r);
        tma_load_2d(smem_u32(vt + HALF_ATOM), &tm_kv64, fb, col_v + 64, r);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    constexpr uint32_t idesc_sp = idesc_bf16(128, 64, false, false);  // S = Q K^T, dP = dO V^T
    constexpr uint32_t idesc_dq = idesc_bf16(128, D, false, true);    // dQ += dS K (K is MN-major)
    const uint32_t q_base = smem_u32(smem + DQ_OFF_Q), o_base = smem_u32(smem + DQ_OFF_O);
    bool ok = warp_wait(smem_u32(q_full), 0, abort_flag, err, DEV_ERR_TIMEOUT_MMA);
    auto issue_sp = [&](int j) -> bool {
      const int st = j & 1;
      if (!warp_wait(smem_u32(&kv_full[st]), (j >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) return false;
      fence_after();
      if (lane == 0) {
        const uint32_t k_base = smem_u32(smem + DQ_OFF_KV + st * 2 * HALF_TILE);
        const uint32_t v_base = k_base + HALF_TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off_a = static_cast<uint32_t>((kk >> 2) * ATOM + (kk & 3) * 32);
          const uint32_t off_b = static_cast<uint32_t>((kk >> 2) * HALF_ATOM + (kk & 3) * 32);
          umma_bf16(tmem + DQ_COL_S + st * 64, smem_desc(q_base + off_a, 16, 1024),
                    smem_desc(k_base + off_b, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
          umma_bf16(tmem + DQ_COL_DP + st * 64, smem_desc(o_base + off_a, 16, 1024),
                    smem_desc(v_base + off_b, 16, 1024), idesc_sp, kk > 0 ? 1u : 0u);
        }
        umma_commit(smem_u32(&sp_full[st]));
      }
      __syncwarp();
      return true;
    };
    if (ok) ok = issue_sp(0);
    for (int j = 0; j < n_j && ok; ++j) {
      const int st = j & 1;
      if (j + 1 < n_j && !issue_sp(j + 1)) {
        ok = false;
        break;
      }
      if (!warp_wait(smem_u32(&ds_full[st]), (j >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) {
        ok = false;
        break;
      }
      fence_after();
      if (lane == 0) {
        const uint32_t ds = smem_u32(smem + DQ_OFF_DS + st * ATOM);
        const uint32_t k_base = smem_u32(smem + DQ_OFF_KV + st * 2 * HALF_TILE);
#pragma unroll
        for (int kk = 0; kk < 64 / 16; ++kk)
          umma_bf16(tmem + DQ_COL_DQ, smem_desc(ds + kk * 32, 16, 1024), smem_desc(k_base + kk * 2048, HALF_ATOM, 1024),
                    idesc_dq, (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(smem_u32(&kv_empty[st]));
        umma_commit(smem_u32(&mma_done[st]));
      }
      __syncwarp();
    }
    if (lane == 0) umma_commit(smem_u32(fin));
    __syncwarp();
  } else {
    const int g = (warp - 2) >> 2;  // key columns [32 g, 32 g + 32) of each 64-column block
    const int qw = warp & 3;
    const int r = qw * 32 + lane;
    const int q_row = q0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(qw * 32) << 16;
    const int64_t sb = (static_cast<int64_t>(b) * nq + h) * T;
    const float lse2 = q_row < T ? lse[sb + q_row] * LOG2E : 0.f;
    const float dl = q_row < T ? delta[sb + q_row] : 0.f;
    bool ok = true;
    for (int j = 0; j < n_j; ++j) {
      const int st = j & 1;
      if (!warp_wait(smem_u32(&sp_full[st]), (j >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
        ok = false;
        break;
      }
      fence_after();
      float sv[32], dv[32];
      {
        uint32_t u[32];
        tmem_ld32(tmem + lane_base + DQ_COL_S + st * 64 + g * 32, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[e] = __uint_as_float(u[e]);
        tmem_ld32(tmem + lane_base + DQ_COL_DP + st * 64 + g * 32, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) dv[e] = __uint_as_float(u[e]);
      }
      const int k0 = j * 64 + g * 32;
      const bool diag = k0 + 31 > q0;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        float p = exp2f(sv[e] * scale_log2 - lse2);
        if (diag && k0 + e > q_row) p = 0.f;
        dv[e] = p * (dv[e] - dl);
      }
      if (j >= 2) {
        if (!warp_wait(smem_u32(&mma_done[st]), ((j - 2) >> 1) & 1, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
          ok = false;
          break;
        }
      }
      uint8_t* drow = smem + DQ_OFF_DS + st * ATOM + r * 128;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const int c16 = g * 4 + ch;
        uint4 w;
        w.x = pack_bf16(dv[ch * 8 + 0], dv[ch * 8 + 1]);
        w.y = pack_bf16(dv[ch * 8 + 2], dv[ch * 8 + 3]);
        w.z = pack_bf16(dv[ch * 8 + 4], dv[ch * 8 + 5]);
        w.w = pack_bf16(dv[ch * 8 + 6], dv[ch * 8 + 7]);
        *reinterpret_cast<uint4*>(drow + ((c16 ^ (r & 7)) << 4)) = w;
      }
      fence_proxy_async_smem();
      fence_before();
      mbar_arrive(smem_u32(&ds_full[st]));
    }
    if (ok && warp_wait(smem_u32(fin), 0, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
      fence_after();
      __nv_bfloat16* out = dqkv + (static_cast<int64_t>(row0) + q_row) * ld + static_cast<int64_t>(h) * D + g * 64;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {  // group g writes dQ columns [64 g, 64 g + 64)
        uint32_t u[32];
        tmem_ld32(tmem + lane_base + DQ_COL_DQ + g * 64 + ch * 32, u);
        if (q_row < T) {
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(u[qd * 8 + 0]) * scale, __uint_as_float(u[qd * 8 + 1]) * scale);
            w.y = pack_bf16(__uint_as_float(u[qd * 8 + 2]) * scale, __uint_as_float(u[qd * 8 + 3]) * scale);
            w.z = pack_bf16(__uint_as_float(u[qd * 8 + 4]) * scale, __uint_as_float(u[qd * 8 + 5]) * scale);
            w.w = pack_bf16(__uint_as_float(u[qd * 8 + 6]) * scale, __uint_as_float(u[qd * 8 + 7]) * scale);
            *reinterpret_cast<uint4*>(out + ch * 32 + qd * 8) = w;
          }
        }
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

// dQ, dK, dV on the tensor cores (head_dim 128); delta = rowsum(dO * O) must be in `delta`.
mt_status attn_bwd_tc_launch(const mt_bf16* qkv, int64_t ld, const mt_bf16* d_o, int64_t ld_o, const float* lse,
                             const float* delta, mt_bf16* dqkv, int B, int T, int nq, int nkv, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(attn_bwd_dkv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, KV_SMEM_BYTES);
    if (attr == cudaSuccess)
      attr = cudaFuncSetAttribute(attn_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_SMEM_BYTES);
  });
  if (attr != cudaSuccess) return fail(MT_ERR_CUDA, "attention smem attribute: %s", cudaGetErrorString(attr));
  const uint64_t rows = static_cast<uint64_t>(B) * T;
  const uint64_t qkv_cols = static_cast<uint64_t>((nq + 2 * nkv) * D), o_cols = static_cast<uint64_t>(nq * D);
  CUtensorMap qkv128, qkv64, do128, do64;
  MT_TRY(tma_map_2d(&qkv128, qkv, qkv_cols, rows, static_cast<uint64_t>(ld), 64, 128));
  MT_TRY(tma_map_2d(&qkv64, qkv, qkv_cols, rows, static_cast<uint64_t>(ld), 64, 64));
  MT_TRY(tma_map_2d(&do128, d_o, o_cols, rows, static_cast<uint64_t>(ld_o), 64, 128));
  MT_TRY(tma_map_2d(&do64, d_o, o_cols, rows, static_cast<uint64_t>(ld_o), 64, 64));
  int32_t* err = device_error_word();
  if (!err) return fail(MT_ERR_CUDA, "device error word unavailable");
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  const float scale_log2 = LOG2E * scale;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(dqkv);
  dim3 gq((T + 127) / 128, nq, B);
  attn_bwd_dq_tc_kernel<<<gq, BWD_THREADS, DQ_SMEM_BYTES, st>>>(qkv128, do128, qkv64, lse, delta, out, ld, T, nq, nkv,
                                                                scale_log2, scale, err);
  MT_TRY(launch_check("attn_bwd_dq_tc_kernel"));
  dim3 gk((T + 127) / 128, nkv, B);
  attn_bwd_dkv_tc_kernel<<<gk, BWD_THREADS, KV_SMEM_BYTES, st>>>(qkv128, qkv64, do64, lse, delta, out, ld, T, nq, nkv,
                                                                 scale_log2, scale, err);
  MT_TRY(launch_check("attn_bwd_dkv_tc_kernel"));
  // dq: QK^T, dO V^T, dS K; dkv: QK^T, dO V^T, P^T dO, dS^T Q (causal half)
  add_exec_flops(14.0 * B * nq * D * (0.5 * double(T) * double(T)));
  return MT_OK;
}

}  // namespace mt
