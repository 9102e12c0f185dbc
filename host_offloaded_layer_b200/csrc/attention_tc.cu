// Causal grouped-query flash attention forward on the sm_100a tensor cores
// (head_dim 128): S = Q K^T and O += P V are tcgen05.mma with both
// accumulators in tensor memory, the operands staged by TMA.
//
// Persistent: one CTA per SM walks the (128 query rows, query head, sequence)
// tiles, longest rows first in a snake order, so the next tile's Q load and
// first two S MMAs overlap the current tile's output epilogue.
//   warp 0     TMA: lane 0 loads Q per tile and K_j, lane 1 V_j (128 key
//              rows each), each into its own three-stage ring: a K stage is
//              free once S_j is done, a V stage once O += P_j V_j is;
//   warp 1     TMEM allocation and the MMA issuer: S_{j+1} = Q K_{j+1}^T is
//              issued before O += P_j V_j so the tensor cores work while the
//              softmax of block j runs;
//   warps 2-9  softmax in two groups of four warps, one thread per query row
//              and group. Group g owns key columns [64 g, 64 g + 64) of every
//              block and its own output accumulator O_g = sum_j P_j,g V_j,g
//              with its own running maximum and sum (a split of the key axis
//              inside the CTA), so the groups never synchronise inside the
//              key loop; the two partial results meet once per tile:
//              O = (O_0 2^(m_0 - m) + O_1 2^(m_1 - m)) / (l_0 2^(m_0 - m) + l_1 2^(m_1 - m)).
// P never touches shared memory: each thread writes its row of P_g (bf16
// pairs) over the first 32 columns of its own half of the S buffer it just
// read, and O_g += P_g V_g takes its A operand from tensor memory. The
// tensor core runs one CTA's MMAs in issue order, so S_{j+2}, issued after
// O += P_j V_j, cannot overwrite P_j before that MMA has read it.
// Scores are handled in the log2 domain. TMEM: two S buffers (128 columns
// each), O_0 and O_1 (128 columns each). O_g is rescaled only when its row
// maximum grows by more than 8 (a factor 256 in the exponent); otherwise the
// stale maximum stays, which keeps P <= 256 and the result exact up to
// rounding (the final combination uses the same maxima as every P). Every
// mbarrier wait is bounded.
#include <mutex>

#include "mt_internal.h"
#include "tcgen05.cuh"

namespace mt {
namespace {

using namespace tc;

constexpr int D = 128, BQ = 128, BKV = 128;
constexpr int TILE = BQ * D * 2;  // 32 KiB: a 128 x 128 bf16 tile (two 64-column swizzle atoms)
constexpr int ATOM = 128 * 64 * 2;  // 16 KiB
// shared memory: Q | K0 V0 | K1 V1 | K2 V2 | row exchange [3][128] floats
constexpr int KV_STAGES = 3;
constexpr int OFF_Q = 0, OFF_KV = TILE, OFF_X = TILE + KV_STAGES * 2 * TILE;
constexpr int SMEM_TILES = OFF_X + 3 * 128 * 4;
constexpr int SMEM_BYTES = SMEM_TILES + 256 + 1024;  // tiles, barriers, alignment
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S0 = 0, COL_O = 256;  // S_s at 128 s, O_g at 256 + 128 g
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;
constexpr int FWD_THREADS = 64 + 256;

// 2^x by the MUFU instruction (flush-to-zero; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One arrival per warp: the warp's lanes are ordered by __syncwarp, then
// lane 0 arrives (release) on behalf of all of them.
__device__ __forceinline__ void warp_arrive(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Bounded barrier among groups of warps on an mbarrier initialised with the
// number of warps: arrive once per warp, then every thread waits for the phase
// to flip. `phase` counts this thread's uses. Returns false when the wait ran out.
__device__ __forceinline__ bool warps_sync(uint32_t bar, uint32_t& phase, volatile int* abort_flag, int32_t* err) {
  warp_arrive(bar);
  const bool ok = mbar_wait(bar, phase & 1u, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE);
  ++phase;
  return ok;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Each thread of the warp writes 16 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// One 256-bit store (16 bf16 values, a whole 32-byte sector); p 32-byte aligned.
__device__ __forceinline__ void st_v8(void* p, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// The k-th tile of this CTA in a persistent walk over tiles sorted longest first: round k hands
// out tiles [k G, k G + G) to the G CTAs in alternating directions (a snake), so the CTA that
// takes the longest tile of one round takes the shortest of the next and the work stays even.
__device__ __forceinline__ int snake_tile(int k) {
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  return k * G + ((k & 1) ? G - 1 - c : c);
}

// D (+)= A B with A (M = 128 rows in the lanes, 16 bf16 of K packed in pairs
// along 8 columns) read from tensor memory and B from shared memory.
__device__ __forceinline__ void umma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Tile t of the persistent walk: query blocks from the last (longest rows)
// down, then query head, then sequence.
struct FwdTile {
  int qb, h, b;
};
__device__ __forceinline__ FwdTile fwd_tile(int t, int n_qb, int nq, int B) {
  const int per_qb = nq * B;
  const int rest = t % per_qb;
  return {n_qb - 1 - t / per_qb, rest % nq, rest / nq};
}

__global__ void __launch_bounds__(FWD_THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, __nv_bfloat16* __restrict__ o, int64_t ld_o,
                       int o_v8, float* __restrict__ lse, int B, int T, int nq, int nkv, float scale_log2,
                       int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_TILES);
  uint64_t* q_full = bars;        // 1: Q of the tile loaded
  uint64_t* q_empty = bars + 1;   // 1: the tile's S MMAs (the readers of Q) are done
  uint64_t* k_full = bars + 2;    // 3
  uint64_t* k_empty = bars + 5;   // 3
  uint64_t* v_full = bars + 8;    // 3
  uint64_t* v_empty = bars + 11;  // 3
  uint64_t* s_full = bars + 14;   // 2
  uint64_t* p_full = bars + 16;   // [group][buffer]: 4, one arrival per warp of the group
  uint64_t* o_done = bars + 20;   // [group][buffer]: 4
  uint64_t* o_free = bars + 24;   // 1: the tile's O accumulators have been read (8 warps)
  uint64_t* x_bar = bars + 25;    // 1: row exchange between the groups (8 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 26);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xch = reinterpret_cast<float*>(smem + OFF_X);  // [3][128]: group 1's (m, l), then group 0's (f0, f1, 1/l)

  const int n_qb = (T + BQ - 1) / BQ;
  const int n_tiles = n_qb * nq * B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    mbar_init(smem_u32(q_empty), 1);
    for (int i = 0; i < KV_STAGES; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1);
      mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 1);
      mbar_init(smem_u32(&v_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&s_full[i]), 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(&p_full[i]), 4);
      mbar_init(smem_u32(&o_done[i]), 1);
    }
    mbar_init(smem_u32(o_free), 8);
    mbar_init(smem_u32(x_bar), 8);
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
    // ------------------------------------------------------------ TMA producer (lane 0: Q, K; lane 1: V)
    if (lane < 2) {
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int t = snake_tile(0), k = 0; t < n_tiles && ok; t = snake_tile(++k), ++tl) {
        const FwdTile w = fwd_tile(t, n_qb, nq, B);
        const int c = (w.h * nkv) / nq;
        const int row0 = w.b * T, q0 = w.qb * BQ;
        const int n_kv = min(n_qb, w.qb + 1);
        if (lane == 0) {
          if (tl > 0 && !mbar_wait(smem_u32(q_empty), (tl - 1) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_PRODUCER)) break;
          const uint32_t qb_bar = smem_u32(q_full);
          const int col_q = w.h * D;
          mbar_expect_tx(qb_bar, TILE);
          tma_load_2d(smem_u32(smem + OFF_Q), &tm_qkv, qb_bar, col_q, row0 + q0);
          tma_load_2d(smem_u32(smem + OFF_Q + ATOM), &tm_qkv, qb_bar, col_q + 64, row0 + q0);
        }
        const int col = lane == 0 ? (nq + c) * D : (nq + nkv + c) * D;  // K or V columns
        uint64_t* full = lane == 0 ? k_full : v_full;
        uint64_t* empty = lane == 0 ? k_empty : v_empty;
        const int off = lane == 0 ? 0 : TILE;
        for (int j = 0; j < n_kv; ++j, ++it) {
          const int s = it % KV_STAGES;
          if (!mbar_wait(smem_u32(&empty[s]), ((it / KV_STAGES) & 1u) ^ 1u, abort_flag, err,
                         DEV_ERR_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[s]);
          uint8_t* dst = smem + OFF_KV + s * 2 * TILE + off;
          const int r = row0 + j * BKV;
          mbar_expect_tx(fb, TILE);
          tma_load_2d(smem_u32(dst), &tm_qkv, fb, col, r);
          tma_load_2d(smem_u32(dst + ATOM), &tm_qkv, fb, col + 64, r);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, BKV, false, false);  // S = Q K^T: both K-major
    constexpr uint32_t idesc_o = idesc_bf16(128, D, false, true);     // O_g += P_g V_g: V is MN-major (d contiguous)
    const uint32_t q_base = smem_u32(smem + OFF_Q);
    auto issue_s = [&](uint32_t i) -> bool {
      const int s = i & 1, sk = i % KV_STAGES;
      if (!warp_wait(smem_u32(&k_full[sk]), (i / KV_STAGES) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) return false;
      fence_after();
      if (lane == 0) {
        const uint32_t k_base = smem_u32(smem + OFF_KV + sk * 2 * TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk >> 2) * ATOM + (kk & 3) * 32);
          umma_bf16(tmem + COL_S0 + s * BKV, smem_desc(q_base + off, 16, 1024), smem_desc(k_base + off, 16, 1024),
                    idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(smem_u32(&s_full[s]));
        umma_commit(smem_u32(&k_empty[sk]));
      }
      __syncwarp();
      return true;
    };
    uint32_t it = 0, tl = 0;
    bool ok = true;
    for (int t = snake_tile(0), k = 0; t < n_tiles && ok; t = snake_tile(++k), ++tl) {
      const FwdTile w = fwd_tile(t, n_qb, nq, B);
      const int n_kv = min(n_qb, w.qb + 1);
      if (!warp_wait(smem_u32(q_full), tl & 1u, abort_flag, err, DEV_ERR_TIMEOUT_MMA) || !issue_s(it)) break;
      for (int j = 0; j < n_kv && ok; ++j) {
        const uint32_t i = it + j;
        const int s = i & 1;
        if (j + 1 < n_kv) {
          if (!issue_s(i + 1)) {
            ok = false;
            break;
          }
        } else {
          if (lane == 0) umma_commit(smem_u32(q_empty));  // every S MMA of the tile is issued
          __syncwarp();
        }
        // the first P V of a tile overwrites O: the previous tile's epilogue must have read it
        if (j == 0 && tl > 0 && !warp_wait(smem_u32(o_free), (tl - 1) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        const int sv = i % KV_STAGES;
        const uint32_t v_base = smem_u32(smem + OFF_KV + sv * 2 * TILE + TILE);
        if (!warp_wait(smem_u32(&v_full[sv]), (i / KV_STAGES) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        for (int g = 0; g < 2; ++g) {
          if (!warp_wait(smem_u32(&p_full[g * 2 + s]), (i >> 1) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          fence_after();
          if (lane == 0) {
            // P_g sits in the first 32 columns of group g's half of S buffer s
            const uint32_t p_tmem = tmem + COL_S0 + s * BKV + g * 64;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              umma_bf16_tmem_a(tmem + COL_O + g * D, p_tmem + kk * 8, smem_desc(v_base + (g * 4 + kk) * 2048, ATOM, 1024),
                               idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(smem_u32(&o_done[g * 2 + s]));
            if (g == 1) umma_commit(smem_u32(&v_empty[sv]));
          }
          __syncwarp();
        }
      }
      it += n_kv;
    }
  } else {
    // ------------------------------------------------------------ softmax (one thread per query row and group)
    const int g = (warp - 2) >> 2;  // key columns [64 g, 64 g + 64) of every block, accumulator O_g
    const int qw = warp & 3;        // TMEM lanes [32 qw, 32 qw + 32)
    const int r = qw * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(qw * 32) << 16;
    const uint32_t col_og = COL_O + g * D;
    uint32_t it = 0, tl = 0, xph = 0;
    bool ok = true;
    for (int t = snake_tile(0), k = 0; t < n_tiles && ok; t = snake_tile(++k), ++tl) {
      const FwdTile w = fwd_tile(t, n_qb, nq, B);
      const int q0 = w.qb * BQ, q_row = q0 + r, row0 = w.b * T;
      const int n_kv = min(n_qb, w.qb + 1);
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < n_kv; ++j) {
        const uint32_t i = it + j;
        const int s = i & 1;
        if (!warp_wait(smem_u32(&s_full[s]), (i >> 1) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
          ok = false;
          break;
        }
        fence_after();
        float sv[64];
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t u[32];
          tmem_ld32(tmem + lane_base + COL_S0 + s * BKV + g * 64 + ch * 32, u);
#pragma unroll
          for (int e = 0; e < 32; ++e) sv[ch * 32 + e] = __uint_as_float(u[e]);
        }
        const int k0 = j * BKV + g * 64;
        if (k0 + 63 > q0) {  // a block on the diagonal: keys after the row are masked
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (k0 + e > q_row) sv[e] = -INFINITY;
        }
        // row maximum over eight independent partial maxima (short dependency chains)
        float m8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = sv[e];
#pragma unroll
        for (int e = 8; e < 64; ++e) m8[e & 7] = fmaxf(m8[e & 7], sv[e]);
        float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        mx *= scale_log2;
        // rescale O_g only when some row of the warp raised its maximum by more than the threshold
        if (__any_sync(0xffffffffu, mx > m_run + RESCALE_THRESHOLD)) {
          const float m_new = fmaxf(m_run, mx);
          const float alpha = m_new == -INFINITY ? 1.f : ex2(m_run - m_new);  // 0 while m_run = -inf
          if (j > 0) {
            // O_g must hold P_{j-1} V_{j-1} before it is rescaled
            const uint32_t ip = i - 1;
            if (!warp_wait(smem_u32(&o_done[g * 2 + (ip & 1)]), (ip >> 1) & 1u, abort_flag, err,
                           DEV_ERR_TIMEOUT_EPILOGUE)) {
              ok = false;
              break;
            }
            fence_after();
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              uint32_t u[32];
              tmem_ld32(tmem + lane_base + col_og + ch * 32, u);
#pragma unroll
              for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
              tmem_st32(tmem + lane_base + col_og + ch * 32, u);
            }
          }
          l_run *= alpha;
          m_run = m_new;
        }
        // P over the S values just read (its MMA reader of two blocks ago finished before S_i was
        // written: the tensor core runs the CTA's MMAs in order and s_full covers all earlier ones)
        const float mb = m_run == -INFINITY ? 0.f : m_run;  // a fully masked row half gives P = 0
        float l8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // eight partial sums, added in a fixed tree
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = ex2(fmaf(sv[2 * e], scale_log2, -mb));
          const float p1 = ex2(fmaf(sv[2 * e + 1], scale_log2, -mb));
          l8[e & 7] += p0 + p1;
          pk[e] = pack_bf16(p0, p1);
        }
        const float lsum = ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
        tmem_st32(tmem + lane_base + COL_S0 + s * BKV + g * 64, pk);
        l_run += lsum;
        fence_before();
        warp_arrive(smem_u32(&p_full[g * 2 + s]));
      }
      if (!ok) break;
      it += n_kv;
      // ---- the two groups' partial results meet: O = (O_0 f_0 + O_1 f_1) / l. Both groups' last
      // P V are done first, so O is final and neither P buffer is read any more.
      const uint32_t il = it - 1;
      if (!warp_wait(smem_u32(&o_done[il & 1]), (il >> 1) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE) ||
          !warp_wait(smem_u32(&o_done[2 + (il & 1)]), (il >> 1) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
        ok = false;
        break;
      }
      fence_after();
      // group 1 hands its (m, l) to group 0, which forms the combination and hands back (f0, f1, 1/l)
      if (g == 1) {
        xch[r] = m_run;
        xch[128 + r] = l_run;
      }
      if (!warps_sync(smem_u32(x_bar), xph, abort_flag, err)) break;
      float f0, f1, inv;
      if (g == 0) {
        const float m1 = xch[r], l1 = xch[128 + r];
        const float m = fmaxf(m_run, m1);
        f0 = ex2(m_run - m);
        f1 = ex2(m1 - m);
        const float l_tot = l_run * f0 + l1 * f1;
        inv = 1.f / l_tot;
        xch[r] = f0;
        xch[128 + r] = f1;
        xch[256 + r] = inv;
        if (q_row < T) lse[(static_cast<int64_t>(w.b) * nq + w.h) * T + q_row] = (m + log2f(l_tot)) * LN2;
      }
      if (!warps_sync(smem_u32(x_bar), xph, abort_flag, err)) break;
      if (g == 1) {
        f0 = xch[r];
        f1 = xch[128 + r];
        inv = xch[256 + r];
      }
      __nv_bfloat16* orow = o + (static_cast<int64_t>(row0) + q_row) * ld_o + static_cast<int64_t>(w.h) * D;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {  // this group writes output columns [64 g, 64 g + 64)
        const int oc = g * 64 + ch * 32;
        uint32_t u0[32], u1[32];
        tmem_ld32(tmem + lane_base + COL_O + oc, u0);
        tmem_ld32(tmem + lane_base + COL_O + D + oc, u1);
        if (q_row < T && o_v8) {
          // whole 32-byte sectors: two 256-bit stores of 16 columns
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int c0 = hh * 16 + 2 * e;
              w[e] = pack_bf16((__uint_as_float(u0[c0]) * f0 + __uint_as_float(u1[c0]) * f1) * inv,
                               (__uint_as_float(u0[c0 + 1]) * f0 + __uint_as_float(u1[c0 + 1]) * f1) * inv);
            }
            asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(orow + oc + hh * 16), "r"(w[0]),
                         "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                         : "memory");
          }
        } else if (q_row < T) {
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              v[e] = (__uint_as_float(u0[qd * 8 + e]) * f0 + __uint_as_float(u1[qd * 8 + e]) * f1) * inv;
            uint4 wv;
            wv.x = pack_bf16(v[0], v[1]);
            wv.y = pack_bf16(v[2], v[3]);
            wv.z = pack_bf16(v[4], v[5]);
            wv.w = pack_bf16(v[6], v[7]);
            *reinterpret_cast<uint4*>(orow + oc + qd * 8) = wv;
          }
        }
      }
      fence_before();
      warp_arrive(smem_u32(o_free));
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
  const int64_t n_tiles = static_cast<int64_t>((T + BQ - 1) / BQ) * nq * B;
  if (n_tiles >= (1ll << 31)) return fail(MT_ERR_INVALID_ARG, "attention: too many tiles");
  const int grid = static_cast<int>(std::min<int64_t>(n_tiles, num_sms()));
  const float scale_log2 = LOG2E / sqrtf(static_cast<float>(D));
  // 256-bit stores of O when every row's 32-column chunk is 32-byte aligned
  const int o_v8 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0 && (ld_o * 2) % 32 == 0;
  attn_fwd_tc_kernel<<<grid, FWD_THREADS, SMEM_BYTES, st>>>(tm, reinterpret_cast<__nv_bfloat16*>(o), ld_o, o_v8, lse,
                                                            B, T, nq, nkv, scale_log2, err);
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
// smem: K | V | Q0 dO0 | .. | Q3 dO3 | lse/delta [4][2][64]
// Four Q / dO stages: the load of block it + 4 starts when the dV / dK MMAs of
// block it are done, which leaves three blocks of work to cover its latency.
// P^T and dS^T never touch shared memory: each thread writes its key row of
// them (bf16 pairs) over the first 16 columns of its group's half of the S^T
// and dP^T buffers it just read, and dV += P^T dO, dK += dS^T Q take their A
// operand from tensor memory (the tensor core runs the CTA's MMAs in issue
// order, so S^T / dP^T of block it + 2 cannot overwrite them before they are read).
constexpr int KV_QO_STAGES = 4;
constexpr int KV_OFF_K = 0, KV_OFF_V = TILE, KV_OFF_QO = 2 * TILE;
constexpr int KV_OFF_LD = KV_OFF_QO + KV_QO_STAGES * 2 * HALF_TILE;
constexpr int KV_SMEM_TILES = KV_OFF_LD + KV_QO_STAGES * 128 * 4;
constexpr int KV_SMEM_BYTES = KV_SMEM_TILES + 256 + 1024;
constexpr uint32_t KV_COL_ST = 0, KV_COL_DPT = 128, KV_COL_DV = 256, KV_COL_DK = 384;
// Both backward kernels run two groups of four compute warps (warps 2-5 and 6-9),
// each on half of a block's 64 columns: no row reduction crosses the halves.
constexpr int BWD_THREADS = 64 + 256;

__global__ void __launch_bounds__(BWD_THREADS, 1)
    attn_bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_kv128, const __grid_constant__ CUtensorMap tm_q64,
                           const __grid_constant__ CUtensorMap tm_do64, const float* __restrict__ lse,
                           const float* __restrict__ delta, __nv_bfloat16* __restrict__ dqkv, int64_t ld, int v8,
                           int T, int nq, int nkv, float scale_log2, float scale, const float2* __restrict__ rope,
                           int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* lsd = reinterpret_cast<float*>(smem + KV_OFF_LD);  // [stage][lse2 | delta][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + KV_SMEM_TILES);
  uint64_t* kv_full = bars;       // 1
  uint64_t* qo_full = bars + 1;   // 4
  uint64_t* qo_empty = bars + 5;  // 4
  uint64_t* l_full = bars + 9;    // 4: lse/delta of a stage written by the producer warp
  uint64_t* sp_full = bars + 13;  // 2
  uint64_t* pd_full = bars + 15;  // 2
  uint64_t* fin = bars + 17;      // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // key blocks vary slowest, so the launch order is small key blocks (the most query blocks) first
  const int kb = blockIdx.z;
  const int c = blockIdx.x, b = blockIdx.y;
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
    for (int i = 0; i < KV_QO_STAGES; ++i) {
      mbar_init(smem_u32(&qo_full[i]), 1);
      mbar_init(smem_u32(&qo_empty[i]), 1);
      mbar_init(smem_u32(&l_full[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sp_full[i]), 1);
      mbar_init(smem_u32(&pd_full[i]), 8);
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
      const int st = it % KV_QO_STAGES;
      const uint32_t par = static_cast<uint32_t>(it / KV_QO_STAGES) & 1u;
      if (!warp_wait(smem_u32(&qo_empty[st]), par ^ 1u, abort_flag, err, DEV_ERR_TIMEOUT_PRODUCER)) break;
      const int h = c * grp + it / per_head;
      const int q0 = (qb0 + it % per_head) * 64;
      if (lane == 0) {
        const uint32_t fb = smem_u32(&qo_full[st]);
        uint8_t* qt = smem + KV_OFF_QO + st * 2 * HALF_TILE;
        uint8_t* ot = qt + HALF_TILE;
        mbar_expect_tx(fb, 2 * HALF_TILE);
        tma_load_2d(smem_u32(qt), &tm_q64, fb, h * D, row0 + q0);
        tma_load_2d(smem_u32(qt + HALF_ATOM), &tm_q64, fb, h * D + 64, row0 + q0);
        tma_load_2d(smem_u32(ot), &tm_do64, fb, h * D, row0 + q0);
        tma_load_2d(smem_u32(ot + HALF_ATOM), &tm_do64, fb, h * D + 64, row0 + q0);
      }
      // this block's log-sum-exp (log2 domain) and delta, shared by all key rows; rows past T give P = 0
      const int64_t sb = (static_cast<int64_t>(b) * nq + h) * T;
      float* l2 = lsd + st * 128;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int q = q0 + hh * 32 + lane;
        l2[hh * 32 + lane] = q < T ? lse[sb + q] * LOG2E : INFINITY;
        l2[64 + hh * 32 + lane] = q < T ? delta[sb + q] : 0.f;
      }
      warp_arrive(smem_u32(&l_full[st]));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_sp = idesc_bf16(128, 64, false, false);  // S^T = K Q^T, dP^T = V dO^T
    constexpr uint32_t idesc_acc = idesc_bf16(128, D, false, true);   // dV += P^T dO, dK += dS^T Q
    const uint32_t k_base = smem_u32(smem + KV_OFF_K), v_base = smem_u32(smem + KV_OFF_V);
    bool ok = n_it == 0 || warp_wait(smem_u32(kv_full), 0, abort_flag, err, DEV_ERR_TIMEOUT_MMA);
    auto issue_sp = [&](int it) -> bool {
      const int st = it & 1, sq = it % KV_QO_STAGES;
      if (!warp_wait(smem_u32(&qo_full[sq]), static_cast<uint32_t>(it / KV_QO_STAGES) & 1u, abort_flag, err,
                     DEV_ERR_TIMEOUT_MMA))
        return false;
      fence_after();
      if (lane == 0) {
        const uint32_t q_base = smem_u32(smem + KV_OFF_QO + sq * 2 * HALF_TILE);
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
        const int sq = it % KV_QO_STAGES;
        const uint32_t q_base = smem_u32(smem + KV_OFF_QO + sq * 2 * HALF_TILE);
        const uint32_t o_base = q_base + HALF_TILE;
#pragma unroll
        for (int kk = 0; kk < 64 / 16; ++kk) {
          // query columns [16 kk, 16 kk + 16): group kk / 2's packed columns, second half at + 8
          const uint32_t a_col = static_cast<uint32_t>(st * 64 + (kk >> 1) * 32 + (kk & 1) * 8);
          umma_bf16_tmem_a(tmem + KV_COL_DV, tmem + KV_COL_ST + a_col, smem_desc(o_base + kk * 2048, HALF_ATOM, 1024),
                           idesc_acc, (it > 0 || kk > 0) ? 1u : 0u);
          umma_bf16_tmem_a(tmem + KV_COL_DK, tmem + KV_COL_DPT + a_col, smem_desc(q_base + kk * 2048, HALF_ATOM, 1024),
                           idesc_acc, (it > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&qo_empty[sq]));
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
    const int kv_row = k0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(qw * 32) << 16;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int st = it & 1, sq = it % KV_QO_STAGES;
      const int q0 = (qb0 + it % per_head) * 64;
      if (!warp_wait(smem_u32(&l_full[sq]), static_cast<uint32_t>(it / KV_QO_STAGES) & 1u, abort_flag, err,
                     DEV_ERR_TIMEOUT_EPILOGUE)) {
        ok = false;
        break;
      }
      __syncwarp();  // lane 0's acquire of the producer's lse / delta stores covers the whole warp
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
      // this group's 32 log-sum-exp and delta values (16-byte aligned: vector broadcast loads)
      const float4* L4 = reinterpret_cast<const float4*>(lsd + sq * 128 + g * 32);
      const float4* D4 = reinterpret_cast<const float4*>(lsd + sq * 128 + 64 + g * 32);
      const int qc0 = q0 + g * 32;
      const bool diag = qc0 < k0 + 127;
#pragma unroll
      for (int v4 = 0; v4 < 8; ++v4) {
        const float4 l4 = L4[v4], d4 = D4[v4];
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dl[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int e = v4 * 4 + c;
          float p = ex2(fmaf(sv[e], scale_log2, -lv[c]));
          if (diag && kv_row > qc0 + e) p = 0.f;
          sv[e] = p;
          dv[e] = p * (dv[e] - dl[c]);
        }
      }
      {  // P^T and dS^T over the S^T / dP^T values just read
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          pp[e] = pack_bf16(sv[2 * e], sv[2 * e + 1]);
          pd[e] = pack_bf16(dv[2 * e], dv[2 * e + 1]);
        }
        tmem_st16(tmem + lane_base + KV_COL_ST + st * 64 + g * 32, pp);
        tmem_st16(tmem + lane_base + KV_COL_DPT + st * 64 + g * 32, pd);
      }
      fence_before();
      warp_arrive(smem_u32(&pd_full[st]));
    }
    if (ok && n_it > 0 && warp_wait(smem_u32(fin), 0, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
      fence_after();
      __nv_bfloat16* drow = dqkv + (static_cast<int64_t>(row0) + kv_row) * ld;
      if (g == 0 && rope) {
        // dK with the inverse rotation of its position: (a, b) -> (a cos + b sin, b cos - a sin)
        // for the pair (i, i + 64), columns 32 cp + e and 32 cp + e + 64
        __nv_bfloat16* out = drow + col_k;
#pragma unroll
        for (int cp = 0; cp < 2; ++cp) {
          uint32_t ua[32], ub[32];
          tmem_ld32(tmem + lane_base + KV_COL_DK + cp * 32, ua);
          tmem_ld32(tmem + lane_base + KV_COL_DK + (cp + 2) * 32, ub);
          if (kv_row < T) {
            const float4* tab = reinterpret_cast<const float4*>(rope + static_cast<int64_t>(kv_row) * (D / 2) + cp * 32);
            uint32_t pa[16], pb[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float4 cs = __ldg(tab + q);
              const float a0 = __uint_as_float(ua[2 * q]) * scale, b0 = __uint_as_float(ub[2 * q]) * scale;
              const float a1 = __uint_as_float(ua[2 * q + 1]) * scale, b1 = __uint_as_float(ub[2 * q + 1]) * scale;
              pa[q] = pack_bf16(a0 * cs.x + b0 * cs.y, a1 * cs.z + b1 * cs.w);
              pb[q] = pack_bf16(b0 * cs.x - a0 * cs.y, b1 * cs.z - a1 * cs.w);
            }
            if (v8) {
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                st_v8(out + cp * 32 + hh * 16, pa + 8 * hh);
                st_v8(out + (cp + 2) * 32 + hh * 16, pb + 8 * hh);
              }
            } else {
#pragma unroll
              for (int qd = 0; qd < 4; ++qd) {
                *reinterpret_cast<uint4*>(out + cp * 32 + qd * 8) =
                    make_uint4(pa[4 * qd], pa[4 * qd + 1], pa[4 * qd + 2], pa[4 * qd + 3]);
                *reinterpret_cast<uint4*>(out + (cp + 2) * 32 + qd * 8) =
                    make_uint4(pb[4 * qd], pb[4 * qd + 1], pb[4 * qd + 2], pb[4 * qd + 3]);
              }
            }
          }
        }
      } else {
        const int which = g;  // group 0 writes dK (scaled), group 1 dV
        const uint32_t col = which == 0 ? KV_COL_DK : KV_COL_DV;
        const float f = which == 0 ? scale : 1.f;
        __nv_bfloat16* out = drow + (which == 0 ? col_k : col_v);
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t u[32];
          tmem_ld32(tmem + lane_base + col + ch * 32, u);
          if (kv_row < T && v8) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = pack_bf16(__uint_as_float(u[2 * e]) * f, __uint_as_float(u[2 * e + 1]) * f);
            st_v8(out + ch * 32, w);
            st_v8(out + ch * 32 + 16, w + 8);
          } else if (kv_row < T) {
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
// smem: Q | dO | K0 V0 | .. | K4 V4
// Five K / V stages: the load of block j + 5 starts when the dQ MMAs of block j
// are done, which leaves four blocks of work to cover its latency. dS never
// touches shared memory: each thread writes its row of it (bf16 pairs) over
// the first 16 columns of its group's half of the S buffer it just read, and
// dQ += dS K takes its A operand from tensor memory.
constexpr int DQ_KV_STAGES = 5;
constexpr int DQ_OFF_Q = 0, DQ_OFF_O = TILE, DQ_OFF_KV = 2 * TILE;
constexpr int DQ_SMEM_TILES = DQ_OFF_KV + DQ_KV_STAGES * 2 * HALF_TILE;
constexpr int DQ_SMEM_BYTES = DQ_SMEM_TILES + 256 + 1024;
constexpr uint32_t DQ_COL_S = 0, DQ_COL_DP = 128, DQ_COL_DQ = 256;

__global__ void __launch_bounds__(BWD_THREADS, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q128, const __grid_constant__ CUtensorMap tm_do128,
                          const __grid_constant__ CUtensorMap tm_kv64, const float* __restrict__ lse,
                          const float* __restrict__ delta, __nv_bfloat16* __restrict__ dqkv, int64_t ld, int v8, int B,
                          int T, int nq, int nkv, float scale_log2, float scale, const float2* __restrict__ rope,
                          int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DQ_SMEM_TILES);
  uint64_t* q_full = bars;         // 1: Q and dO of the tile loaded
  uint64_t* q_empty = bars + 1;    // 1: the tile's S / dP MMAs (the readers of Q and dO) are done
  uint64_t* kv_full = bars + 2;    // 5
  uint64_t* kv_empty = bars + 7;   // 5
  uint64_t* sp_full = bars + 12;   // 2
  uint64_t* ds_full = bars + 14;   // 2
  uint64_t* dq_full = bars + 16;   // 1: the tile's dQ MMAs are done
  uint64_t* dq_free = bars + 17;   // 1: the tile's dQ has been read out (8 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // persistent: tile t is (128 query rows, head, sequence), query blocks from the last (the most
  // key blocks) down, so the next tile's Q / dO load and first S / dP MMAs overlap this tile's end
  const int n_qb = (T + 127) / 128;
  const int n_tiles = n_qb * nq * B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  struct Tile {
    int qb, h, b, c, q0, n_j, row0;
  };
  auto tile = [&](int t) {
    const int per = nq * B, rest = t % per;
    Tile w;
    w.qb = n_qb - 1 - t / per;
    w.h = rest % nq;
    w.b = rest / nq;
    w.c = (w.h * nkv) / nq;
    w.q0 = w.qb * 128;
    w.n_j = min((T + 63) / 64, (w.q0 + 128) / 64);
    w.row0 = w.b * T;
    return w;
  };

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    mbar_init(smem_u32(q_empty), 1);
    mbar_init(smem_u32(dq_full), 1);
    mbar_init(smem_u32(dq_free), 8);
    for (int i = 0; i < DQ_KV_STAGES; ++i) {
      mbar_init(smem_u32(&kv_full[i]), 1);
      mbar_init(smem_u32(&kv_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sp_full[i]), 1);
      mbar_init(smem_u32(&ds_full[i]), 8);
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
    // ------------------------------------------------------------ TMA producer
    uint32_t jg = 0, tl = 0;
    bool ok = true;
    for (int t = snake_tile(0), k = 0; t < n_tiles && ok; t = snake_tile(++k), ++tl) {
      const Tile w = tile(t);
      const int col_k = (nq + w.c) * D, col_v = (nq + nkv + w.c) * D;
      if (tl > 0 && !warp_wait(smem_u32(q_empty), (tl - 1) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_PRODUCER)) break;
      if (lane == 0) {
        const uint32_t fb = smem_u32(q_full);
        mbar_expect_tx(fb, 2 * TILE);
        tma_load_2d(smem_u32(smem + DQ_OFF_Q), &tm_q128, fb, w.h * D, w.row0 + w.q0);
        tma_load_2d(smem_u32(smem + DQ_OFF_Q + ATOM), &tm_q128, fb, w.h * D + 64, w.row0 + w.q0);
        tma_load_2d(smem_u32(smem + DQ_OFF_O), &tm_do128, fb, w.h * D, w.row0 + w.q0);
        tma_load_2d(smem_u32(smem + DQ_OFF_O + ATOM), &tm_do128, fb, w.h * D + 64, w.row0 + w.q0);
      }
      __syncwarp();
      for (int j = 0; j < w.n_j; ++j, ++jg) {
        const int st = jg % DQ_KV_STAGES;
        const uint32_t par = (jg / DQ_KV_STAGES) & 1u;
        if (!warp_wait(smem_u32(&kv_empty[st]), par ^ 1u, abort_flag, err, DEV_ERR_TIMEOUT_PRODUCER)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const uint32_t fb = smem_u32(&kv_full[st]);
          uint8_t* kt = smem + DQ_OFF_KV + st * 2 * HALF_TILE;
          uint8_t* vt = kt + HALF_TILE;
          const int r = w.row0 + j * 64;
          mbar_expect_tx(fb, 2 * HALF_TILE);
          tma_load_2d(smem_u32(kt), &tm_kv64, fb, col_k, r);
          tma_load_2d(smem_u32(kt + HALF_ATOM), &tm_kv64, fb, col_k + 64, r);
          tma_load_2d(smem_u32(vt), &tm_kv64, fb, col_v, r);
          tma_load_2d(smem_u32(vt + HALF_ATOM), &tm_kv64, fb, col_v + 64, r);
        }
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_sp = idesc_bf16(128, 64, false, false);  // S = Q K^T, dP = dO V^T
    constexpr uint32_t idesc_dq = idesc_bf16(128, D, false, true);    // dQ += dS K (K is MN-major)
    const uint32_t q_base = smem_u32(smem + DQ_OFF_Q), o_base = smem_u32(smem + DQ_OFF_O);
    auto issue_sp = [&](uint32_t i) -> bool {
      const int st = i & 1, sk = i % DQ_KV_STAGES;
      if (!warp_wait(smem_u32(&kv_full[sk]), (i / DQ_KV_STAGES) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_MMA))
        return false;
      fence_after();
      if (lane == 0) {
        const uint32_t k_base = smem_u32(smem + DQ_OFF_KV + sk * 2 * HALF_TILE);
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
    uint32_t jg = 0, tl = 0;
    bool ok = true;
    for (int t = snake_tile(0), k = 0; t < n_tiles && ok; t = snake_tile(++k), ++tl) {
      const Tile w = tile(t);
      if (!warp_wait(smem_u32(q_full), tl & 1u, abort_flag, err, DEV_ERR_TIMEOUT_MMA) || !issue_sp(jg)) break;
      for (int j = 0; j < w.n_j && ok; ++j) {
        const uint32_t i = jg + j;
        const int st = i & 1;
        if (j + 1 < w.n_j) {
          if (!issue_sp(i + 1)) {
            ok = false;
            break;
          }
        } else {
          if (lane == 0) umma_commit(smem_u32(q_empty));  // every S / dP MMA of the tile is issued
          __syncwarp();
        }
        if (!warp_wait(smem_u32(&ds_full[st]), (i >> 1) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        // the first dQ MMA of a tile overwrites dQ: the previous tile's must have been read out
        if (j == 0 && tl > 0 && !warp_wait(smem_u32(dq_free), (tl - 1) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        fence_after();
        if (lane == 0) {
          const int sk = i % DQ_KV_STAGES;
          const uint32_t k_base = smem_u32(smem + DQ_OFF_KV + sk * 2 * HALF_TILE);
#pragma unroll
          for (int kk = 0; kk < 64 / 16; ++kk) {
            // key columns [16 kk, 16 kk + 16): group kk / 2's packed columns, second half at + 8
            const uint32_t a_col = static_cast<uint32_t>(st * 64 + (kk >> 1) * 32 + (kk & 1) * 8);
            umma_bf16_tmem_a(tmem + DQ_COL_DQ, tmem + DQ_COL_S + a_col,
                             smem_desc(k_base + kk * 2048, HALF_ATOM, 1024), idesc_dq, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(&kv_empty[sk]));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) umma_commit(smem_u32(dq_full));
      __syncwarp();
      jg += w.n_j;
    }
  } else {
    // ------------------------------------------------------------ dS, one thread per query row and group
    const int g = (warp - 2) >> 2;  // key columns [32 g, 32 g + 32) of each 64-column block
    const int qw = warp & 3;
    const int r = qw * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(qw * 32) << 16;
    uint32_t jg = 0, tl = 0;
    bool ok = true;
    for (int t = snake_tile(0), k = 0; t < n_tiles && ok; t = snake_tile(++k), ++tl) {
      const Tile w = tile(t);
      const int q_row = w.q0 + r;
      const int64_t sb = (static_cast<int64_t>(w.b) * nq + w.h) * T;
      const float lse2 = q_row < T ? lse[sb + q_row] * LOG2E : 0.f;
      const float dl = q_row < T ? delta[sb + q_row] : 0.f;
      for (int j = 0; j < w.n_j; ++j) {
        const uint32_t i = jg + j;
        const int st = i & 1;
        if (!warp_wait(smem_u32(&sp_full[st]), (i >> 1) & 1u, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) {
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
        const bool diag = k0 + 31 > w.q0;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float p = ex2(fmaf(sv[e], scale_log2, -lse2));
          if (diag && k0 + e > q_row) p = 0.f;
          dv[e] = p * (dv[e] - dl);
        }
        {  // dS over the S values just read
          uint32_t pd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pd[e] = pack_bf16(dv[2 * e], dv[2 * e + 1]);
          tmem_st16(tmem + lane_base + DQ_COL_S + st * 64 + g * 32, pd);
        }
        fence_before();
        warp_arrive(smem_u32(&ds_full[st]));
      }
      if (!ok) break;
      jg += w.n_j;
      if (!warp_wait(smem_u32(dq_full), tl & 1u, abort_flag, err, DEV_ERR_TIMEOUT_EPILOGUE)) break;
      fence_after();
      __nv_bfloat16* out = dqkv + (static_cast<int64_t>(w.row0) + q_row) * ld + static_cast<int64_t>(w.h) * D + g * 64;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {  // group g writes dQ columns [64 g, 64 g + 64)
        uint32_t u[32];
        tmem_ld32(tmem + lane_base + DQ_COL_DQ + g * 64 + ch * 32, u);
        if (rope) {
          // the inverse rotation of the row's position pairs column i with i + 64, which the
          // other group writes: read those partners too. Lower half (g = 0): a cos + b sin;
          // upper half (g = 1): b cos - a sin, with a the lower and b the upper value.
          uint32_t w[32];
          tmem_ld32(tmem + lane_base + DQ_COL_DQ + (1 - g) * 64 + ch * 32, w);
          if (q_row < T) {
            const float4* tab = reinterpret_cast<const float4*>(rope + static_cast<int64_t>(q_row) * (D / 2) + ch * 32);
            const float sg = g == 0 ? 1.f : -1.f;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float4 cs = __ldg(tab + q);
              const float v0 = __uint_as_float(u[2 * q]), p0 = __uint_as_float(w[2 * q]);
              const float v1 = __uint_as_float(u[2 * q + 1]), p1 = __uint_as_float(w[2 * q + 1]);
              u[2 * q] = __float_as_uint(v0 * cs.x + sg * p0 * cs.y);
              u[2 * q + 1] = __float_as_uint(v1 * cs.z + sg * p1 * cs.w);
            }
          }
        }
        if (q_row < T && v8) {
          uint32_t wv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            wv[e] = pack_bf16(__uint_as_float(u[2 * e]) * scale, __uint_as_float(u[2 * e + 1]) * scale);
          st_v8(out + ch * 32, wv);
          st_v8(out + ch * 32 + 16, wv + 8);
        } else if (q_row < T) {
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            uint4 wv;
            wv.x = pack_bf16(__uint_as_float(u[qd * 8 + 0]) * scale, __uint_as_float(u[qd * 8 + 1]) * scale);
            wv.y = pack_bf16(__uint_as_float(u[qd * 8 + 2]) * scale, __uint_as_float(u[qd * 8 + 3]) * scale);
            wv.z = pack_bf16(__uint_as_float(u[qd * 8 + 4]) * scale, __uint_as_float(u[qd * 8 + 5]) * scale);
            wv.w = pack_bf16(__uint_as_float(u[qd * 8 + 6]) * scale, __uint_as_float(u[qd * 8 + 7]) * scale);
            *reinterpret_cast<uint4*>(out + ch * 32 + qd * 8) = wv;
          }
        }
      }
      fence_before();
      warp_arrive(smem_u32(dq_free));
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
// With rope_tab (the (cos, sin) table of rope_table_launch) dq and dk come out with the
// inverse rotation of their positions applied, i.e. as gradients of the unrotated q, k.
mt_status attn_bwd_tc_launch(const mt_bf16* qkv, int64_t ld, const mt_bf16* d_o, int64_t ld_o, const float* lse,
                             const float* delta, mt_bf16* dqkv, int B, int T, int nq, int nkv, const float* rope_tab,
                             cudaStream_t st) {
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
  if (B > 65535 || (T + 127) / 128 > 65535 || nq > 65535)
    return fail(MT_ERR_INVALID_ARG, "attention backward: B and T / 128 must be at most 65535");
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  const float scale_log2 = LOG2E * scale;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(dqkv);
  const int64_t dq_tiles = static_cast<int64_t>((T + 127) / 128) * nq * B;
  const int gq = static_cast<int>(std::min<int64_t>(dq_tiles, num_sms()));
  const float2* rope = reinterpret_cast<const float2*>(rope_tab);
  // 256-bit stores of dq, dk, dv when every row's 32-column chunk is 32-byte aligned
  const int v8 = (reinterpret_cast<uintptr_t>(dqkv) & 31u) == 0 && (ld * 2) % 32 == 0;
  attn_bwd_dq_tc_kernel<<<gq, BWD_THREADS, DQ_SMEM_BYTES, st>>>(qkv128, do128, qkv64, lse, delta, out, ld, v8, B, T, nq,
                                                                nkv, scale_log2, scale, rope, err);
  MT_TRY(launch_check("attn_bwd_dq_tc_kernel"));
  dim3 gk(nkv, B, (T + 127) / 128);
  attn_bwd_dkv_tc_kernel<<<gk, BWD_THREADS, KV_SMEM_BYTES, st>>>(qkv128, qkv64, do64, lse, delta, out, ld, v8, T, nq,
                                                                 nkv, scale_log2, scale, rope, err);
  MT_TRY(launch_check("attn_bwd_dkv_tc_kernel"));
  // dq: QK^T, dO V^T, dS K; dkv: QK^T, dO V^T, P^T dO, dS^T Q (causal half)
  add_exec_flops(14.0 * B * nq * D * (0.5 * double(T) * double(T)));
  return MT_OK;
}

}  // namespace mt
