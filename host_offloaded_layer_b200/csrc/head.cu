// Final RMSNorm, LM head and mean token cross-entropy, forward and backward,
// over vocabulary chunks (the [tokens, V] logits never exist at once), and the
// embedding gather / deterministic scatter-add.
//
// The MegaTrain pages count the embedding and LM head in the parameters
// (Table 5) without writing them out; the plainest Qwen2.5 reading is an
// untied embedding E [V, H], a final RMSNorm (gain gf), an LM head W [V, H]
// and the mean cross-entropy against next-token targets. Per vocabulary
// chunk the logits z = h W_c^T come from the tcgen05 GEMM in fp32; pass 1
// keeps a running row maximum / sum of exponentials (the log-sum-exp) and the
// target logit; pass 2 recomputes z, forms dz = (softmax - onehot) / n in bf16
// and runs dW_c = dz^T h and dh += dz W_c on the GEMM (fp32 accumulation in a
// fixed chunk order, so the result is bitwise repeatable).
#include <vector>

#include "mt_internal.h"

namespace mt {

mt_status rmsnorm_fwd_launch(const mt_bf16*, const mt_bf16*, mt_bf16*, float*, int64_t, int, float, cudaStream_t);
mt_status rmsnorm_bwd_launch(const mt_bf16*, const mt_bf16*, const mt_bf16*, const float*, const mt_bf16*, mt_bf16*,
                             float*, int64_t, int, void*, cudaStream_t);
uint64_t colsum_ws_bytes(int64_t rows, int64_t cols);

namespace {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Pass 1 for one chunk: one warp per row folds the chunk's maximum and sum of
// exponentials into the running (m, l) and picks up the target logit.
__global__ void lse_update_kernel(const float* __restrict__ z, int64_t M, int vc, int c0, const int32_t* __restrict__ tgt,
                                  float* __restrict__ m_run, float* __restrict__ l_run, float* __restrict__ zt) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float* zr = z + row * vc;
  float mx = -INFINITY;
  for (int j = lane; j < vc; j += 32) mx = fmaxf(mx, zr[j]);
  mx = warp_max(mx);
  float s = 0.f;
  for (int j = lane; j < vc; j += 32) s += expf(zr[j] - mx);
  s = warp_sum(s);
  if (lane == 0) {
    const float m0 = m_run[row];
    const float mn = fmaxf(m0, mx);
    l_run[row] = l_run[row] * expf(m0 - mn) + s * expf(mx - mn);
    m_run[row] = mn;
    const int t = tgt[row];
    if (t >= c0 && t < c0 + vc) zt[row] = zr[t - c0];
  }
}

__global__ void lse_init_kernel(int64_t M, float* m_run, float* l_run, float* zt) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < M) {
    m_run[i] = -INFINITY;
    l_run[i] = 0.f;
    zt[i] = 0.f;
  }
}

// loss = mean over rows of (m + log l - z_target), one block in a fixed order;
// m_run becomes the log-sum-exp for pass 2.
__global__ void loss_kernel(int64_t M, float* __restrict__ m_run, const float* __restrict__ l_run,
                            const float* __restrict__ zt, float* __restrict__ loss) {
  __shared__ float part[1024];
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < M; i += blockDim.x) {
    const float lse = m_run[i] + logf(l_run[i]);
    m_run[i] = lse;
    s += lse - zt[i];
  }
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = part[0] / static_cast<float>(M);
}

// dz = (exp(z - lse) - [v == target]) / M for one chunk, bf16.
__global__ void dlogits_kernel(const float* __restrict__ z, int64_t M, int vc, int c0, const int32_t* __restrict__ tgt,
                               const float* __restrict__ lse, __nv_bfloat16* __restrict__ dz, float inv_m) {
  const int64_t n = M * vc;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / vc;
    const int j = static_cast<int>(i - row * vc);
    float p = expf(z[i] - lse[row]);
    if (tgt[row] == c0 + j) p -= 1.f;
    dz[i] = __float2bfloat16_rn(p * inv_m);
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = __float2bfloat16_rn(x[i]);
}

// Token ids outside [0, V) read row 0 and are counted in *bad (a caller error).
__global__ void embed_gather_kernel(const int32_t* __restrict__ tok, const uint4* __restrict__ E, uint4* __restrict__ x,
                                    int64_t M, int hc, int V, int32_t* bad) {
  const int64_t n = M * hc;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / hc;
    const int c = static_cast<int>(i - row * hc);
    int t = tok[row];
    if (t < 0 || t >= V) {
      if (c == 0) atomicAdd(bad, 1);
      t = 0;
    }
    x[i] = E[static_cast<int64_t>(t) * hc + c];
  }
}

// dE[v] = sum of dx0 over the rows whose token is v, in increasing row order:
// `order` lists the rows sorted by token (stable), `start[v]..start[v+1]` are
// token v's rows. One block per vocabulary row with a non-empty range.
__global__ void embed_scatter_kernel(const int32_t* __restrict__ order, const int32_t* __restrict__ start,
                                     const __nv_bfloat16* __restrict__ dx, float* __restrict__ dE, int H, int V) {
  const int v = blockIdx.x;
  if (v >= V) return;
  const int a = start[v], b = start[v + 1];
  for (int c = threadIdx.x; c < H; c += blockDim.x) {
    float s = 0.f;
    for (int k = a; k < b; ++k) s += __bfloat162float(dx[static_cast<int64_t>(order[k]) * H + c]);
    dE[static_cast<int64_t>(v) * H + c] = s;
  }
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  return static_cast<int>(std::max<int64_t>(1, std::min(b, cap)));
}

struct HeadWs {
  mt_bf16* h;
  float *rstd, *m, *l, *zt, *z, *dh_acc;
  mt_bf16 *dz, *dh;
  float* red;
};

Bump carve_head(int64_t M, int H, int vc, void* base, uint64_t cap, HeadWs* w) {
  Bump bp(base, cap);
  w->h = bp.take<mt_bf16>(M * H);
  w->rstd = bp.take<float>(M);
  w->m = bp.take<float>(M);
  w->l = bp.take<float>(M);
  w->zt = bp.take<float>(M);
  w->z = bp.take<float>(M * vc);
  w->dz = bp.take<mt_bf16>(M * vc);
  w->dh_acc = bp.take<float>(M * H);
  w->dh = bp.take<mt_bf16>(M * H);
  w->red = bp.take<float>(static_cast<int64_t>(colsum_ws_bytes(M, H) / 4));
  return bp;
}

}  // namespace
}  // namespace mt

using namespace mt;

extern "C" {

uint64_t mt_head_workspace_bytes(int64_t M, int32_t H, int32_t V, int32_t vocab_chunk) {
  if (M <= 0 || H <= 0 || V <= 0 || vocab_chunk <= 0) return 0;
  HeadWs w;
  return carve_head(M, H, std::min(vocab_chunk, V), nullptr, 0, &w).used;
}

mt_status mt_head_loss_fwd_bwd(const mt_bf16* y, const mt_bf16* gf, const mt_bf16* W, const int32_t* targets,
                               int64_t M, int32_t H, int32_t V, float eps, int32_t vocab_chunk, float* loss,
                               mt_bf16* dy, float* dgf, float* dW, void* ws, uint64_t ws_bytes, void* stream) {
  if (!y || !gf || !W || !targets || !loss || !dy || !dgf || !dW || !ws)
    return fail(MT_ERR_INVALID_ARG, "head: NULL pointer");
  if (M <= 0 || M >= (1ll << 31) || H <= 0 || H % 8 || V <= 0 || V % 8 || vocab_chunk <= 0 || vocab_chunk % 8)
    return fail(MT_ERR_INVALID_ARG, "head: need M > 0 and H, V, vocab_chunk positive multiples of 8");
  if (!aligned16(y) || !aligned16(gf) || !aligned16(W) || !aligned16(dy) || !aligned16(dW) || !aligned16(ws))
    return fail(MT_ERR_ALIGNMENT, "head: 16-byte alignment");
  const int vc_max = std::min(vocab_chunk, V);
  HeadWs w;
  Bump bp = carve_head(M, H, vc_max, ws, ws_bytes, &w);
  if (!bp.ok()) return fail(MT_ERR_WORKSPACE, "head: workspace %llu < %llu bytes", (unsigned long long)ws_bytes,
                            (unsigned long long)bp.used);
  cudaStream_t st = as_stream(stream);
  MT_TRY(rmsnorm_fwd_launch(y, gf, w.h, w.rstd, M, H, eps, st));
  lse_init_kernel<<<grid_for(M, 256), 256, 0, st>>>(M, w.m, w.l, w.zt);
  MT_TRY(launch_check("lse_init_kernel"));
  // pass 1: log-sum-exp and target logits
  for (int c0 = 0; c0 < V; c0 += vc_max) {
    const int vc = std::min(vc_max, V - c0);
    MT_TRY(gemm_launch(w.h, H, false, W + static_cast<int64_t>(c0) * H, H, false, w.z, vc, true, false, M, vc, H,
                       nullptr, nullptr, 0, st));
    lse_update_kernel<<<static_cast<unsigned>((M + 7) / 8), 256, 0, st>>>(w.z, M, vc, c0, targets, w.m, w.l, w.zt);
    MT_TRY(launch_check("lse_update_kernel"));
  }
  loss_kernel<<<1, 1024, 0, st>>>(M, w.m, w.l, w.zt, loss);
  MT_TRY(launch_check("loss_kernel"));
  // pass 2: dz per chunk; dW_c = dz^T h; dh += dz W_c
  const float inv_m = 1.0f / static_cast<float>(M);
  for (int c0 = 0; c0 < V; c0 += vc_max) {
    const int vc = std::min(vc_max, V - c0);
    const mt_bf16* Wc = W + static_cast<int64_t>(c0) * H;
    MT_TRY(gemm_launch(w.h, H, false, Wc, H, false, w.z, vc, true, false, M, vc, H, nullptr, nullptr, 0, st));
    dlogits_kernel<<<grid_for(M * vc, 256), 256, 0, st>>>(w.z, M, vc, c0, targets, w.m, reinterpret_cast<__nv_bfloat16*>(w.dz),
                                                           inv_m);
    MT_TRY(launch_check("dlogits_kernel"));
    MT_TRY(gemm_launch(w.dz, vc, true, w.h, H, true, dW + static_cast<int64_t>(c0) * H, H, true, false, vc, H, M,
                       nullptr, nullptr, 0, st));
    MT_TRY(gemm_launch(w.dz, vc, false, Wc, H, true, w.dh_acc, H, true, c0 > 0, M, H, vc, nullptr, nullptr, 0, st));
  }
  f32_to_bf16_kernel<<<grid_for(M * H, 256), 256, 0, st>>>(w.dh_acc, reinterpret_cast<__nv_bfloat16*>(w.dh), M * H);
  MT_TRY(launch_check("f32_to_bf16_kernel"));
  return rmsnorm_bwd_launch(w.dh, y, gf, w.rstd, nullptr, dy, dgf, M, H, w.red, st);
}

mt_status mt_embed_fwd(const int32_t* tokens, const mt_bf16* E, mt_bf16* x, int64_t M, int32_t H, int32_t V,
                       int32_t* bad_tokens, void* stream) {
  if (!tokens || !E || !x || !bad_tokens) return fail(MT_ERR_INVALID_ARG, "embed_fwd: NULL pointer");
  if (M < 0 || H <= 0 || H % 8 || V <= 0) return fail(MT_ERR_INVALID_ARG, "embed_fwd: need H % 8 == 0, V > 0");
  if (!aligned16(E) || !aligned16(x)) return fail(MT_ERR_ALIGNMENT, "embed_fwd: 16-byte alignment");
  if (M == 0) return MT_OK;
  const int hc = H / 8;
  embed_gather_kernel<<<grid_for(M * hc, 256), 256, 0, as_stream(stream)>>>(
      tokens, reinterpret_cast<const uint4*>(E), reinterpret_cast<uint4*>(x), M, hc, V, bad_tokens);
  return launch_check("embed_gather_kernel");
}

mt_status mt_embed_sort(const int32_t* tokens, int64_t M, int32_t V, int32_t* order, int32_t* start) {
  if (!tokens || !order || !start) return fail(MT_ERR_INVALID_ARG, "embed_sort: NULL pointer");
  if (M < 0 || M >= (1ll << 31) || V <= 0) return fail(MT_ERR_INVALID_ARG, "embed_sort: bad sizes");
  for (int32_t v = 0; v <= V; ++v) start[v] = 0;
  for (int64_t i = 0; i < M; ++i) {
    if (tokens[i] < 0 || tokens[i] >= V) return fail(MT_ERR_INVALID_ARG, "embed_sort: token %d out of range", tokens[i]);
    ++start[tokens[i] + 1];
  }
  for (int32_t v = 0; v < V; ++v) start[v + 1] += start[v];
  std::vector<int32_t> pos(start, start + V);
  for (int64_t i = 0; i < M; ++i) order[pos[tokens[i]]++] = static_cast<int32_t>(i);  // stable: rows in order
  return MT_OK;
}

mt_status mt_embed_bwd(const int32_t* order, const int32_t* start, const mt_bf16* dx, float* dE, int32_t H, int32_t V,
                       void* stream) {
  if (!order || !start || !dx || !dE) return fail(MT_ERR_INVALID_ARG, "embed_bwd: NULL pointer");
  if (H <= 0 || V <= 0) return fail(MT_ERR_INVALID_ARG, "embed_bwd: bad sizes");
  embed_scatter_kernel<<<V, 256, 0, as_stream(stream)>>>(order, start, reinterpret_cast<const __nv_bfloat16*>(dx), dE,
                                                         H, V);
  return launch_check("embed_scatter_kernel");
}

}  // extern "C"
