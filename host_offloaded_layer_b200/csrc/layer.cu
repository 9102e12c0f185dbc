// Stateless decoder-layer templates: forward, and recompute + backward.
//
// MegaTrain (abstract; blog summary, design point 4) replaces a persistent
// autograd graph with layer templates that hold no state: the weights of one
// layer are bound at call time (a pointer to its streamed bf16 record) and
// every intermediate lives in a caller workspace whose size depends only on
// the layer shape and the batch, never on the depth of the model.
//
// Forward (the Qwen2.5-style block, MegaTrain Table 2 models):
//   h1 = RMSNorm(x; g1); qkv = h1 Wqkv^T + bqkv; RoPE(q, k);
//   o = causal GQA attention; x2 = x + o Wo^T; h2 = RMSNorm(x2; g2);
//   per MLP chunk: [g|u] = h2 Wgu^T; m = silu(g) * u; y = x2 + m Wd^T.
// Recompute + backward ("R" and "B" of Fig. 3) rebuilds h1, qkv, o, lse, x2,
// h2 (and per chunk g, u, m) and then runs the adjoint of every step; weight
// gradients are fp32 GEMM outputs written straight into the gradient record,
// bias and gain gradients are fixed-order column sums.
#include "mt_internal.h"

namespace mt {

mt_status layer_recompute_bwd_ev(const mt_layer_cfg* cfg, const mt_bf16* w_dev, const mt_bf16* x, const mt_bf16* dy,
                                 mt_bf16* dx, float* dw_dev, int32_t B, int32_t T, int32_t mlp_chunk, void* ws_int,
                                 uint64_t int_bytes, void* ws_scr, uint64_t scr_bytes, void* stream,
                                 cudaEvent_t mlp_done, bool reuse_fwd, cudaEvent_t wd_done);
mt_status layer_fwd_keep(const mt_layer_cfg* cfg, const mt_bf16* w_dev, const mt_bf16* x, mt_bf16* y, int32_t B,
                         int32_t T, int32_t mlp_chunk, void* ws_int, uint64_t int_bytes, void* stream, bool keep,
                         cudaEvent_t mlp_weights);
mt_status layer_ws_sizes(const mt_layer_cfg* cfg, int32_t B, int32_t T, int32_t mlp_chunk, uint64_t* internals,
                         uint64_t* scratch);
mt_status rmsnorm_fwd_launch(const mt_bf16*, const mt_bf16*, mt_bf16*, float*, int64_t, int, float, cudaStream_t);
mt_status rmsnorm_bwd_launch(const mt_bf16*, const mt_bf16*, const mt_bf16*, const float*, const mt_bf16*, mt_bf16*,
                             float*, int64_t, int, void*, cudaStream_t);
mt_status rope_launch(mt_bf16*, int64_t, int, int, int, int, float, bool, cudaStream_t);

mt_status colsum_launch(const mt_bf16*, const mt_bf16*, const float*, int64_t, int64_t, int64_t, float*, void*,
                        cudaStream_t);
uint64_t colsum_ws_bytes(int64_t rows, int64_t cols);
mt_status attn_fwd_launch(const mt_bf16*, int64_t, mt_bf16*, int64_t, float*, int, int, int, int, int, cudaStream_t);
mt_status attn_bwd_launch(const mt_bf16*, int64_t, const mt_bf16*, const mt_bf16*, int64_t, const float*, mt_bf16*,
                          int, int, int, int, int, void*, cudaStream_t);
uint64_t attn_bwd_ws_bytes(int B, int T, int nq);
mt_status attn_bwd_delta_launch(const mt_bf16* qkv, int64_t ld, const mt_bf16* d_o, int64_t ld_o, const float* lse,
                                const float* delta, mt_bf16* dqkv, int B, int T, int nq, int nkv, int d,
                                const float* rope_tab, cudaStream_t st);
mt_status gemm_swiglu_launch(const mt_bf16* A, int64_t lda, const mt_bf16* Wgu, int64_t ldw, mt_bf16* m, int64_t ldm,
                             mt_bf16* gu, int64_t ld_gu, int64_t M, int64_t F, int64_t K, cudaStream_t st);

namespace {

struct LayerWs {
  mt_bf16 *h1, *qkv, *o, *x2, *h2, *gu, *m;
  float *rstd1, *rstd2, *lse;
  float* rope;  // (cos, sin) of every position and rotation pair: [T][d/2] float pairs
  mt_bf16 *dh2, *dx2, *d_o, *dqkv;  // dm reuses m, dgu reuses gu, dh1 reuses dh2
  float* red;
};

// The layer's workspace in two parts. The internals are what a forward leaves for
// its backward (h1, qkv after RoPE, o, x2, h2, the MLP chunk's g|u and m, the two
// rstd vectors, lse and the RoPE table); the scratch holds the backward's own
// buffers. The forward uses only the internals.
Bump carve_internals(const Geom& G, int B, int T, int64_t Mc, void* base, uint64_t cap, LayerWs* w) {
  const int64_t M = static_cast<int64_t>(B) * T;
  Bump bp(base, cap);
  w->h1 = bp.take<mt_bf16>(M * G.H);
  w->qkv = bp.take<mt_bf16>(M * G.Nqkv);
  w->o = bp.take<mt_bf16>(M * G.Nq);
  w->x2 = bp.take<mt_bf16>(M * G.H);
  w->h2 = bp.take<mt_bf16>(M * G.H);
  w->gu = bp.take<mt_bf16>(Mc * 2 * G.F);
  w->m = bp.take<mt_bf16>(Mc * G.F);
  w->rstd1 = bp.take<float>(M);
  w->rstd2 = bp.take<float>(M);
  w->lse = bp.take<float>(static_cast<int64_t>(B) * G.nq * T);
  w->rope = bp.take<float>(static_cast<int64_t>(T) * G.d);
  return bp;
}

Bump carve_scratch(const Geom& G, int B, int T, void* base, uint64_t cap, LayerWs* w) {
  const int64_t M = static_cast<int64_t>(B) * T;
  Bump bp(base, cap);
  w->dh2 = bp.take<mt_bf16>(M * G.H);
  w->dx2 = bp.take<mt_bf16>(M * G.H);
  w->d_o = bp.take<mt_bf16>(M * G.Nq);
  w->dqkv = bp.take<mt_bf16>(M * G.Nqkv);
  uint64_t red = std::max<uint64_t>(colsum_ws_bytes(M, G.H), colsum_ws_bytes(M, G.Nqkv));
  red = std::max<uint64_t>(red, attn_bwd_ws_bytes(B, T, static_cast<int>(G.nq)));
  w->red = bp.take<float>(static_cast<int64_t>(red / 4));
  return bp;
}

int64_t chunk_rows(int64_t M, int mlp_chunk) { return (mlp_chunk <= 0 || mlp_chunk >= M) ? M : mlp_chunk; }

mt_status check_layer_args(const mt_layer_cfg* cfg, Geom* G, int B, int T, int mlp_chunk) {
  MT_TRY(make_geom(cfg, G));
  if (B <= 0 || T <= 0) return fail(MT_ERR_INVALID_ARG, "B and T must be positive");
  if (mlp_chunk < 0) return fail(MT_ERR_INVALID_ARG, "mlp_chunk must be >= 0");
  if (G->d != 64 && G->d != 128) return fail(MT_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (static_cast<int64_t>(B) * T >= (1ll << 31)) return fail(MT_ERR_INVALID_ARG, "B*T too large");
  return MT_OK;
}

// h1, qkv (bias, RoPE), o, lse, x2 = x + o Wo^T, h2 (with rstd1, rstd2).
mt_status attention_half(const Geom& G, const mt_bf16* w, const mt_bf16* x, int B, int T, const LayerWs& ws,
                         cudaStream_t st) {
  const int64_t M = static_cast<int64_t>(B) * T;
  const mt_param_offsets& O = G.off;
  MT_TRY(rmsnorm_fwd_launch(x, w + O.g1, ws.h1, ws.rstd1, M, static_cast<int>(G.H), G.eps, st));
  // qkv = h1 Wqkv^T + bqkv with q and k rotated in the GEMM's epilogue
  MT_TRY(rope_table_launch(ws.rope, T, static_cast<int>(G.d), G.theta, st));
  MT_TRY(gemm_rope_launch(ws.h1, G.H, w + O.wq, G.H, ws.qkv, G.Nqkv, M, G.Nqkv, G.H, G.bias ? w + O.bq : nullptr,
                          ws.rope, static_cast<int>((G.nq + G.nkv) * G.d), static_cast<int>(G.d), T, st));
  MT_TRY(attn_fwd_launch(ws.qkv, G.Nqkv, ws.o, G.Nq, ws.lse, B, T, static_cast<int>(G.nq), static_cast<int>(G.nkv),
                         static_cast<int>(G.d), st));
  MT_TRY(gemm_launch(ws.o, G.Nq, false, w + O.wo, G.Nq, false, ws.x2, G.H, false, false, M, G.H, G.Nq, nullptr, x, G.H,
                     st));
  MT_TRY(rmsnorm_fwd_launch(ws.x2, w + O.g2, ws.h2, ws.rstd2, M, static_cast<int>(G.H), G.eps, st));
  return MT_OK;
}

// [g|u] = h2c Wgu^T; m = silu(g) * u for one chunk of rows, the SwiGLU in the
// GEMM's epilogue (m from the fp32 accumulators; g and u are only written when
// the backward needs them).
mt_status mlp_up(const Geom& G, const mt_bf16* w, const mt_bf16* h2c, int64_t rows, const LayerWs& ws, bool need_gu,
                 cudaStream_t st) {
  const mt_param_offsets& O = G.off;
  return gemm_swiglu_launch(h2c, G.H, w + O.wg, G.H, ws.m, G.F, need_gu ? ws.gu : nullptr, 2 * G.F, rows, G.F, G.H,
                            st);
}

}  // namespace
}  // namespace mt

using namespace mt;

extern "C" {

uint64_t mt_layer_workspace_bytes(const mt_layer_cfg* cfg, int32_t B, int32_t T, int32_t mlp_chunk) {
  uint64_t a = 0, b = 0;
  if (layer_ws_sizes(cfg, B, T, mlp_chunk, &a, &b) != MT_OK) return 0;
  return a + b;
}

// The one workspace of the public entry points: internals first, then scratch.
static mt_status split_ws(const mt_layer_cfg* cfg, int32_t B, int32_t T, int32_t mlp_chunk, void* ws,
                          uint64_t ws_bytes, void** scr, uint64_t* int_bytes, uint64_t* scr_bytes, const char* who) {
  MT_TRY(layer_ws_sizes(cfg, B, T, mlp_chunk, int_bytes, scr_bytes));
  if (ws_bytes < *int_bytes + *scr_bytes)
    return fail(MT_ERR_WORKSPACE, "%s: workspace %llu < %llu bytes", who, (unsigned long long)ws_bytes,
                (unsigned long long)(*int_bytes + *scr_bytes));
  *scr = ws ? static_cast<char*>(ws) + *int_bytes : nullptr;
  return MT_OK;
}

mt_status mt_layer_fwd(const mt_layer_cfg* cfg, const mt_bf16* w_dev, const mt_bf16* x, mt_bf16* y, int32_t B,
                       int32_t T, int32_t mlp_chunk, void* ws, uint64_t ws_bytes, void* stream) {
  void* scr = nullptr;
  uint64_t ni = 0, ns = 0;
  MT_TRY(split_ws(cfg, B, T, mlp_chunk, ws, ws_bytes, &scr, &ni, &ns, "layer_fwd"));
  return layer_fwd_keep(cfg, w_dev, x, y, B, T, mlp_chunk, ws, ni, stream, false, nullptr);
}

mt_status mt_layer_recompute_bwd(const mt_layer_cfg* cfg, const mt_bf16* w_dev, const mt_bf16* x, const mt_bf16* dy,
                                 mt_bf16* dx, float* dw_dev, int32_t B, int32_t T, int32_t mlp_chunk, void* ws,
                                 uint64_t ws_bytes, void* stream) {
  void* scr = nullptr;
  uint64_t ni = 0, ns = 0;
  MT_TRY(split_ws(cfg, B, T, mlp_chunk, ws, ws_bytes, &scr, &ni, &ns, "layer_recompute_bwd"));
  return layer_recompute_bwd_ev(cfg, w_dev, x, dy, dx, dw_dev, B, T, mlp_chunk, ws, ni, scr, ns, stream, nullptr,
                                false, nullptr);
}

}  // extern "C"

mt_status mt::layer_ws_sizes(const mt_layer_cfg* cfg, int32_t B, int32_t T, int32_t mlp_chunk, uint64_t* internals,
                             uint64_t* scratch) {
  Geom G;
  MT_TRY(check_layer_args(cfg, &G, B, T, mlp_chunk));
  LayerWs w;
  *internals = carve_internals(G, B, T, chunk_rows(static_cast<int64_t>(B) * T, mlp_chunk), nullptr, 0, &w).used;
  *scratch = carve_scratch(G, B, T, nullptr, 0, &w).used;
  return MT_OK;
}

// The layer forward. With `keep` the workspace is left holding everything the
// layer's backward would recompute (h1, qkv after RoPE, o, lse, x2, h2, and
// with a single MLP chunk also g, u and m), so that a backward called right
// after it on the same workspace and weights can skip the recompute. When
// `mlp_weights` is given the stream waits for it between the attention half
// and the MLP (the streaming engine uploads a record in two pieces).
mt_status mt::layer_fwd_keep(const mt_layer_cfg* cfg, const mt_bf16* w_dev, const mt_bf16* x, mt_bf16* y, int32_t B,
                             int32_t T, int32_t mlp_chunk, void* ws, uint64_t ws_bytes, void* stream, bool keep,
                             cudaEvent_t mlp_weights) {
  Geom G;
  MT_TRY(check_layer_args(cfg, &G, B, T, mlp_chunk));
  if (!w_dev || !x || !y || !ws) return fail(MT_ERR_INVALID_ARG, "layer_fwd: NULL pointer");
  if (!aligned16(w_dev) || !aligned16(x) || !aligned16(y) || !aligned16(ws))
    return fail(MT_ERR_ALIGNMENT, "layer_fwd: pointers must be 16-byte aligned");
  if (x == y) return fail(MT_ERR_INVALID_ARG, "layer_fwd: x and y must not overlap");
  const int64_t M = static_cast<int64_t>(B) * T;
  const int64_t Mc = chunk_rows(M, mlp_chunk);
  LayerWs w;
  Bump bp = carve_internals(G, B, T, Mc, ws, ws_bytes, &w);
  if (!bp.ok()) return fail(MT_ERR_WORKSPACE, "layer_fwd: workspace %llu < %llu bytes", (unsigned long long)ws_bytes,
                            (unsigned long long)bp.used);
  cudaStream_t st = as_stream(stream);
  MT_TRY(attention_half(G, w_dev, x, B, T, w, st));
  if (mlp_weights) MT_CUDA(cudaStreamWaitEvent(st, mlp_weights, 0));
  const mt_param_offsets& O = G.off;
  for (int64_t r0 = 0; r0 < M; r0 += Mc) {
    const int64_t rows = std::min(Mc, M - r0);
    MT_TRY(mlp_up(G, w_dev, w.h2 + r0 * G.H, rows, w, keep && Mc == M, st));
    MT_TRY(gemm_launch(w.m, G.F, false, w_dev + O.wd, G.F, false, y + r0 * G.H, G.H, false, false, rows, G.H, G.F,
                       nullptr, w.x2 + r0 * G.H, G.H, st));
  }
  return MT_OK;
}

// The layer backward; when mlp_done is given it is recorded on the stream as
// soon as the MLP weights' gradients (Wg, Wu, Wd) are final. With reuse_fwd
// the workspace still holds what layer_fwd_keep(keep = true) left in it for
// these weights and this x, and the recompute is skipped (the values are the
// ones it would produce: every kernel is deterministic).
mt_status mt::layer_recompute_bwd_ev(const mt_layer_cfg* cfg, const mt_bf16* w_dev, const mt_bf16* x,
                                     const mt_bf16* dy, mt_bf16* dx, float* dw_dev, int32_t B, int32_t T,
                                     int32_t mlp_chunk, void* ws_int, uint64_t int_bytes, void* ws_scr,
                                     uint64_t scr_bytes, void* stream, cudaEvent_t mlp_done, bool reuse_fwd,
                                     cudaEvent_t wd_done) {
  Geom G;
  MT_TRY(check_layer_args(cfg, &G, B, T, mlp_chunk));
  if (!w_dev || !x || !dy || !dx || !dw_dev || !ws_int || !ws_scr)
    return fail(MT_ERR_INVALID_ARG, "layer_recompute_bwd: NULL pointer");
  if (!aligned16(w_dev) || !aligned16(x) || !aligned16(dy) || !aligned16(dx) || !aligned16(dw_dev) ||
      !aligned16(ws_int) || !aligned16(ws_scr))
    return fail(MT_ERR_ALIGNMENT, "layer_recompute_bwd: pointers must be 16-byte aligned");
  if (dx == x) return fail(MT_ERR_INVALID_ARG, "layer_recompute_bwd: dx must not alias x");
  const int64_t M = static_cast<int64_t>(B) * T;
  const int64_t Mc = chunk_rows(M, mlp_chunk);
  LayerWs w;
  Bump bi = carve_internals(G, B, T, Mc, ws_int, int_bytes, &w);
  Bump bs = carve_scratch(G, B, T, ws_scr, scr_bytes, &w);
  if (!bi.ok() || !bs.ok())
    return fail(MT_ERR_WORKSPACE, "layer_recompute_bwd: workspace %llu + %llu < %llu + %llu bytes",
                (unsigned long long)int_bytes, (unsigned long long)scr_bytes, (unsigned long long)bi.used,
                (unsigned long long)bs.used);
  cudaStream_t st = as_stream(stream);
  const mt_param_offsets& O = G.off;
  const int H = static_cast<int>(G.H);

  // ---- recompute (R)
  if (!reuse_fwd) MT_TRY(attention_half(G, w_dev, x, B, T, w, st));

  // ---- MLP backward, chunk by chunk in token order
  for (int64_t r0 = 0; r0 < M; r0 += Mc) {
    const int64_t rows = std::min(Mc, M - r0);
    const bool acc = r0 > 0;
    const mt_bf16* h2c = w.h2 + r0 * G.H;
    const mt_bf16* dyc = dy + r0 * G.H;
    if (!(reuse_fwd && Mc == M)) MT_TRY(mlp_up(G, w_dev, h2c, rows, w, true, st));
    // dWd (+)= dy^T m
    MT_TRY(gemm_launch(dyc, G.H, true, w.m, G.F, true, dw_dev + O.wd, G.F, true, acc, G.H, G.F, rows, nullptr, nullptr,
                       0, st));
    if (wd_done && r0 + rows >= M) MT_CUDA(cudaEventRecord(wd_done, st));  // dWd is final after the last chunk
    // dm = dy Wd, and in the same GEMM's epilogue [dg|du] in place over [g|u]
    MT_TRY(gemm_swiglu_bwd_launch(dyc, G.H, false, w_dev + O.wd, G.F, true, w.gu, 2 * G.F, rows, G.F, G.H, st));
    // dWgu (+)= dgu^T h2
    MT_TRY(gemm_launch(w.gu, 2 * G.F, true, h2c, G.H, true, dw_dev + O.wg, G.H, true, acc, 2 * G.F, G.H, rows, nullptr,
                       nullptr, 0, st));
    // dh2 = dgu Wgu
    MT_TRY(gemm_launch(w.gu, 2 * G.F, false, w_dev + O.wg, G.H, true, w.dh2 + r0 * G.H, G.H, false, false, rows, G.H,
                       2 * G.F, nullptr, nullptr, 0, st));
  }
  if (mlp_done) MT_CUDA(cudaEventRecord(mlp_done, st));
  // dx2 = dy + RMSNorm2^T(dh2); dg2
  MT_TRY(rmsnorm_bwd_launch(w.dh2, w.x2, w_dev + O.g2, w.rstd2, dy, w.dx2, dw_dev + O.g2, M, H, w.red, st));
  // dWo = dx2^T o ; do = dx2 Wo
  MT_TRY(gemm_launch(w.dx2, G.H, true, w.o, G.Nq, true, dw_dev + O.wo, G.Nq, true, false, G.H, G.Nq, M, nullptr,
                     nullptr, 0, st));
  // do = dx2 Wo, and in the same GEMM's epilogue delta = rowsum(do * o) per head (the attention
  // backward's D term), into the partial-sum buffer that the column sums reuse only later
  MT_TRY(gemm_dot_launch(w.dx2, G.H, false, w_dev + O.wo, G.Nq, true, w.d_o, G.Nq, M, G.Nq, G.H, w.o, G.Nq, w.red,
                         static_cast<int>(G.d), T, st));
  // attention backward -> dq, dk, dv, with dq and dk un-rotated (the adjoint of RoPE) in the
  // tcgen05 kernels' epilogues for head_dim 128, by a separate pass for head_dim 64
  const bool d128 = G.d == 128;
  MT_TRY(attn_bwd_delta_launch(w.qkv, G.Nqkv, w.d_o, G.Nq, w.lse, w.red, w.dqkv, B, T, static_cast<int>(G.nq),
                               static_cast<int>(G.nkv), static_cast<int>(G.d), d128 ? w.rope : nullptr, st));
  if (!d128)
    MT_TRY(rope_launch(w.dqkv, G.Nqkv, B, T, static_cast<int>(G.nq + G.nkv), static_cast<int>(G.d), G.theta, true,
                       st));
  if (G.bias) MT_TRY(colsum_launch(w.dqkv, nullptr, nullptr, M, G.Nqkv, G.Nqkv, dw_dev + O.bq, w.red, st));
  // dWqkv = dqkv^T h1 ; dh1 = dqkv Wqkv (into the dh2 buffer)
  MT_TRY(gemm_launch(w.dqkv, G.Nqkv, true, w.h1, G.H, true, dw_dev + O.wq, G.H, true, false, G.Nqkv, G.H, M, nullptr,
                     nullptr, 0, st));
  MT_TRY(gemm_launch(w.dqkv, G.Nqkv, false, w_dev + O.wq, G.H, true, w.dh2, G.H, false, false, M, G.H, G.Nqkv, nullptr,
                     nullptr, 0, st));
  // dx = dx2 + RMSNorm1^T(dh1); dg1
  MT_TRY(rmsnorm_bwd_launch(w.dh2, x, w_dev + O.g1, w.rstd1, w.dx2, dx, dw_dev + O.g1, M, H, w.red, st));
  return MT_OK;
}
