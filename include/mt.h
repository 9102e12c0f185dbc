/*
 * mt.h - C ABI of the B200 layer-streaming training hot path.
 *
 * What the library computes comes from the MegaTrain pages ("MegaTrain: Full
 * Precision Training of 100B+ Parameter Large Language Models on a Single
 * GPU"): parameters live in host memory, the GPU is a transient engine that
 * streams each layer's weights in and its gradients out (abstract; Fig. 2),
 * a double-buffered pipeline over three CUDA streams overlaps weight prefetch
 * (W), compute (F/R/B) and gradient offload (G) (abstract; Fig. 3), stateless
 * layer templates bind weights at call time (abstract; blog summary, design
 * point 4), and activations are checkpointed every K layers and recomputed
 * (blog summary, design point 3). The layer is a Qwen2.5-style decoder block
 * (Table 2 models): pre-RMSNorm, QKV with bias, rotate-half RoPE, causal
 * grouped-query attention, output projection, RMSNorm, SwiGLU MLP, residuals.
 *
 * Conventions shared by every entry point
 * - Every call returns mt_status. Nothing throws, aborts or traps. On an error
 *   mt_last_error() returns a thread-local message describing it.
 * - Arguments are validated before anything is enqueued on a stream.
 * - Device pointers, workspaces and streams belong to the caller. The library
 *   owns only what its *_create calls allocate, freed by the matching
 *   *_destroy.
 * - Kernel and layer entry points are asynchronous on the given stream
 *   (a cudaStream_t passed as void*; NULL is the legacy default stream).
 * - bf16 tensors are passed as raw 16-bit patterns (mt_bf16).
 * - Activations are row-major [B, T, hidden] with token t at position t of its
 *   sequence. Weights follow nn.Linear: W[out, in], y = x W^T.
 * - Kernels that wait on barriers wait a bounded time; a wait that runs out
 *   sets a device error word (read with mt_device_error) and the kernel
 *   returns without finishing its output.
 * - The library caches per-device state (kernel attributes, device addresses
 *   of its own arrays) for the life of the process: no call may follow a
 *   cudaDeviceReset of a device it has used.
 */
#ifndef MT_H
#define MT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t mt_bf16;

typedef enum mt_status {
  MT_OK = 0,
  MT_ERR_INVALID_ARG = 1,  /* null pointer, bad size or shape, mismatched config */
  MT_ERR_ALIGNMENT = 2,    /* pointer or leading dimension not 16-byte aligned */
  MT_ERR_WORKSPACE = 3,    /* workspace smaller than the *_workspace_bytes value */
  MT_ERR_OOM = 4,          /* host (pinned) allocation failed */
  MT_ERR_CUDA = 5,         /* a CUDA runtime call failed; message has its string */
  MT_ERR_TIMEOUT = 6,      /* a bounded host wait ran out */
  MT_ERR_SINK = 7,         /* the gradient sink returned non-zero */
  MT_ERR_INJECTED = 8,     /* a failure injected through mt_engine_opts */
  MT_ERR_UNSUPPORTED = 9,  /* shape the kernels do not implement (e.g. head_dim != 128 or 64) */
  MT_ERR_DEVICE = 10       /* a kernel's bounded wait ran out (see mt_device_error) */
} mt_status;

/* One Qwen2.5-style decoder layer (MegaTrain, Table 2 models; the pages do
 * not write the block out, the plain Qwen2.5 reading is used). */
typedef struct mt_layer_cfg {
  int32_t hidden;      /* H */
  int32_t n_q_heads;   /* nq */
  int32_t n_kv_heads;  /* nkv, divides nq; query head h reads kv head h*nkv/nq */
  int32_t head_dim;    /* d: 64 or 128 */
  int32_t ffn;         /* F */
  int32_t qkv_bias;    /* 1: q, k, v projections carry a bias */
  float rms_eps;       /* RMSNorm epsilon, inside the square root */
  float rope_theta;    /* RoPE base: angle t * theta^(-2i/d) */
} mt_layer_cfg;

/* Element offsets of each tensor inside one layer record (the flat layout of
 * the blog summary's "flat tensor layout"). Record order: g1, Wq, Wk, Wv, bq,
 * bk, bv, Wo, g2, Wg, Wu, Wd. Wq/Wk/Wv are contiguous (one GEMM covers them),
 * so are bq/bk/bv and Wg/Wu. Blocks g1, Wqkv, bqkv, Wo, g2, Wgu, Wd each start
 * on a multiple of 128 elements (256 bytes in bf16, 512 bytes in fp32). The
 * same offsets index the bf16 weight record and the fp32 gradient record. */
typedef struct mt_param_offsets {
  uint64_t g1, wq, wk, wv, bq, bk, bv, wo, g2, wg, wu, wd;
  uint64_t record_elems; /* padded length of one record, a multiple of 128 */
  uint64_t param_count;  /* logical parameter count (no padding) */
} mt_param_offsets;

/* Thread-local description of the last error returned on this thread. */
const char* mt_last_error(void);

/* Reads (and with clear != 0, zeroes) the device error word that kernels set
 * when a bounded wait runs out. Synchronous on the device. */
mt_status mt_device_error(int32_t* out_code, int32_t clear);

/* ------------------------------------------------------------------------ */
/* Layer geometry                                                            */
/* ------------------------------------------------------------------------ */

/* Logical parameter count of one layer: 233,057,792 for the Qwen2.5-7B shape
 * (MegaTrain Table 5: depth deltas of the 7B-width models). Returns 0 for an
 * invalid cfg. */
uint64_t mt_layer_param_count(const mt_layer_cfg* cfg);

/* Fills *out with the record layout described above. */
mt_status mt_layer_param_offsets(const mt_layer_cfg* cfg, mt_param_offsets* out);

/* Bytes of device workspace mt_layer_fwd and mt_layer_recompute_bwd need for
 * B sequences of T tokens. mlp_chunk = 0 runs the MLP over all B*T tokens at
 * once; otherwise over consecutive chunks of that many tokens (MegaTrain
 * Table 7 footnote: chunked MLP execution for ultra-long contexts). */
uint64_t mt_layer_workspace_bytes(const mt_layer_cfg* cfg, int32_t B, int32_t T, int32_t mlp_chunk);

/* ------------------------------------------------------------------------ */
/* Stateless layer templates (MegaTrain abstract: "stateless layer templates, */
/* binding weights dynamically as they stream in")                          */
/* ------------------------------------------------------------------------ */

/* y = layer(x) with the weights of one bf16 record at w_dev (device, layout of
 * mt_layer_param_offsets). x, y: device [B, T, H] bf16; x and y must not
 * overlap. ws: device workspace of at least mt_layer_workspace_bytes. All
 * pointers 16-byte aligned. Asynchronous on stream. */
mt_status mt_layer_fwd(const mt_layer_cfg* cfg, const mt_bf16* w_dev, const mt_bf16* x, mt_bf16* y,
                       int32_t B, int32_t T, int32_t mlp_chunk, void* ws, uint64_t ws_bytes,
                       void* stream);

/* Recompute ("R" in MegaTrain Fig. 3) the layer's internals from its input x,
 * then run its backward ("B"): given dy = dLoss/dy, write dx = dLoss/dx
 * (device [B, T, H] bf16) and the fp32 gradient record dw_dev (device, same
 * offsets as the weights; overwritten, padding untouched). Every weight and
 * bias gradient is summed over all B*T tokens in a fixed order, so the result
 * is bitwise reproducible. dx may alias dy. Asynchronous on stream. */
mt_status mt_layer_recompute_bwd(const mt_layer_cfg* cfg, const mt_bf16* w_dev, const mt_bf16* x,
                                 const mt_bf16* dy, mt_bf16* dx, float* dw_dev, int32_t B, int32_t T,
                                 int32_t mlp_chunk, void* ws, uint64_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Block kernels (each used by the layer templates; exported for testing)   */
/* ------------------------------------------------------------------------ */

/* C = A * B^T on the tcgen05 tensor cores, bf16 operands, fp32 accumulation.
 * Logical A is [M, K], logical B is [N, K].
 *   a_mn_major = 0: A[m,k] = A[m*lda + k];  1: A[m,k] = A[k*lda + m]
 *   b_mn_major = 0: B[n,k] = B[n*ldb + k];  1: B[n,k] = B[k*ldb + n]
 * C[m,n] = C[m*ldc + n], bf16 (c_f32 = 0) or fp32 (c_f32 = 1). Epilogue, in
 * this order: + bias[n] (bf16, may be NULL), + residual[m*ldr + n] (bf16, may
 * be NULL), + previous C (only with c_f32 and accumulate = 1).
 * Pointers 16-byte aligned, lda/ldb/ldc/ldr multiples of 8 elements. */
mt_status mt_gemm_bf16(const mt_bf16* A, int64_t lda, int32_t a_mn_major,
                       const mt_bf16* Bm, int64_t ldb, int32_t b_mn_major,
                       void* C, int64_t ldc, int32_t c_f32, int32_t accumulate,
                       int64_t M, int64_t N, int64_t K,
                       const mt_bf16* bias, const mt_bf16* residual, int64_t ldr, void* stream);

/* The gate/up projection with the SwiGLU activation as its epilogue (2-SM
 * tcgen05 kernel). Wgu is [2F, K] (Wg rows then Wu rows, K-major), A is [M, K]
 * K-major. m[r, j] = silu(g) * u with g = A_r . Wg_j and u = A_r . Wu_j taken
 * from the fp32 accumulators; when gu is not NULL, g and u are also stored
 * (bf16) to gu[r, j] and gu[r, F + j]. Pointers 16-byte aligned; lda, ldw,
 * ldm, ld_gu and F multiples of 8. */
mt_status mt_gemm_swiglu_bf16(const mt_bf16* A, int64_t lda, const mt_bf16* Wgu, int64_t ldw, mt_bf16* m,
                              int64_t ldm, mt_bf16* gu, int64_t ld_gu, int64_t M, int64_t F, int64_t K, void* stream);

/* The MLP's input-gradient GEMM with the SwiGLU backward as its epilogue: dm =
 * dY Wd (dY [M, K] K-major, Wd [K, F] row-major as stored in the layer record,
 * K = hidden) is formed in fp32 and never stored; gu holds [g | u] (row r at
 * gu + r * ld_gu, g in columns [0, F), u in [F, 2F)) on entry and
 * [dg | du] = [dm u silu'(g) | dm silu(g)] (bf16) on return, in place. The
 * SwiGLU derivative follows from the MLP's definition (Qwen2.5 block as read for
 * MegaTrain's layer template). Pointers 16-byte aligned; ld_dy, ldw, ld_gu and
 * F multiples of 8. MT_ERR_INVALID_ARG / MT_ERR_ALIGNMENT before any launch. */
mt_status mt_gemm_swiglu_bwd_bf16(const mt_bf16* dY, int64_t ld_dy, const mt_bf16* Wd, int64_t ldw, mt_bf16* gu,
                                  int64_t ld_gu, int64_t M, int64_t F, int64_t K, void* stream);

/* RMSNorm forward over rows of H: y = x * rstd * g, rstd = 1/sqrt(mean x^2 + eps)
 * (fp32 [rows] out). */
mt_status mt_rmsnorm_fwd(const mt_bf16* x, const mt_bf16* g, mt_bf16* y, float* rstd,
                         int64_t rows, int32_t H, float eps, void* stream);

/* Bytes of workspace mt_rmsnorm_bwd needs (fixed-order partial sums of dg). */
uint64_t mt_rmsnorm_bwd_workspace_bytes(int64_t rows, int32_t H);

/* RMSNorm backward: dx = rstd*(g*dy - xh*mean(xh*g*dy)) + dres (dres may be
 * NULL), xh = x*rstd; dg[j] = sum_rows dy*xh (fp32, fixed summation order).
 * dx may alias dy or dres. */
mt_status mt_rmsnorm_bwd(const mt_bf16* dy, const mt_bf16* x, const mt_bf16* g, const float* rstd,
                         const mt_bf16* dres, mt_bf16* dx, float* dg, int64_t rows, int32_t H,
                         void* ws, uint64_t ws_bytes, void* stream);

/* The same RMSNorm backward for callers that cannot allocate device memory:
 * code whose device memory is owned and budgeted by another allocator (a
 * framework's caching pool, a fixed budget reserved at start-up) and that has
 * no spare buffer to hand over as workspace. It takes no workspace and calls
 * no allocation routine; its scratch is a fixed 8 MiB array inside the library
 * that every GPU which loads the library holds until the process exits. The
 * MegaTrain pages have no counterpart: this is a calling convention only.
 * - Limit: ceil(rows / 64) * H <= 2,097,152 (e.g. 32,768 rows of 3584, or
 *   16,384 rows of 8192); larger calls return MT_ERR_WORKSPACE and change nothing.
 * - The first call on each device looks up the array's device address with
 *   that device current (cudaGetSymbolAddress); make that first call before
 *   any stream capture.
 * - All calls share the one array and it keeps the last call's contents. Every
 *   partial sum a call reads it has written itself, so nothing needs clearing,
 *   but calls that overlap on the GPU (different streams, or different host
 *   threads without ordering) race on it: order them on one stream.
 * Arguments and results are those of mt_rmsnorm_bwd; results are bitwise equal
 * to it. */
mt_status mt_rmsnorm_bwd_noalloc(const mt_bf16* dy, const mt_bf16* x, const mt_bf16* g, const float* rstd,
                                 const mt_bf16* dres, mt_bf16* dx, float* dg, int64_t rows, int32_t H, void* stream);

/* Rotate-half RoPE in place on the first n_heads heads (of head_dim d) of each
 * row of x (row stride ld elements; rows are [B, T], position = t). Pair
 * (i, i+d/2) rotates by t*theta^(-2i/d); inverse = 1 rotates by the negative
 * angle (the adjoint, used in the backward). Angles and their cos/sin are
 * formed in fp64, the rotation is done in fp32. */
mt_status mt_rope(mt_bf16* x, int64_t ld, int32_t B, int32_t T, int32_t n_heads, int32_t head_dim,
                  float theta, int32_t inverse, void* stream);

/* SwiGLU forward: gu is [rows, 2F] (gate in columns [0,F), up in [F,2F));
 * m[r, j] = silu(g) * u, m is [rows, F]. */
mt_status mt_swiglu_fwd(const mt_bf16* gu, mt_bf16* m, int64_t rows, int32_t F, void* stream);

/* SwiGLU backward: dgu[:, :F] = dm*u*sig(g)*(1+g*(1-sig(g))), dgu[:, F:] = dm*silu(g). */
mt_status mt_swiglu_bwd(const mt_bf16* dm, const mt_bf16* gu, mt_bf16* dgu, int64_t rows, int32_t F,
                        void* stream);

/* Bytes of workspace mt_colsum needs. */
uint64_t mt_colsum_workspace_bytes(int64_t rows, int64_t cols);

/* out[j] = sum_r X[r*ld + j] in fp32, fixed summation order (bias gradients). */
mt_status mt_colsum(const mt_bf16* X, int64_t rows, int64_t cols, int64_t ld, float* out,
                    void* ws, uint64_t ws_bytes, void* stream);

/* Causal grouped-query flash attention forward. qkv rows (stride ld_qkv) hold
 * nq query heads, then nkv key heads, then nkv value heads, d each, already
 * rotated. o: [B*T, nq*d] (stride ld_o); lse: fp32 [B, nq, T], natural log of
 * each softmax denominator (scores scaled by 1/sqrt(d)). */
mt_status mt_attention_fwd(const mt_bf16* qkv, int64_t ld_qkv, mt_bf16* o, int64_t ld_o, float* lse,
                           int32_t B, int32_t T, int32_t nq, int32_t nkv, int32_t d, void* stream);

/* Bytes of workspace mt_attention_bwd needs. */
uint64_t mt_attention_bwd_workspace_bytes(int32_t B, int32_t T, int32_t nq);

/* Backward of mt_attention_fwd. d_o: [B*T, nq*d] (stride ld_o, same as o).
 * dqkv gets dq, dk, dv in the qkv column layout (stride ld_qkv), gradients
 * with respect to the rotated q and k. Deterministic: no atomics; each key/value
 * head adds its query heads in a fixed order. */
mt_status mt_attention_bwd(const mt_bf16* qkv, int64_t ld_qkv, const mt_bf16* o, const mt_bf16* d_o,
                           int64_t ld_o, const float* lse, mt_bf16* dqkv, int32_t B, int32_t T,
                           int32_t nq, int32_t nkv, int32_t d, void* ws, uint64_t ws_bytes,
                           void* stream);

/* ------------------------------------------------------------------------ */
/* Host store (MegaTrain Fig. 2: host memory is the authoritative parameter  */
/* store; blog summary: flat layout, host memory linear in parameters)      */
/* ------------------------------------------------------------------------ */

typedef struct mt_host_store mt_host_store;

/* Pinned host store of n_layers records: a bf16 streaming copy and, when
 * keep_fp32_master != 0, the fp32 master values. Contents start zeroed. */
mt_status mt_host_store_create(const mt_layer_cfg* cfg, int32_t n_layers, int32_t keep_fp32_master,
                               mt_host_store** out);
/* Pointers to layer l's records (NULL when out of range / no master). */
float* mt_host_store_master(mt_host_store* s, int32_t layer);
mt_bf16* mt_host_store_bf16(mt_host_store* s, int32_t layer);
/* bf16 copy := round-to-nearest-even(master), on n_threads host threads. */
mt_status mt_host_store_refresh_bf16(mt_host_store* s, int32_t n_threads);
void mt_host_store_destroy(mt_host_store* s);

/* ------------------------------------------------------------------------ */
/* Streaming engine (MegaTrain abstract and Fig. 3: three streams, double   */
/* buffering; blog summary design points 2-4; Table 4: gradient slab pool)  */
/* ------------------------------------------------------------------------ */

typedef struct mt_engine_opts {
  int32_t ckpt_interval;   /* K: layer l's input is kept when l % K == 0 (>= 1) */
  int32_t n_weight_slots;  /* device weight buffers; 0 = max(2, K) */
  int32_t n_host_slabs;    /* pinned fp32 gradient slabs in the pool (>= 1; 0 = 3) */
  int32_t n_dev_grad_slabs;/* device fp32 gradient staging records (>= 1; 0 = 2) */
  int32_t mlp_chunk;       /* 0 = whole batch, else tokens per MLP chunk */
  int32_t resident;        /* 1: every layer's weights stay on the device (no streaming) */
  int32_t timeout_ms;      /* bound of every host wait (0 = 60000) */
  int32_t fail_h2d_at;     /* fault injection: the n-th weight copy fails (0 = off) */
  int32_t time_gemms;      /* 1: time every GEMM launch with CUDA events (stats) */
  int32_t no_slab_pool;    /* 1: pin a gradient record per layer and free it after its sink
                              (the "w/o Gradient Slab Pool" ablation of MegaTrain Table 4) */
  int32_t trace;           /* 1: time every weight upload, layer call and gradient offload of a
                              step with CUDA events (read back with mt_engine_trace) */
  int32_t recompute_internals; /* 0 (default): a segment's re-forward (and the last segment's forward)
                              keeps each layer's internals in a workspace of its own, min(K, L) of
                              them, and the layer's backward reuses them; only the top layer of each
                              earlier segment recomputes its internals. 1: one layer workspace, and
                              every backward but the top layer's recomputes (less device memory). */
} mt_engine_opts;

/* One interval of a traced step (MegaTrain Fig. 3's timeline: H2D, compute and
 * D2H on their three streams). Times are milliseconds on the device clock from
 * an event recorded on the compute stream when the step starts. */
typedef struct mt_trace_rec {
  int32_t kind;     /* 0 weight upload (H2D, prefetch stream), 1 forward, 2 segment re-forward,
                       3 recompute + backward (compute stream), 4 gradient offload (D2H, offload stream) */
  int32_t layer;
  float begin_ms, end_ms;
} mt_trace_rec;

/* Gradient sink: called on a library thread, in backward order, with layer l's
 * fp32 gradient record (n_elems = record_elems) in a pinned slab. The slab is
 * valid until the sink returns and is then reused. Return 0 on success. */
typedef int32_t (*mt_grad_sink)(int32_t layer, const float* host_slab, uint64_t n_elems, void* user);

typedef struct mt_engine mt_engine;

/* What a traced step's timeline says about overlap (mt_trace_summarize).
 * Times in milliseconds on the device clock. The compute stream is "idle" at
 * an instant inside the step when none of its layer calls is running; the
 * idle time is attributed to the weight uploads when one is in flight then,
 * else to the gradient offloads when one is in flight, else to neither. */
typedef struct mt_trace_summary {
  double span_ms;          /* step origin (0) to the end of the last interval */
  double h2d_ms;           /* sum of the weight-upload intervals (all pieces of a record) */
  double d2h_ms;           /* sum of the gradient-offload intervals (first piece's start to last piece's end) */
  double fwd_ms, refwd_ms, bwd_ms;  /* compute-stream time of forwards, segment re-forwards, recompute+backward */
  double exposed_h2d_ms;   /* compute stream idle while a weight upload is in flight */
  double exposed_d2h_ms;   /* compute stream idle while a gradient offload but no upload is in flight
                              (this includes the drain after the last backward) */
  double idle_other_ms;    /* compute stream idle with no copy in flight (host enqueue, a loss-head hook) */
} mt_trace_summary;

/* Host-only (no CUDA): summarizes n timeline records (mt_trace_rec, any
 * order; kinds 0-4 as mt_engine_trace gives them). MT_ERR_INVALID_ARG on a
 * NULL pointer, n < 0, an unknown kind or an interval that ends before it
 * begins. */
mt_status mt_trace_summarize(const mt_trace_rec* recs, int32_t n, mt_trace_summary* out);

typedef struct mt_stats {
  double step_ms;             /* host wall time of the last step */
  uint64_t h2d_bytes, d2h_bytes;
  uint64_t layer_fwd_calls, layer_bwd_calls, weight_loads;
  double exec_flops;          /* FLOPs the kernels executed in the last step */
  double gemm_ms;             /* device time of all GEMM launches (time_gemms = 1) */
  double gemm_flops;          /* algorithmic FLOPs of those launches */
  uint64_t gemm_launches;
  uint64_t device_bytes;      /* device workspace bytes the engine uses */
  double sink_ms;             /* host time inside the sink */
  uint64_t kernel_launches;   /* kernels the library launched in the last step */
  int32_t traced;             /* 1 when `trace` below describes the last step (engine created with trace = 1) */
  mt_trace_summary trace;     /* per-phase device times and exposed transfer time of the last step */
} mt_stats;

/* Device workspace the engine needs (weight slots, gradient staging,
 * checkpoints, segment activations, the layer internals sets of
 * recompute_internals and one backward scratch). */
uint64_t mt_engine_workspace_bytes(const mt_layer_cfg* cfg, int32_t n_layers, int32_t B, int32_t T,
                                   const mt_engine_opts* opts);

/* Creates an engine over caller-owned device memory and streams (compute,
 * prefetch and offload must be three distinct streams). Allocates the pinned
 * slab pool and the CUDA events. */
mt_status mt_engine_create(const mt_layer_cfg* cfg, int32_t n_layers, int32_t B, int32_t T,
                           const mt_engine_opts* opts, void* dev_ws, uint64_t dev_ws_bytes,
                           void* compute_stream, void* prefetch_stream, void* offload_stream,
                           mt_engine** out);

/* One training step over the whole stack: forward with checkpoints every K
 * layers, then per segment (last to first) re-forward, recompute and backward,
 * streaming each layer's bf16 weights from the store and each layer's fp32
 * gradients out to the sink. x0, dy_top (inputs) and y_top, dx0 (outputs) are
 * device [B, T, H] bf16. Synchronous: returns after the last sink call. */
mt_status mt_stream_step(mt_engine* e, mt_host_store* store, const mt_bf16* x0, const mt_bf16* dy_top,
                         mt_bf16* y_top, mt_bf16* dx0, mt_grad_sink sink, void* user);

/* Called on the enqueuing thread once per step, after the last layer's
 * forward has been enqueued and before the first backward work: enqueue, on
 * compute_stream, whatever turns y_top into dy_top (a final norm, LM head and
 * loss, for instance). Return MT_OK to continue the step. */
typedef mt_status (*mt_head_hook)(const mt_bf16* y_top, mt_bf16* dy_top, void* compute_stream, void* user);

/* mt_stream_step with a head between forward and backward: when hook is not
 * NULL, dy_top is written by the hook instead of being an input. */
mt_status mt_stream_step_hooked(mt_engine* e, mt_host_store* store, const mt_bf16* x0, mt_bf16* dy_top,
                                mt_bf16* y_top, mt_bf16* dx0, mt_grad_sink sink, void* user, mt_head_hook hook,
                                void* hook_user);

/* Same step with x0/dy_top/y_top/dx0 in host memory (pinned for full speed):
 * the inputs are copied in and the outputs copied out inside the call. */
mt_status mt_stream_step_host(mt_engine* e, mt_host_store* store, const mt_bf16* x0_host,
                              const mt_bf16* dy_top_host, mt_bf16* y_top_host, mt_bf16* dx0_host,
                              mt_grad_sink sink, void* user);

/* Counters of the engine's last step (mt_stats above; its `trace` part is filled when
 * the engine was created with trace = 1). MT_ERR_INVALID_ARG on NULL. */
mt_status mt_engine_stats(const mt_engine* e, mt_stats* out);
/* The timeline of the engine's last completed step, in issue order (engine
 * created with trace = 1; call after mt_stream_step returned MT_OK). Writes
 * min(*n, cap) records to out and the number available to *n.
 * MT_ERR_INVALID_ARG when tracing is off or no traced step has run. */
mt_status mt_engine_trace(mt_engine* e, mt_trace_rec* out, int32_t cap, int32_t* n);
/* Waits (bounded) for the engine's streams and clears a failed step's state. */
mt_status mt_engine_reset(mt_engine* e);
void mt_engine_destroy(mt_engine* e);

/* ------------------------------------------------------------------------ */
/* Embedding, final norm, LM head and loss (the pages count embedding and   */
/* head in the parameters, Table 5; the Qwen2.5 reading: untied E and W)    */
/* ------------------------------------------------------------------------ */

/* x[r] = E[tokens[r]] for M rows of H (bf16). tokens: device int32. A token
 * outside [0, V) reads row 0 and increments *bad_tokens (device int32). */
mt_status mt_embed_fwd(const int32_t* tokens, const mt_bf16* E, mt_bf16* x, int64_t M, int32_t H, int32_t V,
                       int32_t* bad_tokens, void* stream);

/* Host helper (no CUDA): the rows 0..M-1 stably sorted by token into order[M],
 * and start[V+1] with token v's rows at order[start[v] .. start[v+1]). */
mt_status mt_embed_sort(const int32_t* tokens, int64_t M, int32_t V, int32_t* order, int32_t* start);

/* dE[v] = sum over token v's rows of dx (fp32 [V, H], every row written),
 * added in increasing row order (bitwise repeatable). order/start: device
 * copies of mt_embed_sort's output. */
mt_status mt_embed_bwd(const int32_t* order, const int32_t* start, const mt_bf16* dx, float* dE, int32_t H, int32_t V,
                       void* stream);

/* Workspace of mt_head_loss_fwd_bwd. */
uint64_t mt_head_workspace_bytes(int64_t M, int32_t H, int32_t V, int32_t vocab_chunk);

/* Final RMSNorm (gain gf, eps) + LM head W [V, H] + mean cross-entropy over M
 * rows of the stack output y against targets (device int32 in [0, V)), and its
 * backward, over vocabulary chunks of vocab_chunk rows of W (the full logits
 * never exist). Outputs: *loss (device fp32), dy [M, H] bf16, dgf [H] fp32,
 * dW [V, H] fp32 (overwritten). H, V and vocab_chunk multiples of 8. */
mt_status mt_head_loss_fwd_bwd(const mt_bf16* y, const mt_bf16* gf, const mt_bf16* W, const int32_t* targets,
                               int64_t M, int32_t H, int32_t V, float eps, int32_t vocab_chunk, float* loss,
                               mt_bf16* dy, float* dgf, float* dW, void* ws, uint64_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* CPU optimizer (blog summary, design point 1: the optimizer step runs on   */
/* the CPU with Adam momentum and variance in host memory)                   */
/* ------------------------------------------------------------------------ */

typedef struct mt_adamw_cfg {
  float lr, beta1, beta2, eps, weight_decay;  /* AdamW, decoupled weight decay */
  int32_t n_threads;                           /* host threads (0 = all cores, up to 32) */
} mt_adamw_cfg;

/* One AdamW step (t >= 1) on n host fp32 elements, in place:
 * m = b1 m + (1-b1) g; v = b2 v + (1-b2) g^2;
 * w -= lr * (m/(1-b1^t) / (sqrt(v/(1-b2^t)) + eps) + weight_decay * w). No CUDA. */
mt_status mt_adamw_update(float* w, float* m, float* v, const float* g, uint64_t n, const mt_adamw_cfg* cfg,
                          int64_t t);

typedef struct mt_host_optimizer mt_host_optimizer;

/* AdamW state (m, v zeroed, one step counter per layer) for every record of a
 * store that keeps its fp32 master copy. */
mt_status mt_host_optimizer_create(mt_host_store* store, const mt_adamw_cfg* cfg, mt_host_optimizer** out);
/* A gradient sink for mt_stream_step (user = the optimizer): applies one AdamW
 * step to layer `layer`'s fp32 master from the gradient record and refreshes
 * that layer's bf16 streaming copy (round to nearest even). Returns 0, or 1 on
 * a mismatched layer or record size. */
int32_t mt_host_optimizer_sink(int32_t layer, const float* host_slab, uint64_t n_elems, void* user);
void mt_host_optimizer_destroy(mt_host_optimizer* o);

/* Host-side schedule (no CUDA): for n_layers and interval K, the sequence of
 * layer uses in compute order and, for a pool of n_slots weight buffers, the
 * slot of each use and whether it needs a fresh copy (furthest-next-use
 * eviction). kind[i]: 0 forward, 1 segment re-forward, 2 recompute+backward.
 * Arrays must hold mt_schedule_len(n_layers, K) entries. */
int32_t mt_schedule_len(int32_t n_layers, int32_t K);
mt_status mt_schedule(int32_t n_layers, int32_t K, int32_t n_slots, int32_t* layer, int32_t* kind,
                      int32_t* slot, int32_t* load);

#ifdef __cplusplus
}
#endif

#endif /* MT_H */
