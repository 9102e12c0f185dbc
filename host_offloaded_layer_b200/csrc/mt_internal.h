// Internal helpers shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <string>

#include "mt.h"

namespace mt {

// Thread-local error message (mt_last_error).
void set_error(const char* fmt, ...);
mt_status fail(mt_status s, const char* fmt, ...);

inline mt_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return MT_OK;
  return fail(MT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define MT_TRY(expr)                  \
  do {                                \
    mt_status _s = (expr);            \
    if (_s != MT_OK) return _s;       \
  } while (0)

#define MT_CUDA(expr) MT_TRY(::mt::cuda_check((expr), #expr))

// Running count of kernel launches on this thread (engine statistics).
void count_launch();
uint64_t launch_counter();

// Kernel launch check (configuration errors are reported synchronously).
inline mt_status launch_check(const char* name) {
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return MT_OK;
  return fail(MT_ERR_CUDA, "launch of %s: %s", name, cudaGetErrorString(e));
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Number of SMs of the current device (cached per device).
int num_sms();

// Device error word set by bounded waits that ran out (one per device image).
int32_t* device_error_word();

// Error codes written to the device error word.
enum : int32_t {
  DEV_ERR_TIMEOUT_PRODUCER = 1,
  DEV_ERR_TIMEOUT_MMA = 2,
  DEV_ERR_TIMEOUT_EPILOGUE = 3,
};

// Layer geometry derived from mt_layer_cfg.
struct Geom {
  int64_t H, nq, nkv, d, F;
  int64_t Nq, Nkv, Nqkv;  // nq*d, nkv*d, nq*d + 2*nkv*d
  bool bias;
  float eps, theta;
  mt_param_offsets off;
};
mt_status make_geom(const mt_layer_cfg* cfg, Geom* g);

inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// Simple bump allocator over a caller workspace (256-byte aligned slices).
struct Bump {
  char* base;
  uint64_t used, cap;
  explicit Bump(void* b, uint64_t c) : base(static_cast<char*>(b)), used(0), cap(c) {}
  template <class T>
  T* take(int64_t n) {
    uint64_t bytes = static_cast<uint64_t>(align_up(n * static_cast<int64_t>(sizeof(T)), 256));
    T* p = reinterpret_cast<T*>(base ? base + used : nullptr);
    used += bytes;
    return p;
  }
  bool ok() const { return used <= cap; }
};

// Launch-level wrappers used by the layer templates (no argument checks).
mt_status gemm_launch(const mt_bf16* A, int64_t lda, bool a_mn, const mt_bf16* B, int64_t ldb, bool b_mn,
                      void* C, int64_t ldc, bool c_f32, bool accumulate, int64_t M, int64_t N, int64_t K,
                      const mt_bf16* bias, const mt_bf16* residual, int64_t ldr, cudaStream_t st);

// dm = A B (M x F) with the SwiGLU backward in the epilogue: gu holds [g | u]
// (row stride ld_gu) on entry and [dg | du] on return; dm itself is not stored.
mt_status gemm_swiglu_bwd_launch(const mt_bf16* A, int64_t lda, bool a_mn, const mt_bf16* B, int64_t ldb, bool b_mn,
                                 mt_bf16* gu, int64_t ld_gu, int64_t M, int64_t F, int64_t K, cudaStream_t st);

// C = A B^T (both K-major, bf16 C) with bias and rotate-half RoPE applied to the
// fp32 accumulators of the first rope_cols columns (heads of head_dim) at
// position row % T; rope_tab holds (cos, sin) pairs, [T][head_dim / 2] (rope_table_launch).
mt_status gemm_rope_launch(const mt_bf16* A, int64_t lda, const mt_bf16* B, int64_t ldb, mt_bf16* C, int64_t ldc,
                           int64_t M, int64_t N, int64_t K, const mt_bf16* bias, const float* rope_tab, int rope_cols,
                           int head_dim, int T, cudaStream_t st);

// C = A B^T (bf16 C) that also writes, per row and head of head_dim columns, the
// dot product of the stored C with dot_with into dot_out[seq][head][t] (fp32).
mt_status gemm_dot_launch(const mt_bf16* A, int64_t lda, bool a_mn, const mt_bf16* B, int64_t ldb, bool b_mn,
                          mt_bf16* C, int64_t ldc, int64_t M, int64_t N, int64_t K, const mt_bf16* dot_with,
                          int64_t ld_dot, float* dot_out, int head_dim, int T, cudaStream_t st);

// (cos, sin) of angle t * theta^(-2i/d) for t < T, i < d/2 as fp32 pairs, formed in fp64.
mt_status rope_table_launch(float* tab, int T, int d, float theta, cudaStream_t st);

// GEMM launch observer (engine statistics): called around each GEMM launch.
struct GemmTimer {
  virtual void before(cudaStream_t st) = 0;
  virtual void after(cudaStream_t st, double flops) = 0;
  virtual ~GemmTimer() {}
};
void set_gemm_timer(GemmTimer* t);  // thread-local
// Running count of executed FLOPs on this thread (engine statistics).
void add_exec_flops(double f);
double exec_flops_counter();

}  // namespace mt
