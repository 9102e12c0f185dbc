// Bandwidth-bound kernels of the decoder layer: RMSNorm forward/backward,
// rotate-half RoPE, SwiGLU forward/backward and fixed-order column sums
// (bias and norm-gain gradients). Each is a single pass over its operands in
// HBM with 16-byte vector accesses; reductions over tokens use per-block
// partial rows reduced in a fixed order, so results are bitwise repeatable.
#include <mutex>

#include "mt_internal.h"

namespace mt {
namespace {

constexpr int COLSUM_ROWS = 64;  // rows per partial-sum block

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return u;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp per row. H is a multiple of 8.
__global__ void rmsnorm_fwd_kernel(const uint4* __restrict__ x, const uint4* __restrict__ g, uint4* __restrict__ y,
                                   float* __restrict__ rstd, int64_t rows, int H, float eps) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int nc = H / 8;
  const uint4* xr = x + row * nc;
  float ss = 0.f;
  for (int c = lane; c < nc; c += 32) {
    float f[8];
    unpack8(xr[c], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss += f[i] * f[i];
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / static_cast<float>(H) + eps);
  if (lane == 0) rstd[row] = r;
  uint4* yr = y + row * nc;
  for (int c = lane; c < nc; c += 32) {
    float f[8], w[8];
    unpack8(xr[c], f);
    unpack8(__ldg(g + c), w);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = f[i] * r * w[i];
    yr[c] = pack8(f);
  }
}

// dx = rstd*(g*dy - xh*mean(xh*g*dy)) + dres; one warp per row.
__global__ void rmsnorm_bwd_kernel(const uint4* dy, const uint4* __restrict__ x, const uint4* __restrict__ g,
                                   const float* __restrict__ rstd, const uint4* dres, uint4* dx, int64_t rows,
                                   int H) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int nc = H / 8;
  const float r = rstd[row];
  const uint4* dyr = dy + row * nc;
  const uint4* xr = x + row * nc;
  float dot = 0.f;
  for (int c = lane; c < nc; c += 32) {
    float a[8], b[8], w[8];
    unpack8(dyr[c], a);
    unpack8(xr[c], b);
    unpack8(__ldg(g + c), w);
#pragma unroll
    for (int i = 0; i < 8; ++i) dot += (b[i] * r) * w[i] * a[i];
  }
  dot = warp_sum(dot) / static_cast<float>(H);
  uint4* dxr = dx + row * nc;
  const uint4* drr = dres ? dres + row * nc : nullptr;
  for (int c = lane; c < nc; c += 32) {
    float a[8], b[8], w[8], o[8];
    unpack8(dyr[c], a);
    unpack8(xr[c], b);
    unpack8(__ldg(g + c), w);
    if (drr) {
      unpack8(drr[c], o);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] += r * (w[i] * a[i] - (b[i] * r) * dot);
    dxr[c] = pack8(o);
  }
}

// partial[rb][j] = sum over rows r of block rb of X[r, j] (* Y[r, j] * rstd[r]).
// Each thread owns two adjacent columns; rows are visited in increasing order.
template <bool PROD>
__global__ void colpartial_kernel(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ Y,
                                  const float* __restrict__ rstd, int64_t rows, int64_t cols, int64_t ld,
                                  float* __restrict__ partial) {
  const int64_t j = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
  const int64_t rb = blockIdx.y;
  if (j >= cols) return;
  const int64_t r0 = rb * COLSUM_ROWS;
  const int64_t r1 = min(rows, r0 + COLSUM_ROWS);
  float a0 = 0.f, a1 = 0.f;
  const bool pair = j + 1 < cols;
  for (int64_t r = r0; r < r1; ++r) {
    const __nv_bfloat16* xp = X + r * ld + j;
    float x0, x1 = 0.f;
    if (pair) {
      float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(xp));
      x0 = t.x;
      x1 = t.y;
    } else {
      x0 = __bfloat162float(xp[0]);
    }
    if (PROD) {
      const float s = rstd[r];
      const __nv_bfloat16* yp = Y + r * ld + j;
      float y0, y1 = 0.f;
      if (pair) {
        float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(yp));
        y0 = t.x;
        y1 = t.y;
      } else {
        y0 = __bfloat162float(yp[0]);
      }
      x0 = x0 * (y0 * s);
      x1 = x1 * (y1 * s);
    }
    a0 += x0;
    a1 += x1;
  }
  partial[rb * cols + j] = a0;
  if (pair) partial[rb * cols + j + 1] = a1;
}

__global__ void colreduce_kernel(const float* __restrict__ partial, int64_t nrb, int64_t cols, float* __restrict__ out) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= cols) return;
  float a = 0.f;
  for (int64_t rb = 0; rb < nrb; ++rb) a += partial[rb * cols + j];
  out[j] = a;
}

// Rotate-half RoPE. One thread per (token, i < d/2); loops over the heads.
__global__ void rope_kernel(__nv_bfloat16* x, int64_t ld, int64_t rows, int T, int n_heads, int d, double theta,
                            int inverse) {
  const int half = d / 2;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = gid / half;
  const int i = static_cast<int>(gid % half);
  if (row >= rows) return;
  const int t = static_cast<int>(row % T);
  const double omega = pow(theta, -2.0 * static_cast<double>(i) / static_cast<double>(d));
  double sd, cd;
  sincos(static_cast<double>(t) * omega, &sd, &cd);
  const float c = static_cast<float>(cd);
  const float s = inverse ? -static_cast<float>(sd) : static_cast<float>(sd);
  __nv_bfloat16* p = x + row * ld + i;
  for (int h = 0; h < n_heads; ++h, p += d) {
    const float a = __bfloat162float(p[0]);
    const float b = __bfloat162float(p[half]);
    p[0] = __float2bfloat16_rn(a * c - b * s);
    p[half] = __float2bfloat16_rn(b * c + a * s);
  }
}

// (cos, sin) of t * theta^(-2i/d) for every position t < T and pair i < d/2, formed
// in fp64 like rope_kernel's and rounded to fp32: the table the RoPE epilogue of
// the QKV projection reads.
__global__ void rope_table_kernel(float2* tab, int64_t n, int half, int d, double theta) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= n) return;
  const int64_t t = gid / half;
  const int i = static_cast<int>(gid % half);
  const double omega = pow(theta, -2.0 * static_cast<double>(i) / static_cast<double>(d));
  double sd, cd;
  sincos(static_cast<double>(t) * omega, &sd, &cd);
  tab[gid] = make_float2(static_cast<float>(cd), static_cast<float>(sd));
}

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }

__global__ void swiglu_fwd_kernel(const uint4* __restrict__ gu, uint4* __restrict__ m, int64_t rows, int F) {
  const int fc = F / 8;
  const int64_t n = rows * fc;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = idx / fc;
    const int c = static_cast<int>(idx % fc);
    float g[8], u[8];
    unpack8(gu[r * 2 * fc + c], g);
    unpack8(gu[r * 2 * fc + fc + c], u);
#pragma unroll
    for (int i = 0; i < 8; ++i) g[i] = g[i] * sigmoidf_(g[i]) * u[i];
    m[idx] = pack8(g);
  }
}

__global__ void swiglu_bwd_kernel(const uint4* __restrict__ dm, const uint4* __restrict__ gu, uint4* __restrict__ dgu,
                                  int64_t rows, int F) {
  const int fc = F / 8;
  const int64_t n = rows * fc;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = idx / fc;
    const int c = static_cast<int>(idx % fc);
    float d[8], g[8], u[8], dg[8], du[8];
    unpack8(dm[idx], d);
    unpack8(gu[r * 2 * fc + c], g);
    unpack8(gu[r * 2 * fc + fc + c], u);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float sg = sigmoidf_(g[i]);
      dg[i] = d[i] * u[i] * sg * (1.0f + g[i] * (1.0f - sg));
      du[i] = d[i] * g[i] * sg;
    }
    dgu[r * 2 * fc + c] = pack8(dg);
    dgu[r * 2 * fc + fc + c] = pack8(du);
  }
}

int ew_grid(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (b > cap) b = cap;
  if (b < 1) b = 1;
  return static_cast<int>(b);
}

}  // namespace

// ---------------------------------------------------------------- launchers
mt_status rmsnorm_fwd_launch(const mt_bf16* x, const mt_bf16* g, mt_bf16* y, float* rstd, int64_t rows, int H,
                             float eps, cudaStream_t st) {
  if (rows == 0) return MT_OK;
  const int wpb = 8;
  const int64_t blocks = (rows + wpb - 1) / wpb;
  rmsnorm_fwd_kernel<<<static_cast<unsigned>(blocks), wpb * 32, 0, st>>>(
      reinterpret_cast<const uint4*>(x), reinterpret_cast<const uint4*>(g), reinterpret_cast<uint4*>(y), rstd, rows, H,
      eps);
  return launch_check("rmsnorm_fwd_kernel");
}

uint64_t colsum_ws_bytes(int64_t rows, int64_t cols) {
  const int64_t nrb = (rows + COLSUM_ROWS - 1) / COLSUM_ROWS;
  return static_cast<uint64_t>(align_up(nrb * cols * 4, 256));
}

mt_status colsum_launch(const mt_bf16* X, const mt_bf16* Y, const float* rstd, int64_t rows, int64_t cols, int64_t ld,
                        float* out, void* ws, cudaStream_t st) {
  const int64_t nrb = (rows + COLSUM_ROWS - 1) / COLSUM_ROWS;
  float* partial = static_cast<float*>(ws);
  if (rows > 0) {
    const int threads = 256;
    dim3 grid(static_cast<unsigned>((cols + 2 * threads - 1) / (2 * threads)), static_cast<unsigned>(nrb));
    if (Y)
      colpartial_kernel<true><<<grid, threads, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(X),
                                                        reinterpret_cast<const __nv_bfloat16*>(Y), rstd, rows, cols, ld,
                                                        partial);
    else
      colpartial_kernel<false><<<grid, threads, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(X), nullptr, nullptr,
                                                         rows, cols, ld, partial);
    MT_TRY(launch_check("colpartial_kernel"));
  }
  colreduce_kernel<<<static_cast<unsigned>((cols + 255) / 256), 256, 0, st>>>(partial, nrb, cols, out);
  return launch_check("colreduce_kernel");
}

mt_status rmsnorm_bwd_launch(const mt_bf16* dy, const mt_bf16* x, const mt_bf16* g, const float* rstd,
                             const mt_bf16* dres, mt_bf16* dx, float* dg, int64_t rows, int H, void* ws,
                             cudaStream_t st) {
  // dg first: it reads dy, which dx may overwrite.
  MT_TRY(colsum_launch(dy, x, rstd, rows, H, H, dg, ws, st));
  if (rows == 0) return MT_OK;
  const int wpb = 8;
  const int64_t blocks = (rows + wpb - 1) / wpb;
  rmsnorm_bwd_kernel<<<static_cast<unsigned>(blocks), wpb * 32, 0, st>>>(
      reinterpret_cast<const uint4*>(dy), reinterpret_cast<const uint4*>(x), reinterpret_cast<const uint4*>(g), rstd,
      reinterpret_cast<const uint4*>(dres), reinterpret_cast<uint4*>(dx), rows, H);
  return launch_check("rmsnorm_bwd_kernel");
}

mt_status rope_launch(mt_bf16* x, int64_t ld, int B, int T, int n_heads, int d, float theta, bool inverse,
                      cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(B) * T;
  const int64_t n = rows * (d / 2);
  if (n == 0) return MT_OK;
  const int threads = 256;
  rope_kernel<<<static_cast<unsigned>((n + threads - 1) / threads), threads, 0, st>>>(
      reinterpret_cast<__nv_bfloat16*>(x), ld, rows, T, n_heads, d, static_cast<double>(theta), inverse ? 1 : 0);
  return launch_check("rope_kernel");
}

mt_status rope_table_launch(float* tab, int T, int d, float theta, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(T) * (d / 2);
  if (n == 0) return MT_OK;
  const int threads = 256;
  rope_table_kernel<<<static_cast<unsigned>((n + threads - 1) / threads), threads, 0, st>>>(
      reinterpret_cast<float2*>(tab), n, d / 2, d, static_cast<double>(theta));
  return launch_check("rope_table_kernel");
}

mt_status swiglu_fwd_launch(const mt_bf16* gu, mt_bf16* m, int64_t rows, int F, cudaStream_t st) {
  const int64_t n = rows * (F / 8);
  if (n == 0) return MT_OK;
  swiglu_fwd_kernel<<<ew_grid(n, 256), 256, 0, st>>>(reinterpret_cast<const uint4*>(gu), reinterpret_cast<uint4*>(m),
                                                      rows, F);
  return launch_check("swiglu_fwd_kernel");
}

mt_status swiglu_bwd_launch(const mt_bf16* dm, const mt_bf16* gu, mt_bf16* dgu, int64_t rows, int F,
                            cudaStream_t st) {
  const int64_t n = rows * (F / 8);
  if (n == 0) return MT_OK;
  swiglu_bwd_kernel<<<ew_grid(n, 256), 256, 0, st>>>(reinterpret_cast<const uint4*>(dm),
                                                      reinterpret_cast<const uint4*>(gu), reinterpret_cast<uint4*>(dgu),
                                                      rows, F);
  return launch_check("swiglu_bwd_kernel");
}

}  // namespace mt

using namespace mt;

extern "C" {

mt_status mt_rmsnorm_fwd(const mt_bf16* x, const mt_bf16* g, mt_bf16* y, float* rstd, int64_t rows, int32_t H,
                         float eps, void* stream) {
  if (!x || !g || !y || !rstd) return fail(MT_ERR_INVALID_ARG, "rmsnorm_fwd: NULL pointer");
  if (rows < 0 || H <= 0 || H % 8) return fail(MT_ERR_INVALID_ARG, "rmsnorm_fwd: need rows >= 0, H > 0, H %% 8 == 0");
  if (!aligned16(x) || !aligned16(g) || !aligned16(y)) return fail(MT_ERR_ALIGNMENT, "rmsnorm_fwd: 16-byte alignment");
  return rmsnorm_fwd_launch(x, g, y, rstd, rows, H, eps, as_stream(stream));
}

uint64_t mt_rmsnorm_bwd_workspace_bytes(int64_t rows, int32_t H) { return colsum_ws_bytes(rows, H); }

mt_status mt_rmsnorm_bwd(const mt_bf16* dy, const mt_bf16* x, const mt_bf16* g, const float* rstd, const mt_bf16* dres,
                         mt_bf16* dx, float* dg, int64_t rows, int32_t H, void* ws, uint64_t ws_bytes, void* stream) {
  if (!dy || !x || !g || !rstd || !dx || !dg || !ws) return fail(MT_ERR_INVALID_ARG, "rmsnorm_bwd: NULL pointer");
  if (rows < 0 || H <= 0 || H % 8) return fail(MT_ERR_INVALID_ARG, "rmsnorm_bwd: need rows >= 0, H > 0, H %% 8 == 0");
  if (ws_bytes < colsum_ws_bytes(rows, H)) return fail(MT_ERR_WORKSPACE, "rmsnorm_bwd: workspace too small");
  if (!aligned16(dy) || !aligned16(x) || !aligned16(g) || !aligned16(dx) || (dres && !aligned16(dres)))
    return fail(MT_ERR_ALIGNMENT, "rmsnorm_bwd: 16-byte alignment");
  return rmsnorm_bwd_launch(dy, x, g, rstd, dres, dx, dg, rows, H, ws, as_stream(stream));
}

mt_status mt_rope(mt_bf16* x, int64_t ld, int32_t B, int32_t T, int32_t n_heads, int32_t head_dim, float theta,
                  int32_t inverse, void* stream) {
  if (!x) return fail(MT_ERR_INVALID_ARG, "rope: NULL pointer");
  if (B < 0 || T <= 0 || n_heads < 0 || head_dim <= 0 || head_dim % 2 || !(theta > 0.f))
    return fail(MT_ERR_INVALID_ARG, "rope: bad sizes");
  if (ld < static_cast<int64_t>(n_heads) * head_dim) return fail(MT_ERR_INVALID_ARG, "rope: ld too small");
  return rope_launch(x, ld, B, T, n_heads, head_dim, theta, inverse != 0, as_stream(stream));
}

mt_status mt_swiglu_fwd(const mt_bf16* gu, mt_bf16* m, int64_t rows, int32_t F, void* stream) {
  if (!gu || !m) return fail(MT_ERR_INVALID_ARG, "swiglu_fwd: NULL pointer");
  if (rows < 0 || F <= 0 || F % 8) return fail(MT_ERR_INVALID_ARG, "swiglu_fwd: need F %% 8 == 0");
  if (!aligned16(gu) || !aligned16(m)) return fail(MT_ERR_ALIGNMENT, "swiglu_fwd: 16-byte alignment");
  return swiglu_fwd_launch(gu, m, rows, F, as_stream(stream));
}

mt_status mt_swiglu_bwd(const mt_bf16* dm, const mt_bf16* gu, mt_bf16* dgu, int64_t rows, int32_t F, void* stream) {
  if (!dm || !gu || !dgu) return fail(MT_ERR_INVALID_ARG, "swiglu_bwd: NULL pointer");
  if (rows < 0 || F <= 0 || F % 8) return fail(MT_ERR_INVALID_ARG, "swiglu_bwd: need F %% 8 == 0");
  if (!aligned16(dm) || !aligned16(gu) || !aligned16(dgu)) return fail(MT_ERR_ALIGNMENT, "swiglu_bwd: 16-byte alignment");
  return swiglu_bwd_launch(dm, gu, dgu, rows, F, as_stream(stream));
}

uint64_t mt_colsum_workspace_bytes(int64_t rows, int64_t cols) { return colsum_ws_bytes(rows, cols); }

mt_status mt_colsum(const mt_bf16* X, int64_t rows, int64_t cols, int64_t ld, float* out, void* ws, uint64_t ws_bytes,
                    void* stream) {
  if (!X || !out || !ws) return fail(MT_ERR_INVALID_ARG, "colsum: NULL pointer");
  if (rows < 0 || cols <= 0 || ld < cols) return fail(MT_ERR_INVALID_ARG, "colsum: bad sizes");
  if (ld % 2 || cols % 2 || (reinterpret_cast<uintptr_t>(X) & 3u))
    return fail(MT_ERR_ALIGNMENT, "colsum: cols and ld must be even and X 4-byte aligned");
  if (ws_bytes < colsum_ws_bytes(rows, cols)) return fail(MT_ERR_WORKSPACE, "colsum: workspace too small");
  return colsum_launch(X, nullptr, nullptr, rows, cols, ld, out, ws, as_stream(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// mt_rmsnorm_bwd_noalloc: the RMSNorm backward for callers that cannot give a
// workspace. Its partial-sum scratch is this file's own device array.
namespace {

constexpr int64_t NOALLOC_SCRATCH_FLOATS = int64_t(1) << 21;  // 8 MiB per device
static __device__ __align__(256) float g_rmsnorm_scratch[NOALLOC_SCRATCH_FLOATS];

// Device address of g_rmsnorm_scratch, looked up once per device with that
// device current (in host code the symbol is only a host-side stand-in).
mt_status noalloc_scratch(float** out) {
  static std::mutex mu;
  static float* addr[64] = {nullptr};
  int dev = 0;
  MT_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MT_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    MT_CUDA(cudaGetSymbolAddress(&p, g_rmsnorm_scratch));
    addr[dev] = static_cast<float*>(p);
  }
  *out = addr[dev];
  return MT_OK;
}

}  // namespace

extern "C" mt_status mt_rmsnorm_bwd_noalloc(const mt_bf16* dy, const mt_bf16* x, const mt_bf16* g, const float* rstd,
                                            const mt_bf16* dres, mt_bf16* dx, float* dg, int64_t rows, int32_t H,
                                            void* stream) {
  if (!dy || !x || !g || !rstd || !dx || !dg) return fail(MT_ERR_INVALID_ARG, "rmsnorm_bwd_noalloc: NULL pointer");
  if (rows < 0 || H <= 0 || H % 8)
    return fail(MT_ERR_INVALID_ARG, "rmsnorm_bwd_noalloc: need rows >= 0, H > 0, H %% 8 == 0");
  if (!aligned16(dy) || !aligned16(x) || !aligned16(g) || !aligned16(dx) || (dres && !aligned16(dres)))
    return fail(MT_ERR_ALIGNMENT, "rmsnorm_bwd_noalloc: 16-byte alignment");
  const uint64_t need = colsum_ws_bytes(rows, H);
  if (need > static_cast<uint64_t>(NOALLOC_SCRATCH_FLOATS) * 4)
    return fail(MT_ERR_WORKSPACE,
                "rmsnorm_bwd_noalloc: %lld rows x %d columns need %llu bytes of scratch, above its fixed %lld bytes "
                "(ceil(rows/64) * H must be <= %lld); use mt_rmsnorm_bwd with a workspace",
                (long long)rows, H, (unsigned long long)need, (long long)(NOALLOC_SCRATCH_FLOATS * 4),
                (long long)NOALLOC_SCRATCH_FLOATS);
  float* scratch = nullptr;
  MT_TRY(noalloc_scratch(&scratch));
  return rmsnorm_bwd_launch(dy, x, g, rstd, dres, dx, dg, rows, H, scratch, as_stream(stream));
}
