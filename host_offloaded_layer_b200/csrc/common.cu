// Errors, layer geometry and record layout, and the host-side streaming
// schedule (weight-use order and slot plan).
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "mt_internal.h"

namespace mt {

static thread_local char g_err[1024] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

mt_status fail(mt_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

__device__ int32_t g_device_error = 0;

int32_t* device_error_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  return static_cast<int32_t*>(p);
}

int num_sms() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

static thread_local GemmTimer* t_timer = nullptr;
static thread_local double t_flops = 0.0;
void set_gemm_timer(GemmTimer* t) { t_timer = t; }
GemmTimer* current_gemm_timer() { return t_timer; }
void add_exec_flops(double f) { t_flops += f; }
static thread_local uint64_t t_launches = 0;
void count_launch() { ++t_launches; }
uint64_t launch_counter() { return t_launches; }
double exec_flops_counter() { return t_flops; }

mt_status make_geom(const mt_layer_cfg* cfg, Geom* g) {
  if (!cfg) return fail(MT_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->hidden <= 0 || cfg->n_q_heads <= 0 || cfg->n_kv_heads <= 0 || cfg->head_dim <= 0 || cfg->ffn <= 0)
    return fail(MT_ERR_INVALID_ARG, "cfg sizes must be positive");
  if (cfg->n_q_heads % cfg->n_kv_heads != 0)
    return fail(MT_ERR_INVALID_ARG, "n_kv_heads (%d) must divide n_q_heads (%d)", cfg->n_kv_heads,
                cfg->n_q_heads);
  if (cfg->hidden % 8 != 0 || cfg->ffn % 8 != 0)
    return fail(MT_ERR_INVALID_ARG, "hidden and ffn must be multiples of 8 (16-byte rows)");
  if (!(cfg->rms_eps >= 0.0f) || !(cfg->rope_theta > 0.0f))
    return fail(MT_ERR_INVALID_ARG, "rms_eps must be >= 0 and rope_theta > 0");
  g->H = cfg->hidden;
  g->nq = cfg->n_q_heads;
  g->nkv = cfg->n_kv_heads;
  g->d = cfg->head_dim;
  g->F = cfg->ffn;
  g->Nq = g->nq * g->d;
  g->Nkv = g->nkv * g->d;
  g->Nqkv = g->Nq + 2 * g->Nkv;
  g->bias = cfg->qkv_bias != 0;
  g->eps = cfg->rms_eps;
  g->theta = cfg->rope_theta;
  mt_param_offsets& o = g->off;
  const int64_t A = 128;
  int64_t p = 0;
  o.g1 = p;
  p = align_up(p + g->H, A);
  o.wq = p;
  o.wk = o.wq + g->Nq * g->H;
  o.wv = o.wk + g->Nkv * g->H;
  p = align_up(o.wv + g->Nkv * g->H, A);
  o.bq = p;
  o.bk = o.bq + g->Nq;
  o.bv = o.bk + g->Nkv;
  if (g->bias) p = align_up(o.bv + g->Nkv, A);
  o.wo = p;
  p = align_up(p + g->H * g->Nq, A);
  o.g2 = p;
  p = align_up(p + g->H, A);
  o.wg = p;
  o.wu = o.wg + g->F * g->H;
  p = align_up(o.wu + g->F * g->H, A);
  o.wd = p;
  p = align_up(p + g->H * g->F, A);
  o.record_elems = p;
  o.param_count = 2 * g->H + g->Nqkv * g->H + (g->bias ? g->Nqkv : 0) + g->H * g->Nq + 3 * g->F * g->H;
  return MT_OK;
}

// ------------------------------------------------------------- schedule
// Uses in compute order: forward 0..L-1; then for each segment s from last to
// first (layers [sK, min(sK+K, L))): re-forward of all but its last layer,
// then recompute+backward from its last layer down to its first. The last
// segment needs no re-forward: the forward writes its inner activations
// straight into the segment buffers, which the backward reads.
struct Use {
  int32_t layer, kind;
};

std::vector<Use> build_uses(int L, int K) {
  std::vector<Use> u;
  for (int l = 0; l < L; ++l) u.push_back({l, 0});
  int S = (L + K - 1) / K;
  for (int s = S - 1; s >= 0; --s) {
    int a = s * K, b = std::min(L, a + K);
    if (s != S - 1)
      for (int l = a; l < b - 1; ++l) u.push_back({l, 1});
    for (int l = b - 1; l >= a; --l) u.push_back({l, 2});
  }
  return u;
}

// Furthest-next-use slot plan over a static use list.
void plan_slots(const std::vector<Use>& u, int R, std::vector<int>& slot, std::vector<int>& load) {
  const int n = static_cast<int>(u.size());
  slot.assign(n, -1);
  load.assign(n, 0);
  std::vector<int> holds(R, -1);  // layer held by each slot
  for (int i = 0; i < n; ++i) {
    int l = u[i].layer, found = -1;
    for (int r = 0; r < R; ++r)
      if (holds[r] == l) found = r;
    if (found < 0) {
      // empty slot first, else the slot whose layer is next used furthest ahead
      int best = -1;
      long best_next = -1;
      for (int r = 0; r < R; ++r) {
        if (holds[r] < 0) {
          best = r;
          break;
        }
        long nxt = 1L << 40;
        for (int j = i + 1; j < n; ++j)
          if (u[j].layer == holds[r]) {
            nxt = j;
            break;
          }
        // never evict the slot used by the immediately preceding use if another works
        if (i > 0 && slot[i - 1] == r && R > 1) nxt = -2;
        if (nxt > best_next) {
          best_next = nxt;
          best = r;
        }
      }
      found = best;
      holds[found] = l;
      load[i] = 1;
    }
    slot[i] = found;
  }
}

}  // namespace mt

using namespace mt;

extern "C" {

const char* mt_last_error(void) { return g_err; }

mt_status mt_device_error(int32_t* out_code, int32_t clear) {
  if (!out_code) return fail(MT_ERR_INVALID_ARG, "out_code is NULL");
  int32_t v = 0;
  MT_CUDA(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)));
  *out_code = v;
  if (clear) {
    int32_t z = 0;
    MT_CUDA(cudaMemcpyToSymbol(g_device_error, &z, sizeof(z)));
  }
  return MT_OK;
}

uint64_t mt_layer_param_count(const mt_layer_cfg* cfg) {
  Geom g;
  if (make_geom(cfg, &g) != MT_OK) return 0;
  return g.off.param_count;
}

mt_status mt_layer_param_offsets(const mt_layer_cfg* cfg, mt_param_offsets* out) {
  if (!out) return fail(MT_ERR_INVALID_ARG, "out is NULL");
  Geom g;
  MT_TRY(make_geom(cfg, &g));
  *out = g.off;
  return MT_OK;
}

int32_t mt_schedule_len(int32_t n_layers, int32_t K) {
  if (n_layers <= 0 || K <= 0) return 0;
  return static_cast<int32_t>(build_uses(n_layers, K).size());
}

mt_status mt_schedule(int32_t n_layers, int32_t K, int32_t n_slots, int32_t* layer, int32_t* kind,
                      int32_t* slot, int32_t* load) {
  if (n_layers <= 0 || K <= 0 || n_slots <= 0) return fail(MT_ERR_INVALID_ARG, "n_layers, K, n_slots must be > 0");
  if (!layer || !kind || !slot || !load) return fail(MT_ERR_INVALID_ARG, "output arrays must not be NULL");
  auto u = build_uses(n_layers, K);
  std::vector<int> s, ld;
  plan_slots(u, n_slots, s, ld);
  for (size_t i = 0; i < u.size(); ++i) {
    layer[i] = u[i].layer;
    kind[i] = u[i].kind;
    slot[i] = s[i];
    load[i] = ld[i];
  }
  return MT_OK;
}

}  // extern "C"
