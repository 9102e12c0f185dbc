// Host store and streaming engine.
//
// The MegaTrain pages describe a memory-centric executor: parameters live in
// host memory (abstract; Fig. 2; blog design point 1) in a flat layout that
// keeps host memory linear in the parameter count (blog, Performance), and
// each training step streams a layer's weights in and its gradients out
// (blog design point 2) through a pipelined, double-buffered engine on three
// CUDA streams - weight prefetch (W), compute (F/R/B) and gradient offload
// (G) - so that transfers stay off the critical path (abstract; Fig. 3).
// Activations are checkpointed every K layers and recomputed (blog design
// point 3), and gradients pass through a pool of recycled pinned slabs
// (Table 4, "Gradient Slab Pool").
//
// Here one host thread enqueues every copy and kernel of a step ahead of the
// GPU, ordered only by CUDA events:
//   prefetch: wait done[prev user of slot] -> H2D record -> record ready
//   compute : wait ready -> layer template -> record done (and g_ready)
//   offload : wait g_ready -> D2H into a pooled pinned slab -> record d2h_done
// A second host thread polls d2h_done (bounded), hands each slab to the sink
// in backward order and returns it to the pool. Every host wait is bounded by
// the engine's timeout; nothing waits on the device.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdlib>
#include <condition_variable>
#include <cstring>
#include <deque>
#include <functional>
#include <mutex>
#include <thread>
#include <vector>

#include "mt_internal.h"

namespace mt {
struct Use {
  int32_t layer, kind;
};
std::vector<Use> build_uses(int L, int K);
void plan_slots(const std::vector<Use>& u, int R, std::vector<int>& slot, std::vector<int>& load);
mt_status layer_fwd_keep(const mt_layer_cfg* cfg, const mt_bf16* w_dev, const mt_bf16* x, mt_bf16* y, int32_t B,
                         int32_t T, int32_t mlp_chunk, void* ws, uint64_t ws_bytes, void* stream, bool keep,
                         cudaEvent_t mlp_weights);
mt_status layer_recompute_bwd_ev(const mt_layer_cfg* cfg, const mt_bf16* w_dev, const mt_bf16* x, const mt_bf16* dy,
                                 mt_bf16* dx, float* dw_dev, int32_t B, int32_t T, int32_t mlp_chunk, void* ws_int,
                                 uint64_t int_bytes, void* ws_scr, uint64_t scr_bytes, void* stream,
                                 cudaEvent_t mlp_done, bool reuse_fwd, cudaEvent_t wd_done);
mt_status layer_ws_sizes(const mt_layer_cfg* cfg, int32_t B, int32_t T, int32_t mlp_chunk, uint64_t* internals,
                         uint64_t* scratch);
}  // namespace mt

using namespace mt;

// ======================================================================= host store
struct mt_host_store {
  Geom G;
  int L;
  float* master = nullptr;
  uint16_t* bf = nullptr;
};

static void parallel_for(int64_t n, int threads, const std::function<void(int64_t, int64_t)>& fn) {
  if (threads <= 1 || n < (1 << 20)) {
    fn(0, n);
    return;
  }
  std::vector<std::thread> th;
  const int64_t per = (n + threads - 1) / threads;
  for (int t = 0; t < threads; ++t) {
    const int64_t a = t * per, b = std::min(n, a + per);
    if (a >= b) break;
    th.emplace_back([&fn, a, b] { fn(a, b); });
  }
  for (auto& x : th) x.join();
}

static int default_threads() {
  unsigned n = std::thread::hardware_concurrency();
  return n == 0 ? 4 : static_cast<int>(std::min(n, 32u));
}

extern "C" {

mt_status mt_host_store_create(const mt_layer_cfg* cfg, int32_t n_layers, int32_t keep_fp32_master,
                               mt_host_store** out) {
  if (!out) return fail(MT_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  Geom G;
  MT_TRY(make_geom(cfg, &G));
  if (n_layers <= 0) return fail(MT_ERR_INVALID_ARG, "n_layers must be positive");
  auto* s = new mt_host_store();
  s->G = G;
  s->L = n_layers;
  const uint64_t n = G.off.record_elems * static_cast<uint64_t>(n_layers);
  if (cudaHostAlloc(reinterpret_cast<void**>(&s->bf), n * 2, cudaHostAllocPortable) != cudaSuccess) {
    cudaGetLastError();
    delete s;
    return fail(MT_ERR_OOM, "pinned allocation of %llu bytes (bf16 store) failed", (unsigned long long)(n * 2));
  }
  if (keep_fp32_master) {
    if (cudaHostAlloc(reinterpret_cast<void**>(&s->master), n * 4, cudaHostAllocPortable) != cudaSuccess) {
      cudaGetLastError();
      cudaFreeHost(s->bf);
      delete s;
      return fail(MT_ERR_OOM, "pinned allocation of %llu bytes (fp32 master) failed", (unsigned long long)(n * 4));
    }
  }
  parallel_for(static_cast<int64_t>(n), default_threads(), [s](int64_t a, int64_t b) {
    std::memset(s->bf + a, 0, (b - a) * 2);
    if (s->master) std::memset(s->master + a, 0, (b - a) * 4);
  });
  *out = s;
  return MT_OK;
}

float* mt_host_store_master(mt_host_store* s, int32_t layer) {
  if (!s || !s->master || layer < 0 || layer >= s->L) return nullptr;
  return s->master + static_cast<uint64_t>(layer) * s->G.off.record_elems;
}

mt_bf16* mt_host_store_bf16(mt_host_store* s, int32_t layer) {
  if (!s || layer < 0 || layer >= s->L) return nullptr;
  return s->bf + static_cast<uint64_t>(layer) * s->G.off.record_elems;
}

mt_status mt_host_store_refresh_bf16(mt_host_store* s, int32_t n_threads) {
  if (!s) return fail(MT_ERR_INVALID_ARG, "store is NULL");
  if (!s->master) return fail(MT_ERR_INVALID_ARG, "store has no fp32 master copy");
  const int64_t n = static_cast<int64_t>(s->G.off.record_elems) * s->L;
  parallel_for(n, n_threads > 0 ? n_threads : default_threads(), [s](int64_t a, int64_t b) {
    for (int64_t i = a; i < b; ++i) {
      uint32_t u;
      std::memcpy(&u, s->master + i, 4);
      if ((u & 0x7FFFFFFFu) > 0x7F800000u) {
        s->bf[i] = static_cast<uint16_t>((u >> 16) | 0x40u);  // quiet NaN
      } else {
        s->bf[i] = static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
      }
    }
  });
  return MT_OK;
}

void mt_host_store_destroy(mt_host_store* s) {
  if (!s) return;
  if (s->bf) cudaFreeHost(s->bf);
  if (s->master) cudaFreeHost(s->master);
  delete s;
}

}  // extern "C"

// ======================================================================= timeline summary
namespace {

using Span = std::pair<double, double>;

// Sorted, merged union of intervals.
std::vector<Span> merged(std::vector<Span> v) {
  std::sort(v.begin(), v.end());
  std::vector<Span> out;
  for (const Span& x : v) {
    if (!out.empty() && x.first <= out.back().second)
      out.back().second = std::max(out.back().second, x.second);
    else
      out.push_back(x);
  }
  return out;
}

// Whether instant t lies inside the merged union u.
bool covers(const std::vector<Span>& u, double t) {
  auto it = std::upper_bound(u.begin(), u.end(), Span(t, 1e300));
  return it != u.begin() && t < std::prev(it)->second;
}

}  // namespace

extern "C" mt_status mt_trace_summarize(const mt_trace_rec* recs, int32_t n, mt_trace_summary* out) {
  if (!out || n < 0 || (n > 0 && !recs)) return fail(MT_ERR_INVALID_ARG, "trace_summarize: bad argument");
  std::memset(out, 0, sizeof(*out));
  std::vector<Span> comp, up, off;
  std::vector<double> cuts = {0.0};
  for (int i = 0; i < n; ++i) {
    const mt_trace_rec& r = recs[i];
    if (r.kind < 0 || r.kind > 4) return fail(MT_ERR_INVALID_ARG, "trace_summarize: unknown kind %d", r.kind);
    if (!(r.end_ms >= r.begin_ms)) return fail(MT_ERR_INVALID_ARG, "trace_summarize: interval %d ends before it begins", i);
    const double b = std::max(0.0, double(r.begin_ms)), e = std::max(0.0, double(r.end_ms));
    const double d = e - b;
    out->span_ms = std::max(out->span_ms, e);
    switch (r.kind) {
      case 0: out->h2d_ms += d; up.push_back({b, e}); break;
      case 1: out->fwd_ms += d; comp.push_back({b, e}); break;
      case 2: out->refwd_ms += d; comp.push_back({b, e}); break;
      case 3: out->bwd_ms += d; comp.push_back({b, e}); break;
      default: out->d2h_ms += d; off.push_back({b, e}); break;
    }
    cuts.push_back(b);
    cuts.push_back(e);
  }
  comp = merged(comp);
  up = merged(up);
  off = merged(off);
  std::sort(cuts.begin(), cuts.end());
  // every elementary piece between consecutive boundaries is wholly inside or outside each union
  for (size_t i = 0; i + 1 < cuts.size(); ++i) {
    const double a = cuts[i], b = cuts[i + 1];
    if (b <= a) continue;
    const double mid = 0.5 * (a + b);
    if (covers(comp, mid)) continue;
    if (covers(up, mid))
      out->exposed_h2d_ms += b - a;
    else if (covers(off, mid))
      out->exposed_d2h_ms += b - a;
    else
      out->idle_other_ms += b - a;
  }
  return MT_OK;
}

// ======================================================================= engine
namespace {

using Clock = std::chrono::steady_clock;

struct EventTimer : GemmTimer {
  std::vector<cudaEvent_t> ev;
  std::vector<double> flops;
  size_t n = 0;
  bool overflow = false;
  void before(cudaStream_t st) override {
    if (n + 2 > ev.size()) {
      overflow = true;
      return;
    }
    cudaEventRecord(ev[n], st);
  }
  void after(cudaStream_t st, double f) override {
    if (overflow || n + 2 > ev.size()) return;
    cudaEventRecord(ev[n + 1], st);
    flops.push_back(f);
    n += 2;
  }
};

struct SinkItem {
  int jb, layer, slab;  // slab: pool index, or -1 for a record pinned for this layer only
  float* ptr;
};

}  // namespace

struct mt_engine {
  Geom G;
  mt_layer_cfg cfg;
  int L, B, T, K, R, NS, NG, S;
  int64_t M;
  mt_engine_opts opts;
  cudaStream_t cs, ps, os;
  // device buffers
  std::vector<mt_bf16*> slot;
  std::vector<float*> dgrad;
  std::vector<mt_bf16*> ckpt, seg;
  mt_bf16 *act[2] = {nullptr, nullptr}, *gbuf[2] = {nullptr, nullptr}, *io[4] = {nullptr, nullptr, nullptr, nullptr};
  // layer workspaces: internals sets (one per position in a segment, or one when every
  // backward recomputes its layer's internals) and one scratch set for the backward
  std::vector<void*> lws_int;
  void* lws_scr = nullptr;
  uint64_t int_bytes = 0, scr_bytes = 0, dev_bytes = 0;
  // host slab pool
  std::vector<float*> slab;
  std::mutex mu;
  std::condition_variable cv;
  std::vector<int> free_slabs;
  std::deque<SinkItem> queue;
  bool producer_done = false, abort = false, sink_finished = true;
  mt_status sink_status = MT_OK;
  std::thread sink_thread;
  // schedule and events
  std::vector<Use> uses;
  std::vector<int> uslot, uload, prev_of_slot, load_of_use;
  std::vector<cudaEvent_t> ready, done, g_ready, d2h_done, mlp_done;
  std::vector<cudaEvent_t> ready_attn;  // per use: the record's head (g1 .. g2) is on the device
  std::vector<cudaEvent_t> wd_done;     // per backward: the down projection's gradient is final
  cudaEvent_t fin = nullptr;
  // timeline (opts.trace): timing events, the step's start, and (kind, layer, begin, end) slots
  struct TraceSlot {
    int kind, layer, eb, ee;
  };
  std::vector<cudaEvent_t> tr_ev;
  cudaEvent_t tr_t0 = nullptr;
  std::vector<TraceSlot> tr;
  int tr_used = 0;
  bool tr_valid = false;
  bool resident_loaded = false;
  int64_t h2d_count = 0;
  EventTimer timer;
  mt_stats st;
};

namespace {

mt_bf16* x_loc(mt_engine* e, int j, const mt_bf16* x0, mt_bf16* ytop) {
  if (j == 0) return const_cast<mt_bf16*>(x0);
  if (j == e->L) return ytop;
  if (j % e->K == 0) return e->ckpt[j / e->K - 1];
  return e->act[j % 2];
}

// Layer-internals sets the engine carves: one per position in a segment, or one
// when every backward recomputes its layer's internals.
int internal_sets(const mt_engine_opts& o, int L) {
  return o.recompute_internals ? 1 : std::min(o.ckpt_interval, L);
}

mt_status validate_opts(const mt_engine_opts* in, int L, mt_engine_opts* o) {
  if (!in) return fail(MT_ERR_INVALID_ARG, "opts is NULL");
  *o = *in;
  if (o->ckpt_interval < 1) return fail(MT_ERR_INVALID_ARG, "ckpt_interval must be >= 1");
  if (o->no_slab_pool < 0) return fail(MT_ERR_INVALID_ARG, "no_slab_pool must be 0 or 1");
  if (o->trace < 0 || o->trace > 1) return fail(MT_ERR_INVALID_ARG, "trace must be 0 or 1");
  if (o->recompute_internals < 0 || o->recompute_internals > 1)
    return fail(MT_ERR_INVALID_ARG, "recompute_internals must be 0 or 1");
  if (o->n_weight_slots < 0 || o->n_host_slabs < 0 || o->n_dev_grad_slabs < 0 || o->mlp_chunk < 0 ||
      o->timeout_ms < 0 || o->fail_h2d_at < 0)
    return fail(MT_ERR_INVALID_ARG, "engine options must be >= 0");
  if (o->n_weight_slots == 0) o->n_weight_slots = std::max(2, o->ckpt_interval);
  if (o->resident) o->n_weight_slots = L;
  if (o->n_host_slabs == 0) o->n_host_slabs = 3;
  if (o->n_dev_grad_slabs == 0) o->n_dev_grad_slabs = 2;
  if (o->timeout_ms == 0) o->timeout_ms = 60000;
  return MT_OK;
}

Bump carve_engine(const Geom& G, int L, int B, int T, const mt_engine_opts& o, void* base, uint64_t cap,
                  mt_engine* e) {
  const int64_t M = static_cast<int64_t>(B) * T;
  const int K = o.ckpt_interval;
  const int S = (L + K - 1) / K;
  const int64_t rec = static_cast<int64_t>(G.off.record_elems);
  Bump bp(base, cap);
  for (int r = 0; r < o.n_weight_slots; ++r) {
    mt_bf16* p = bp.take<mt_bf16>(rec);
    if (e) e->slot.push_back(p);
  }
  for (int r = 0; r < o.n_dev_grad_slabs; ++r) {
    float* p = bp.take<float>(rec);
    if (e) e->dgrad.push_back(p);
  }
  for (int s = 1; s < S; ++s) {
    mt_bf16* p = bp.take<mt_bf16>(M * G.H);
    if (e) e->ckpt.push_back(p);
  }
  for (int s = 0; s < K - 1; ++s) {
    mt_bf16* p = bp.take<mt_bf16>(M * G.H);
    if (e) e->seg.push_back(p);
  }
  for (int i = 0; i < 2; ++i) {
    mt_bf16* a = bp.take<mt_bf16>(M * G.H);
    mt_bf16* g = bp.take<mt_bf16>(M * G.H);
    if (e) {
      e->act[i] = a;
      e->gbuf[i] = g;
    }
  }
  for (int i = 0; i < 4; ++i) {
    mt_bf16* p = bp.take<mt_bf16>(M * G.H);
    if (e) e->io[i] = p;
  }
  return bp;
}

mt_status poll_event(cudaEvent_t ev, Clock::time_point deadline, const char* what) {
  for (int spin = 0;; ++spin) {
    cudaError_t r = cudaEventQuery(ev);
    if (r == cudaSuccess) return MT_OK;
    if (r != cudaErrorNotReady) return fail(MT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(r));
    if (Clock::now() > deadline) return fail(MT_ERR_TIMEOUT, "%s: timed out", what);
    if (spin > 64) std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

mt_status poll_stream(cudaStream_t s, Clock::time_point deadline, const char* what) {
  for (int spin = 0;; ++spin) {
    cudaError_t r = cudaStreamQuery(s);
    if (r == cudaSuccess) return MT_OK;
    if (r != cudaErrorNotReady) return fail(MT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(r));
    if (Clock::now() > deadline) return fail(MT_ERR_TIMEOUT, "%s: timed out", what);
    if (spin > 64) std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
}

void sink_loop(mt_engine* e, mt_grad_sink sink, void* user) {
  const uint64_t rec = e->G.off.record_elems;
  for (;;) {
    SinkItem it;
    {
      std::unique_lock<std::mutex> lk(e->mu);
      e->cv.wait(lk, [e] { return !e->queue.empty() || e->producer_done || e->abort; });
      if (e->queue.empty() || e->abort) break;
      it = e->queue.front();
      e->queue.pop_front();
    }
    const auto deadline = Clock::now() + std::chrono::milliseconds(e->opts.timeout_ms);
    mt_status s = poll_event(e->d2h_done[it.jb], deadline, "gradient offload");
    double sink_ms = 0.0;
    if (s == MT_OK && sink) {
      const auto t0 = Clock::now();
      int32_t rc = sink(it.layer, it.ptr, rec, user);
      sink_ms = std::chrono::duration<double, std::milli>(Clock::now() - t0).count();
      if (rc != 0) s = fail(MT_ERR_SINK, "gradient sink returned %d for layer %d", rc, it.layer);
    }
    if (it.slab < 0) cudaFreeHost(it.ptr);  // no pool: the record was pinned for this layer only
    std::lock_guard<std::mutex> lk(e->mu);
    e->st.sink_ms += sink_ms;
    if (it.slab >= 0) e->free_slabs.push_back(it.slab);
    if (s != MT_OK) {
      e->sink_status = s;
      e->abort = true;
    }
    e->cv.notify_all();
    if (s != MT_OK) break;
  }
  std::lock_guard<std::mutex> lk(e->mu);
  e->sink_finished = true;
  e->cv.notify_all();
}

// The schedule of one step, derived from the static use list.
void prepare_schedule(mt_engine* e) {
  e->uses = build_uses(e->L, e->K);
  plan_slots(e->uses, e->R, e->uslot, e->uload);
  const int n = static_cast<int>(e->uses.size());
  e->prev_of_slot.assign(n, -1);
  e->load_of_use.assign(n, -1);
  std::vector<int> last_use(e->R, -1), last_load(e->R, -1);
  for (int i = 0; i < n; ++i) {
    const int s = e->uslot[i];
    e->prev_of_slot[i] = last_use[s];
    if (e->uload[i]) last_load[s] = i;
    e->load_of_use[i] = last_load[s];
    last_use[s] = i;
  }
}

// Interval k of the last traced step, in milliseconds from the step's origin.
mt_status read_trace_rec(mt_engine* e, int k, mt_trace_rec* out) {
  const auto& t = e->tr[k];
  float b = 0.f, en = 0.f;
  MT_CUDA(cudaEventElapsedTime(&b, e->tr_t0, e->tr_ev[t.eb]));
  MT_CUDA(cudaEventElapsedTime(&en, e->tr_t0, e->tr_ev[t.ee]));
  *out = {t.kind, t.layer, b, en};
  return MT_OK;
}

mt_status run_step(mt_engine* e, mt_host_store* store, const mt_bf16* x0, const mt_bf16* dy_top, mt_bf16* y_top,
                   mt_bf16* dx0, mt_grad_sink sink, void* user, mt_head_hook hook, void* hook_user) {
  const uint64_t rec = e->G.off.record_elems;
  const int n = static_cast<int>(e->uses.size());
  const bool skip_loads = e->opts.resident && e->resident_loaded;
  int next_load = 0;
  int jb = 0;  // backward index
  mt_status status = MT_OK;
  const auto timeout = std::chrono::milliseconds(e->opts.timeout_ms);

  // timeline: begin / end events of one interval on a stream (no-ops without opts.trace, and
  // once the event pool is used up)
  const bool tracing = e->opts.trace != 0;
  e->tr.clear();
  e->tr_used = 0;
  e->tr_valid = false;
  auto tr_begin = [e, tracing](int kind, int layer, cudaStream_t stream) -> int {
    if (!tracing || e->tr_used + 2 > static_cast<int>(e->tr_ev.size())) return -1;
    const int k = static_cast<int>(e->tr.size());
    e->tr.push_back({kind, layer, e->tr_used, e->tr_used + 1});
    e->tr_used += 2;
    if (cudaEventRecord(e->tr_ev[e->tr[k].eb], stream) != cudaSuccess) {
      cudaGetLastError();
      e->tr.pop_back();
      return -1;
    }
    return k;
  };
  auto tr_end = [e](int k, cudaStream_t stream) {
    if (k < 0) return;
    if (cudaEventRecord(e->tr_ev[e->tr[k].ee], stream) != cudaSuccess) cudaGetLastError();
  };
  if (tracing) {  // the step's time origin, ahead of everything on all three streams
    MT_CUDA(cudaEventRecord(e->tr_t0, e->cs));
    MT_CUDA(cudaStreamWaitEvent(e->ps, e->tr_t0, 0));
    MT_CUDA(cudaStreamWaitEvent(e->os, e->tr_t0, 0));
  }

  // sink thread for this step
  {
    std::lock_guard<std::mutex> lk(e->mu);
    e->queue.clear();
    e->producer_done = false;
    e->abort = false;
    e->sink_status = MT_OK;
    e->sink_finished = false;
    e->free_slabs.clear();
    for (int i = 0; i < static_cast<int>(e->slab.size()); ++i) e->free_slabs.push_back(i);
  }
  if (e->sink_thread.joinable()) e->sink_thread.join();  // finished: checked by the caller
  e->sink_thread = std::thread(sink_loop, e, sink, user);

  auto enqueue_loads = [&](int computed) -> mt_status {
    // enqueue, in use order, every load whose slot's previous user has been enqueued
    while (next_load < n) {
      if (skip_loads || !e->uload[next_load]) {
        ++next_load;
        continue;
      }
      const int p = e->prev_of_slot[next_load];
      if (p >= computed) break;
      if (e->opts.fail_h2d_at > 0 && e->h2d_count + 1 == e->opts.fail_h2d_at) {
        ++e->h2d_count;
        return fail(MT_ERR_INJECTED, "injected failure of weight copy %lld", (long long)e->h2d_count);
      }
      if (p >= 0) MT_CUDA(cudaStreamWaitEvent(e->ps, e->done[p], 0));
      const int layer = e->uses[next_load].layer;
      // two pieces: the record's head (g1 .. g2, all the attention half reads) first, so that a
      // forward can start its attention while the MLP weights are still crossing the link
      const uint64_t head = e->G.off.wg;
      mt_bf16* dst = e->slot[e->uslot[next_load]];
      const mt_bf16* src = mt_host_store_bf16(store, layer);
      const int tk = tr_begin(0, layer, e->ps);
      MT_CUDA(cudaMemcpyAsync(dst, src, head * 2, cudaMemcpyHostToDevice, e->ps));
      MT_CUDA(cudaEventRecord(e->ready_attn[next_load], e->ps));
      MT_CUDA(cudaMemcpyAsync(dst + head, src + head, (rec - head) * 2, cudaMemcpyHostToDevice, e->ps));
      MT_CUDA(cudaEventRecord(e->ready[next_load], e->ps));
      tr_end(tk, e->ps);
      ++e->h2d_count;
      e->st.h2d_bytes += rec * 2;
      e->st.weight_loads += 1;
      ++next_load;
    }
    return MT_OK;
  };

  for (int i = 0; i < n && status == MT_OK; ++i) {
    {
      std::lock_guard<std::mutex> lk(e->mu);
      if (e->abort) {
        status = e->sink_status != MT_OK ? e->sink_status : fail(MT_ERR_TIMEOUT, "step aborted");
        break;
      }
    }
    status = enqueue_loads(i);
    if (status != MT_OK) break;
    const Use u = e->uses[i];
    if (hook && u.kind != 0 && e->uses[i - 1].kind == 0) {
      // between the forward and the backward: the caller's head turns y_top into dy_top
      status = hook(y_top, const_cast<mt_bf16*>(dy_top), e->cs, hook_user);
      if (status != MT_OK) break;
    }
    const int l = u.layer;
    const int s = l / e->K, a = s * e->K;
    mt_bf16* w = e->slot[e->uslot[i]];
    // a forward waits for the record's head and hands the full-record event to the layer, which
    // waits for it before its MLP; a backward waits for the whole record
    cudaEvent_t mlp_weights = nullptr;
    if (!skip_loads && e->load_of_use[i] >= 0) {
      const int ld = e->load_of_use[i];
      if (u.kind == 2) {
        status = cuda_check(cudaStreamWaitEvent(e->cs, e->ready[ld], 0), "wait weights");
      } else {
        status = cuda_check(cudaStreamWaitEvent(e->cs, e->ready_attn[ld], 0), "wait weights");
        mlp_weights = e->ready[ld];
      }
      if (status != MT_OK) break;
    }
    // Which forwards leave their internals for their backward, and so which backwards skip the
    // recompute. Keeping (the default): every forward of the last segment and every segment
    // re-forward keeps them in the internals set of its position in the segment; only the top
    // layer of each earlier segment, which its re-forward does not reach, recomputes. With
    // recompute_internals there is one set, and only the top layer, whose backward directly
    // follows its forward, reuses it.
    const int a_last = (e->S - 1) * e->K;
    const int b_seg = std::min(e->L, a + e->K);
    const bool keep_all = !e->opts.recompute_internals;
    const int pos = keep_all ? l - a : 0;
    bool keep = false, reuse = false;
    if (keep_all) {
      keep = u.kind == 1 || (u.kind == 0 && l >= a_last);
      reuse = u.kind == 2 && (l >= a_last || l < b_seg - 1);
    } else {
      keep = i + 1 < n && u.kind == 0 && e->uses[i + 1].kind == 2 && e->uses[i + 1].layer == l;
      reuse = i > 0 && u.kind == 2 && e->uses[i - 1].kind == 0 && e->uses[i - 1].layer == l;
    }
    void* lws = e->lws_int[pos];
    const int tk = tr_begin(u.kind + 1, l, e->cs);
    if (u.kind == 0) {
      // inside the last segment the forward keeps its activations in the segment buffers
      const mt_bf16* xin = (l > a_last) ? e->seg[l - a_last - 1] : x_loc(e, l, x0, y_top);
      mt_bf16* xout = (l + 1 < e->L && l + 1 > a_last) ? e->seg[l - a_last] : x_loc(e, l + 1, x0, y_top);
      status = layer_fwd_keep(&e->cfg, w, xin, xout, e->B, e->T, e->opts.mlp_chunk, lws, e->int_bytes, e->cs, keep,
                              mlp_weights);
      e->st.layer_fwd_calls++;
      tr_end(tk, e->cs);
    } else if (u.kind == 1) {
      const mt_bf16* xin = (l == a) ? x_loc(e, a, x0, y_top) : e->seg[l - a - 1];
      status = layer_fwd_keep(&e->cfg, w, xin, e->seg[l - a], e->B, e->T, e->opts.mlp_chunk, lws, e->int_bytes, e->cs,
                              keep, mlp_weights);
      e->st.layer_fwd_calls++;
      tr_end(tk, e->cs);
    } else {
      const mt_bf16* xin = (l == a) ? x_loc(e, a, x0, y_top) : e->seg[l - a - 1];
      const mt_bf16* dy = (jb == 0) ? dy_top : e->gbuf[(jb - 1) % 2];
      mt_bf16* dx = (l == 0) ? dx0 : e->gbuf[jb % 2];
      const int ns = jb % e->NG;
      if (jb >= e->NG) {
        status = cuda_check(cudaStreamWaitEvent(e->cs, e->d2h_done[jb - e->NG], 0), "wait staging slab");
        if (status != MT_OK) break;
      }
      status = layer_recompute_bwd_ev(&e->cfg, w, xin, dy, dx, e->dgrad[ns], e->B, e->T, e->opts.mlp_chunk, lws,
                                      e->int_bytes, e->lws_scr, e->scr_bytes, e->cs, e->mlp_done[jb], reuse,
                                      e->wd_done[jb]);
      e->st.layer_bwd_calls++;
      tr_end(tk, e->cs);
      if (status == MT_OK) status = cuda_check(cudaEventRecord(e->g_ready[jb], e->cs), "record g_ready");
      if (status == MT_OK) {
        // take a pinned slab from the pool (bounded wait), then offload. Without the pool
        // (the Table 4 ablation) a record is pinned for this layer and freed after its sink.
        int p = -1;
        float* dst = nullptr;
        if (e->opts.no_slab_pool) {
          if (cudaHostAlloc(reinterpret_cast<void**>(&dst), rec * 4, cudaHostAllocPortable) != cudaSuccess) {
            cudaGetLastError();
            status = fail(MT_ERR_OOM, "pinned allocation of a gradient record failed");
          }
        } else {
          std::unique_lock<std::mutex> lk(e->mu);
          const bool got = e->cv.wait_for(lk, timeout, [e] { return !e->free_slabs.empty() || e->abort; });
          if (e->abort) {
            status = e->sink_status != MT_OK ? e->sink_status : fail(MT_ERR_TIMEOUT, "step aborted");
          } else if (!got) {
            status = fail(MT_ERR_TIMEOUT, "no free gradient slab within %d ms", e->opts.timeout_ms);
          } else {
            p = e->free_slabs.back();
            e->free_slabs.pop_back();
            dst = e->slab[p];
          }
        }
        // three pieces, each as soon as it is final: the down projection's gradient (the record's
        // tail from Wd on), then the gate / up projections' (Wg, Wu), then the rest when the layer is done
        const uint64_t split = e->G.off.wg, split_d = e->G.off.wd;
        if (status == MT_OK) status = cuda_check(cudaStreamWaitEvent(e->os, e->wd_done[jb], 0), "wait wd_done");
        const int tko = status == MT_OK ? tr_begin(4, l, e->os) : -1;
        if (status == MT_OK)
          status = cuda_check(cudaMemcpyAsync(dst + split_d, e->dgrad[ns] + split_d, (rec - split_d) * 4,
                                              cudaMemcpyDeviceToHost, e->os),
                              "gradient D2H");
        if (status == MT_OK) status = cuda_check(cudaStreamWaitEvent(e->os, e->mlp_done[jb], 0), "wait mlp_done");
        if (status == MT_OK)
          status = cuda_check(cudaMemcpyAsync(dst + split, e->dgrad[ns] + split, (split_d - split) * 4,
                                              cudaMemcpyDeviceToHost, e->os),
                              "gradient D2H");
        if (status == MT_OK) status = cuda_check(cudaStreamWaitEvent(e->os, e->g_ready[jb], 0), "wait g_ready");
        if (status == MT_OK)
          status = cuda_check(
              cudaMemcpyAsync(dst, e->dgrad[ns], split * 4, cudaMemcpyDeviceToHost, e->os), "gradient D2H");
        tr_end(tko, e->os);
        if (status == MT_OK) status = cuda_check(cudaEventRecord(e->d2h_done[jb], e->os), "record d2h_done");
        if (status == MT_OK) {
          e->st.d2h_bytes += rec * 4;
          std::lock_guard<std::mutex> lk(e->mu);
          e->queue.push_back({jb, l, p, dst});
          e->cv.notify_all();
        } else if (p >= 0) {
          std::lock_guard<std::mutex> lk(e->mu);
          e->free_slabs.push_back(p);
        } else if (dst) {
          cudaStreamSynchronize(e->os);
          cudaFreeHost(dst);
        }
      }
      ++jb;
    }
    if (status != MT_OK) break;
    status = cuda_check(cudaEventRecord(e->done[i], e->cs), "record done");
  }
  if (status == MT_OK) status = enqueue_loads(n);

  // let the sink thread drain (bounded), then wait for the compute stream
  {
    std::unique_lock<std::mutex> lk(e->mu);
    e->producer_done = true;
    if (status != MT_OK) e->abort = true;
    e->cv.notify_all();
    const bool fin = e->cv.wait_for(lk, timeout * 2, [e] { return e->sink_finished; });
    if (!fin && status == MT_OK) status = fail(MT_ERR_TIMEOUT, "gradient sink did not finish within the timeout");
    if (status == MT_OK && e->sink_status != MT_OK) status = e->sink_status;
  }
  if (e->sink_finished && e->sink_thread.joinable()) e->sink_thread.join();
  if (status == MT_OK) {
    status = cuda_check(cudaEventRecord(e->fin, e->cs), "record fin");
    if (status == MT_OK) status = poll_event(e->fin, Clock::now() + timeout, "compute stream");
  }
  if (status == MT_OK && e->opts.resident) e->resident_loaded = true;
  if (status == MT_OK && tracing) e->tr_valid = true;
  return status;
}

}  // namespace

extern "C" {

uint64_t mt_engine_workspace_bytes(const mt_layer_cfg* cfg, int32_t n_layers, int32_t B, int32_t T,
                                   const mt_engine_opts* opts) {
  Geom G;
  mt_engine_opts o;
  if (make_geom(cfg, &G) != MT_OK || n_layers <= 0 || validate_opts(opts, n_layers, &o) != MT_OK) return 0;
  Bump bp = carve_engine(G, n_layers, B, T, o, nullptr, 0, nullptr);
  uint64_t wi = 0, wsc = 0;
  if (layer_ws_sizes(cfg, B, T, o.mlp_chunk, &wi, &wsc) != MT_OK) return 0;
  return bp.used + internal_sets(o, n_layers) * wi + wsc;
}

mt_status mt_engine_create(const mt_layer_cfg* cfg, int32_t n_layers, int32_t B, int32_t T,
                           const mt_engine_opts* opts, void* dev_ws, uint64_t dev_ws_bytes, void* compute_stream,
                           void* prefetch_stream, void* offload_stream, mt_engine** out) {
  if (!out) return fail(MT_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  Geom G;
  MT_TRY(make_geom(cfg, &G));
  if (n_layers <= 0 || B <= 0 || T <= 0) return fail(MT_ERR_INVALID_ARG, "n_layers, B, T must be positive");
  mt_engine_opts o;
  MT_TRY(validate_opts(opts, n_layers, &o));
  if (!compute_stream || !prefetch_stream || !offload_stream || compute_stream == prefetch_stream ||
      compute_stream == offload_stream || prefetch_stream == offload_stream)
    return fail(MT_ERR_INVALID_ARG, "compute, prefetch and offload must be three distinct non-default streams");
  const uint64_t need = mt_engine_workspace_bytes(cfg, n_layers, B, T, &o);
  if (need == 0) return fail(MT_ERR_INVALID_ARG, "layer workspace unavailable: %s", mt_last_error());
  if (!dev_ws || !aligned16(dev_ws)) return fail(MT_ERR_ALIGNMENT, "device workspace must be 16-byte aligned");
  if (dev_ws_bytes < need)
    return fail(MT_ERR_WORKSPACE, "engine workspace %llu < %llu bytes", (unsigned long long)dev_ws_bytes,
                (unsigned long long)need);
  auto* e = new mt_engine();
  e->G = G;
  e->cfg = *cfg;
  e->L = n_layers;
  e->B = B;
  e->T = T;
  e->M = static_cast<int64_t>(B) * T;
  e->opts = o;
  e->K = o.ckpt_interval;
  e->R = o.n_weight_slots;
  e->NS = o.n_host_slabs;
  e->NG = o.n_dev_grad_slabs;
  e->S = (n_layers + e->K - 1) / e->K;
  e->cs = as_stream(compute_stream);
  e->ps = as_stream(prefetch_stream);
  e->os = as_stream(offload_stream);
  Bump bp = carve_engine(G, n_layers, B, T, o, dev_ws, dev_ws_bytes, e);
  MT_TRY(layer_ws_sizes(cfg, B, T, o.mlp_chunk, &e->int_bytes, &e->scr_bytes));
  char* lw = static_cast<char*>(dev_ws) + bp.used;
  for (int i = 0; i < internal_sets(o, n_layers); ++i, lw += e->int_bytes) e->lws_int.push_back(lw);
  e->lws_scr = lw;
  e->dev_bytes = need;
  prepare_schedule(e);
  auto cleanup = [e](mt_status s) {
    mt_engine_destroy(e);
    return s;
  };
  const uint64_t rec = G.off.record_elems;
  for (int i = 0; i < (o.no_slab_pool ? 0 : e->NS); ++i) {
    float* p = nullptr;
    if (cudaHostAlloc(reinterpret_cast<void**>(&p), rec * 4, cudaHostAllocPortable) != cudaSuccess) {
      cudaGetLastError();
      return cleanup(fail(MT_ERR_OOM, "pinned gradient slab allocation failed"));
    }
    e->slab.push_back(p);
  }
  const int n = static_cast<int>(e->uses.size());
  auto mk = [](std::vector<cudaEvent_t>& v, int count) -> mt_status {
    v.assign(count, nullptr);
    for (int i = 0; i < count; ++i) MT_CUDA(cudaEventCreateWithFlags(&v[i], cudaEventDisableTiming));
    return MT_OK;
  };
  mt_status s = mk(e->ready, n);
  if (s == MT_OK) s = mk(e->ready_attn, n);
  if (s == MT_OK) s = mk(e->wd_done, n_layers);
  if (s == MT_OK) s = mk(e->done, n);
  if (s == MT_OK) s = mk(e->g_ready, n_layers);
  if (s == MT_OK) s = mk(e->d2h_done, n_layers);
  if (s == MT_OK) s = mk(e->mlp_done, n_layers);
  if (s == MT_OK) s = cuda_check(cudaEventCreateWithFlags(&e->fin, cudaEventDisableTiming), "event");
  if (s == MT_OK && o.trace) {
    // two timing events per upload (at most one per use), layer call and offload
    e->tr_ev.assign(2 * (2 * n + n_layers), nullptr);
    for (auto& ev : e->tr_ev) {
      s = cuda_check(cudaEventCreate(&ev), "trace event");
      if (s != MT_OK) break;
    }
    if (s == MT_OK) s = cuda_check(cudaEventCreate(&e->tr_t0), "trace event");
  }
  if (s == MT_OK && o.time_gemms) {
    e->timer.ev.assign(8192, nullptr);
    for (auto& ev : e->timer.ev) {
      s = cuda_check(cudaEventCreate(&ev), "timing event");
      if (s != MT_OK) break;
    }
  }
  if (s != MT_OK) return cleanup(s);
  std::memset(&e->st, 0, sizeof(e->st));
  e->st.device_bytes = need;
  *out = e;
  return MT_OK;
}

mt_status mt_stream_step(mt_engine* e, mt_host_store* store, const mt_bf16* x0, const mt_bf16* dy_top, mt_bf16* y_top,
                         mt_bf16* dx0, mt_grad_sink sink, void* user) {
  return mt_stream_step_hooked(e, store, x0, const_cast<mt_bf16*>(dy_top), y_top, dx0, sink, user, nullptr, nullptr);
}

mt_status mt_stream_step_hooked(mt_engine* e, mt_host_store* store, const mt_bf16* x0, mt_bf16* dy_top,
                                mt_bf16* y_top, mt_bf16* dx0, mt_grad_sink sink, void* user, mt_head_hook hook,
                                void* hook_user) {
  if (!e || !store || !x0 || !dy_top || !y_top || !dx0) return fail(MT_ERR_INVALID_ARG, "stream_step: NULL argument");
  if (store->L != e->L || store->G.off.record_elems != e->G.off.record_elems)
    return fail(MT_ERR_INVALID_ARG, "host store does not match the engine's layer count or shape");
  if (!aligned16(x0) || !aligned16(dy_top) || !aligned16(y_top) || !aligned16(dx0))
    return fail(MT_ERR_ALIGNMENT, "stream_step: activation pointers must be 16-byte aligned");
  if (!e->sink_finished) return fail(MT_ERR_INVALID_ARG, "engine has an unfinished step; call mt_engine_reset");
  const auto t0 = Clock::now();
  const double f0 = exec_flops_counter();
  const uint64_t k0 = launch_counter();
  const uint64_t h2d0 = e->st.h2d_bytes, d2h0 = e->st.d2h_bytes;
  {
    std::lock_guard<std::mutex> lk(e->mu);
    e->st.sink_ms = 0;
  }
  e->timer.n = 0;
  e->timer.flops.clear();
  e->timer.overflow = false;
  if (e->opts.time_gemms) set_gemm_timer(&e->timer);
  mt_status s = run_step(e, store, x0, dy_top, y_top, dx0, sink, user, hook, hook_user);
  set_gemm_timer(nullptr);
  e->st.step_ms = std::chrono::duration<double, std::milli>(Clock::now() - t0).count();
  e->st.exec_flops = exec_flops_counter() - f0;
  e->st.kernel_launches = launch_counter() - k0;
  e->st.h2d_bytes -= h2d0;
  e->st.d2h_bytes -= d2h0;
  e->st.gemm_ms = 0;
  e->st.gemm_flops = 0;
  e->st.gemm_launches = 0;
  e->st.traced = 0;
  std::memset(&e->st.trace, 0, sizeof(e->st.trace));
  if (s == MT_OK && e->opts.trace && e->tr_valid) {
    std::vector<mt_trace_rec> recs(e->tr.size());
    mt_status ts = MT_OK;
    for (size_t k = 0; k < recs.size() && ts == MT_OK; ++k) ts = read_trace_rec(e, static_cast<int>(k), &recs[k]);
    if (ts == MT_OK) ts = mt_trace_summarize(recs.data(), static_cast<int32_t>(recs.size()), &e->st.trace);
    if (ts != MT_OK) return ts;
    e->st.traced = 1;
  }
  if (s == MT_OK && e->opts.time_gemms) {
    for (size_t k = 0; 2 * k + 1 < e->timer.n; ++k) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, e->timer.ev[2 * k], e->timer.ev[2 * k + 1]) == cudaSuccess) {
        e->st.gemm_ms += ms;
        e->st.gemm_flops += e->timer.flops[k];
        e->st.gemm_launches += 1;
      }
    }
  }
  return s;
}

mt_status mt_stream_step_host(mt_engine* e, mt_host_store* store, const mt_bf16* x0_host, const mt_bf16* dy_top_host,
                              mt_bf16* y_top_host, mt_bf16* dx0_host, mt_grad_sink sink, void* user) {
  if (!e || !x0_host || !dy_top_host || !y_top_host || !dx0_host)
    return fail(MT_ERR_INVALID_ARG, "stream_step_host: NULL argument");
  const uint64_t bytes = static_cast<uint64_t>(e->M) * e->G.H * 2;
  MT_CUDA(cudaMemcpyAsync(e->io[0], x0_host, bytes, cudaMemcpyHostToDevice, e->cs));
  MT_CUDA(cudaMemcpyAsync(e->io[1], dy_top_host, bytes, cudaMemcpyHostToDevice, e->cs));
  MT_TRY(mt_stream_step(e, store, e->io[0], e->io[1], e->io[2], e->io[3], sink, user));
  MT_CUDA(cudaMemcpyAsync(y_top_host, e->io[2], bytes, cudaMemcpyDeviceToHost, e->cs));
  MT_CUDA(cudaMemcpyAsync(dx0_host, e->io[3], bytes, cudaMemcpyDeviceToHost, e->cs));
  MT_CUDA(cudaEventRecord(e->fin, e->cs));
  MT_TRY(poll_event(e->fin, Clock::now() + std::chrono::milliseconds(e->opts.timeout_ms), "output copies"));
  e->st.h2d_bytes += 2 * bytes;
  e->st.d2h_bytes += 2 * bytes;
  return MT_OK;
}

mt_status mt_engine_stats(const mt_engine* e, mt_stats* out) {
  if (!e || !out) return fail(MT_ERR_INVALID_ARG, "NULL argument");
  *out = e->st;
  return MT_OK;
}

mt_status mt_engine_trace(mt_engine* e, mt_trace_rec* out, int32_t cap, int32_t* n) {
  if (!e || !n || cap < 0 || (cap > 0 && !out)) return fail(MT_ERR_INVALID_ARG, "engine_trace: bad argument");
  if (!e->opts.trace || !e->tr_valid)
    return fail(MT_ERR_INVALID_ARG, "engine_trace: the engine has no traced step (create it with trace = 1)");
  const int avail = static_cast<int>(e->tr.size());
  for (int k = 0; k < avail && k < cap; ++k) MT_TRY(read_trace_rec(e, k, &out[k]));
  *n = avail;
  return MT_OK;
}

mt_status mt_engine_reset(mt_engine* e) {
  if (!e) return fail(MT_ERR_INVALID_ARG, "engine is NULL");
  const auto deadline = Clock::now() + std::chrono::milliseconds(e->opts.timeout_ms);
  {
    std::unique_lock<std::mutex> lk(e->mu);
    e->abort = true;
    e->producer_done = true;
    e->cv.notify_all();
    if (!e->cv.wait_until(lk, deadline, [e] { return e->sink_finished; }))
      return fail(MT_ERR_TIMEOUT, "gradient sink still running");
  }
  if (e->sink_thread.joinable()) e->sink_thread.join();
  MT_TRY(poll_stream(e->cs, deadline, "compute stream"));
  MT_TRY(poll_stream(e->ps, deadline, "prefetch stream"));
  MT_TRY(poll_stream(e->os, deadline, "offload stream"));
  std::lock_guard<std::mutex> lk(e->mu);
  e->abort = false;
  for (const SinkItem& it : e->queue)
    if (it.slab < 0) cudaFreeHost(it.ptr);
  e->queue.clear();
  e->sink_status = MT_OK;
  return MT_OK;
}

void mt_engine_destroy(mt_engine* e) {
  if (!e) return;
  {
    std::unique_lock<std::mutex> lk(e->mu);
    e->abort = true;
    e->producer_done = true;
    e->cv.notify_all();
  }
  if (e->sink_thread.joinable()) e->sink_thread.join();
  cudaStreamSynchronize(e->cs);
  cudaStreamSynchronize(e->ps);
  cudaStreamSynchronize(e->os);
  for (auto* v : {&e->ready, &e->ready_attn, &e->wd_done, &e->done, &e->g_ready, &e->d2h_done, &e->mlp_done,
                  &e->timer.ev, &e->tr_ev})
    for (auto ev : *v)
      if (ev) cudaEventDestroy(ev);
  if (e->fin) cudaEventDestroy(e->fin);
  if (e->tr_t0) cudaEventDestroy(e->tr_t0);
  for (float* p : e->slab) cudaFreeHost(p);
  delete e;
}

}  // extern "C"

// ======================================================================= CPU optimizer
// The optimizer step of the memory-centric design runs on the host (blog
// summary, design point 1: "Optimizer steps execute entirely on the CPU",
// with Adam momentum and variance in host memory). AdamW (decoupled weight
// decay): m = b1 m + (1-b1) g; v = b2 v + (1-b2) g^2;
// w -= lr * (m / (1-b1^t) / (sqrt(v / (1-b2^t)) + eps) + wd * w).
struct mt_host_optimizer {
  mt_host_store* store;
  mt_adamw_cfg cfg;
  float* m = nullptr;
  float* v = nullptr;
  std::vector<int64_t> steps;  // per layer: updates applied so far
};

static mt_status adamw_check(const mt_adamw_cfg* c) {
  if (!c) return fail(MT_ERR_INVALID_ARG, "adamw cfg is NULL");
  if (!(c->lr >= 0.f) || !(c->beta1 >= 0.f && c->beta1 < 1.f) || !(c->beta2 >= 0.f && c->beta2 < 1.f) ||
      !(c->eps > 0.f) || !(c->weight_decay >= 0.f))
    return fail(MT_ERR_INVALID_ARG, "adamw: need lr >= 0, 0 <= beta < 1, eps > 0, weight_decay >= 0");
  return MT_OK;
}

static void adamw_range(float* w, float* m, float* v, const float* g, int64_t a, int64_t b, const mt_adamw_cfg& c,
                        double bc1, double bc2) {
  const float b1 = c.beta1, b2 = c.beta2, lr = c.lr, eps = c.eps, wd = c.weight_decay;
  const float ib1 = static_cast<float>(1.0 / bc1), ib2 = static_cast<float>(1.0 / bc2);
  for (int64_t i = a; i < b; ++i) {
    const float gi = g[i];
    const float mi = b1 * m[i] + (1.f - b1) * gi;
    const float vi = b2 * v[i] + (1.f - b2) * gi * gi;
    m[i] = mi;
    v[i] = vi;
    w[i] -= lr * ((mi * ib1) / (std::sqrt(vi * ib2) + eps) + wd * w[i]);
  }
}

extern "C" {

mt_status mt_adamw_update(float* w, float* m, float* v, const float* g, uint64_t n, const mt_adamw_cfg* cfg,
                          int64_t t) {
  MT_TRY(adamw_check(cfg));
  if (!w || !m || !v || !g) return fail(MT_ERR_INVALID_ARG, "adamw: NULL array");
  if (t < 1) return fail(MT_ERR_INVALID_ARG, "adamw: step t must be >= 1");
  const double bc1 = 1.0 - std::pow(static_cast<double>(cfg->beta1), static_cast<double>(t));
  const double bc2 = 1.0 - std::pow(static_cast<double>(cfg->beta2), static_cast<double>(t));
  const mt_adamw_cfg c = *cfg;
  parallel_for(static_cast<int64_t>(n), cfg->n_threads > 0 ? cfg->n_threads : default_threads(),
               [&](int64_t a, int64_t b) { adamw_range(w, m, v, g, a, b, c, bc1, bc2); });
  return MT_OK;
}

mt_status mt_host_optimizer_create(mt_host_store* store, const mt_adamw_cfg* cfg, mt_host_optimizer** out) {
  if (!out || !store) return fail(MT_ERR_INVALID_ARG, "NULL argument");
  *out = nullptr;
  MT_TRY(adamw_check(cfg));
  if (!store->master) return fail(MT_ERR_INVALID_ARG, "the optimizer needs the store's fp32 master copy");
  auto* o = new mt_host_optimizer();
  o->store = store;
  o->cfg = *cfg;
  const uint64_t n = store->G.off.record_elems * static_cast<uint64_t>(store->L);
  o->m = static_cast<float*>(std::calloc(n, sizeof(float)));
  o->v = static_cast<float*>(std::calloc(n, sizeof(float)));
  if (!o->m || !o->v) {
    mt_host_optimizer_destroy(o);
    return fail(MT_ERR_OOM, "optimizer state allocation (%llu floats x 2) failed", (unsigned long long)n);
  }
  o->steps.assign(store->L, 0);
  *out = o;
  return MT_OK;
}

int32_t mt_host_optimizer_sink(int32_t layer, const float* host_slab, uint64_t n_elems, void* user) {
  auto* o = static_cast<mt_host_optimizer*>(user);
  if (!o || !host_slab || layer < 0 || layer >= o->store->L || n_elems != o->store->G.off.record_elems) return 1;
  const mt_param_offsets& off = o->store->G.off;
  const Geom& G = o->store->G;
  const uint64_t base = static_cast<uint64_t>(layer) * off.record_elems;
  float* w = o->store->master + base;
  float* m = o->m + base;
  float* v = o->v + base;
  uint16_t* wb = o->store->bf + base;
  const int64_t t = ++o->steps[layer];
  const double bc1 = 1.0 - std::pow(static_cast<double>(o->cfg.beta1), static_cast<double>(t));
  const double bc2 = 1.0 - std::pow(static_cast<double>(o->cfg.beta2), static_cast<double>(t));
  // the record's tensors (its padding carries no parameter)
  const int64_t blocks[7][2] = {
      {static_cast<int64_t>(off.g1), G.H},
      {static_cast<int64_t>(off.wq), G.Nqkv * G.H},
      {static_cast<int64_t>(off.bq), G.bias ? G.Nqkv : 0},
      {static_cast<int64_t>(off.wo), G.H * G.Nq},
      {static_cast<int64_t>(off.g2), G.H},
      {static_cast<int64_t>(off.wg), 2 * G.F * G.H},
      {static_cast<int64_t>(off.wd), G.H * G.F},
  };
  const mt_adamw_cfg c = o->cfg;
  const int threads = c.n_threads > 0 ? c.n_threads : default_threads();
  for (const auto& blk : blocks) {
    const int64_t s0 = blk[0], len = blk[1];
    if (len == 0) continue;
    parallel_for(len, threads, [&](int64_t a, int64_t b) {
      adamw_range(w + s0, m + s0, v + s0, host_slab + s0, a, b, c, bc1, bc2);
      for (int64_t i = a; i < b; ++i) {  // refresh the streamed bf16 copy (round to nearest even)
        uint32_t u;
        std::memcpy(&u, w + s0 + i, 4);
        wb[s0 + i] = ((u & 0x7FFFFFFFu) > 0x7F800000u) ? static_cast<uint16_t>((u >> 16) | 0x40u)
                                                       : static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
      }
    });
  }
  return 0;
}

void mt_host_optimizer_destroy(mt_host_optimizer* o) {
  if (!o) return;
  std::free(o->m);
  std::free(o->v);
  delete o;
}

}  // extern "C"
