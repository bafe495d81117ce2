// C ABI of the H2O chunk-step library: handle, device state, and the
// stream-ordered sequence attend -> accumulate -> select -> scatter.
// The operation each call performs is documented in include/h2o.h.
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/h2o.h"
#include "h2o_internal.cuh"

namespace {

thread_local std::string g_thread_err = "no error";

struct DevBuf {
  void* p = nullptr;
  size_t cap = 0;
};

}  // namespace

int h2o::set_thread_error(int code, const char* msg) {
  g_thread_err = msg;
  return code;
}

struct h2o_ctx {
  int64_t M = 0, R = 0;
  int Hq = 0, Hkv = 0, d = 0, dtype = 0, G = 0, esize = 0;
  int policy = H2O_POLICY_H2O;
  int B = 0;
  int device = -1;
  int64_t t0 = 0, n_valid = 0, last_S = 0;
  int last_launches = 0;
  bool prefilled = false;
  bool use_umma = false;
  int row_tile = h2o::kSimtRowTile;

  // device state
  void* kc = nullptr;
  void* vc = nullptr;
  float* scores = nullptr;
  int32_t* pos = nullptr;
  // fixed-point summed weights, [B * Hkv][acc_stride] (cleared by the tail each
  // step, so zero between steps); acc_stride = 2 M rounded up to a multiple of
  // 4 holds the M slots and up to M chunk keys
  unsigned long long* colacc = nullptr;
  int64_t acc_stride = 0;
  // device error word: mapped pinned host memory, so kernels report into it
  // directly and no copy is enqueued per step; nonzero only after an error
  int* err = nullptr;
  DevBuf newscore, freed, evicted;
  // stream-partitioned attention: per-piece row statistics, partial O, unit counters
  DevBuf ws_ml, ws_o, ws_count;
  int n_sm = 0;
  // staging for host pointers
  // Host inputs are copied on a stream of the handle's own into one of two
  // staging sets, so the next step's copies overlap this step's kernels: set
  // s is filled once the kernels of the step that last read it are done
  // (ev_free[s]), and the caller's stream waits for its copies (ev_in[s]).
  DevBuf st_q[2], st_k[2], st_v[2], st_out;
  cudaStream_t copy_st = nullptr;
  cudaEvent_t ev_in[2] = {}, ev_free[2] = {};
  // grouped steps led by this handle with host outputs: the layers run in
  // sub-groups of kOutLayers, and each sub-group's outputs are copied to the
  // host on d2h_st while the next sub-group computes (ev_sub: re-recorded after
  // each sub-group's kernels; ev_d2h: every copy is done, waited for by the
  // caller's stream)
  static constexpr int kOutLayers = 4;
  cudaStream_t d2h_st = nullptr;
  cudaEvent_t ev_sub = nullptr, ev_d2h = nullptr;
  bool st_used[2] = {false, false};
  int st_set = 0;
  cudaEvent_t err_ev = nullptr;   // recorded after each step
  bool err_pending = false;

  // fused tail: cluster size for (M, tail_S), 0 = use the three separate kernels
  int64_t tail_S = -1;
  int tail_cs = 0;
  // the same for grouped steps led by this handle: (S, caches) it was chosen for
  int64_t grp_tail_S = -1;
  int grp_tail_n = 0, grp_tail_cs = 0;

  // per-kernel timing: a ring of event sets (start, after attention, after the
  // tail), one set per profiled step
  static constexpr int kProfRing = 64;
  bool prof = false;
  cudaEvent_t ev[kProfRing][3] = {};
  int64_t prof_steps = 0;   // profiled steps recorded so far

  std::string msg = "no error";
};

namespace {

int fail(h2o_ctx* h, int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  if (h) h->msg = buf;
  g_thread_err = buf;
  return code;
}

int cuda_fail(h2o_ctx* h, cudaError_t e, const char* what) {
  const int code = (e == cudaErrorMemoryAllocation) ? H2O_ENOMEM : H2O_ECUDA;
  return fail(h, code, "%s: %s", what, cudaGetErrorString(e));
}

#define H2O_CUDA(h, call, what)                      \
  do {                                               \
    cudaError_t e_ = (call);                         \
    if (e_ != cudaSuccess) return cuda_fail(h, e_, what); \
  } while (0)

bool fault_injected(const char* kind) {
  const char* f = getenv("H2O_FAULT");
  return f && strcmp(f, kind) == 0;
}

cudaError_t dev_alloc(void** p, size_t bytes) {
  if (fault_injected("alloc")) return cudaErrorMemoryAllocation;
  return cudaMalloc(p, bytes);
}

// Grow a scratch buffer (contents are not preserved).
cudaError_t ensure(DevBuf& b, size_t bytes) {
  if (b.cap >= bytes) return cudaSuccess;
  if (b.p) {
    cudaError_t e = cudaFree(b.p);
    b.p = nullptr;
    b.cap = 0;
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = dev_alloc(&b.p, bytes);
  if (e == cudaSuccess) b.cap = bytes;
  return e;
}

bool is_device_ptr(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

// H2O_SPLIT_TAIL=1 runs score accumulation, selection and scatter as three
// kernels instead of the fused cluster kernel (same results).
bool split_tail() {
  const char* s = getenv("H2O_SPLIT_TAIL");
  return s && s[0] == '1';
}

// H2O_ATTN_SPLIT=k asks the tensor-core attention kernel to split each unit of
// work over k CTAs (a cluster; capped by the sizes); unset, it chooses.
int attn_split() {
  const char* s = getenv("H2O_ATTN_SPLIT");
  return s ? atoi(s) : 0;
}

// H2O_ATTN_MODE=fused / stream forces one of the two tensor-core attention
// paths (one kernel with both sweeps / two kernels over equal runs of key
// pairs); unset, the choice below is made per launch.
int attn_mode() {
  const char* s = getenv("H2O_ATTN_MODE");
  if (!s) return 0;
  if (strcmp(s, "fused") == 0) return 1;
  if (strcmp(s, "stream") == 0) return 2;
  return 0;
}

// H2O_INJECT_TIMEOUT=1 (test hook): in the tensor-core attention kernel (the
// one-kernel path, or with H2O_ATTN_MODE=stream the second stream kernel) one
// softmax warpgroup waits on a barrier that nothing completes, with a 1 ms
// limit; the step then fails with H2O_ETIMEOUT and the context stays usable.
bool inject_timeout() {
  const char* s = getenv("H2O_INJECT_TIMEOUT");
  return s && s[0] == '1';
}

bool sync_check_enabled() {
  const char* s = getenv("H2O_SYNC_CHECK");
  return s && s[0] == '1';
}

// Reads the device error word of a finished step; returns a status.
int check_device_error(h2o_ctx* h, bool wait) {
  if (!h->err_pending) return H2O_OK;
  if (wait) {
    cudaError_t e = cudaEventSynchronize(h->err_ev);
    if (e != cudaSuccess) return cuda_fail(h, e, "kernel execution");
  } else {
    cudaError_t e = cudaEventQuery(h->err_ev);
    if (e == cudaErrorNotReady) return H2O_OK;
    if (e != cudaSuccess) return cuda_fail(h, e, "kernel execution");
  }
  h->err_pending = false;
  const int w = *static_cast<volatile int*>(h->err);
  if (w == 0) return H2O_OK;
  // report once: clear the word so the handle's next step starts clean
  *static_cast<volatile int*>(h->err) = 0;
  if (w & h2o::kErrTimeout)
    return fail(h, H2O_ETIMEOUT, "a bounded in-kernel wait timed out (device error word 0x%x)", w);
  if (w & h2o::kErrSelect)
    return fail(h, H2O_ESHAPE, "fewer evictable slots than needed (device error word 0x%x)", w);
  return fail(h, H2O_ECUDA, "device-side check failed (device error word 0x%x)", w);
}

size_t elem_size(int dtype) { return dtype == H2O_F32 ? 4 : 2; }

// One handle's chunk step between its phases: what prepare_chunk decided and
// staged, what the launches and finish_chunk use.
struct ChunkRun {
  h2o_ctx* h = nullptr;
  int64_t S = 0, need = 0;
  size_t q_bytes = 0;
  const void* dq = nullptr;
  const void* dk = nullptr;
  const void* dv = nullptr;
  void* dout = nullptr;
  void* out = nullptr;          // the caller's output (host memory when hout)
  bool hout = false, host_in = false;
  bool out_copied = false;      // the host output's copy was enqueued by run_layers
  bool decode = false, stream = false;
  int fx_shift = 0;
  h2o::StreamPlan pl;
  h2o::AttnArgs a;
  int launches = 0;
};

// Checks, host-pointer staging, the attention path and the scratch of one
// chunk of S tokens (prefill when the cache is empty).  Enqueues only copies.
int prepare_chunk(h2o_ctx* h, const void* q, const void* k, const void* v, void* out, int64_t S,
                  cudaStream_t st, ChunkRun* r) {
  const int BH = h->B * h->Hkv;
  const size_t es = elem_size(h->dtype);
  const size_t q_bytes = (size_t)h->B * h->Hq * S * h->d * es;
  const size_t kv_bytes = (size_t)BH * S * h->d * es;

  int rc = check_device_error(h, sync_check_enabled());
  if (rc != H2O_OK) return rc;

  // token positions are stored as int32
  if (h->t0 + S > (int64_t)INT32_MAX)
    return fail(h, H2O_ESHAPE, "the stream would pass 2^31 - 1 tokens (t0=%lld, S=%lld)",
                (long long)h->t0, (long long)S);

  // need and eligibility are fixed by the bookkeeping: the min(R, t0) most
  // recent tokens are always cached and protected, the rest of the valid slots
  // are evictable.
  const int64_t empties = h->M - h->n_valid;
  const int64_t need = S > empties ? S - empties : 0;
  const int64_t protect = h->R < h->t0 ? h->R : h->t0;
  const int64_t eligible = h->n_valid - (protect < h->n_valid ? protect : h->n_valid);
  if (need > eligible)
    return fail(h, H2O_ESHAPE, "chunk of %lld tokens needs %lld evictions but only %lld slots are "
                "older than the recent window", (long long)S, (long long)need, (long long)eligible);

  // host-pointer staging
  const void* dq = q;
  const void* dk = k;
  const void* dv = v;
  void* dout = out;
  const bool hq = !is_device_ptr(q), hk = !is_device_ptr(k), hv = !is_device_ptr(v);
  const bool hout = out && !is_device_ptr(out);
  const int set = h->st_set;
  if (hq || hk || hv) {
    if (!h->copy_st) {
      H2O_CUDA(h, cudaStreamCreateWithFlags(&h->copy_st, cudaStreamNonBlocking), "copy stream");
      for (int i = 0; i < 2; ++i) {
        H2O_CUDA(h, cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming), "event");
        H2O_CUDA(h, cudaEventCreateWithFlags(&h->ev_free[i], cudaEventDisableTiming), "event");
      }
    }
    // the step that last read this staging set must be done with it
    if (h->st_used[set]) H2O_CUDA(h, cudaStreamWaitEvent(h->copy_st, h->ev_free[set], 0), "event wait");
    if (hq) {
      H2O_CUDA(h, ensure(h->st_q[set], q_bytes), "staging alloc");
      H2O_CUDA(h, cudaMemcpyAsync(h->st_q[set].p, q, q_bytes, cudaMemcpyDefault, h->copy_st), "copy q");
      dq = h->st_q[set].p;
    }
    if (hk) {
      H2O_CUDA(h, ensure(h->st_k[set], kv_bytes), "staging alloc");
      H2O_CUDA(h, cudaMemcpyAsync(h->st_k[set].p, k, kv_bytes, cudaMemcpyDefault, h->copy_st), "copy k");
      dk = h->st_k[set].p;
    }
    if (hv) {
      H2O_CUDA(h, ensure(h->st_v[set], kv_bytes), "staging alloc");
      H2O_CUDA(h, cudaMemcpyAsync(h->st_v[set].p, v, kv_bytes, cudaMemcpyDefault, h->copy_st), "copy v");
      dv = h->st_v[set].p;
    }
    H2O_CUDA(h, cudaEventRecord(h->ev_in[set], h->copy_st), "event");
    H2O_CUDA(h, cudaStreamWaitEvent(st, h->ev_in[set], 0), "event wait");
  }
  if (hout) {
    H2O_CUDA(h, ensure(h->st_out, q_bytes), "staging alloc");
    dout = h->st_out.p;
  }

  // chunks of a few tokens (G * S <= 16 rows per KV head, and a cache whose
  // scores fit the decode kernel's shared memory) take the decode kernel;
  // forcing a tensor-core path (H2O_ATTN_MODE) bypasses it
  const bool decode = h2o::decode_supported(h->G, S, h->n_valid + S) && attn_mode() == 0;
  const int fx_shift = h2o::colsum_shift(S, h->G);

  h2o::AttnArgs& a = r->a;
  a.q = dq;
  a.k = dk;
  a.v = dv;
  a.out = dout;
  a.kc = h->kc;
  a.vc = h->vc;
  a.colacc = h->colacc;
  a.err = h->err;
  a.B = h->B;
  a.Hq = h->Hq;
  a.Hkv = h->Hkv;
  a.d = h->d;
  a.S = S;
  a.M = h->M;
  a.n_valid = h->n_valid;
  a.acc_stride = h->acc_stride;
  a.fx_shift = fx_shift;
  a.split = attn_split();
  a.inject_timeout = inject_timeout() ? 1 : 0;
  a.scale = (float)(1.0 / std::sqrt((double)h->d));

  // tensor-core path: one kernel with both sweeps, or two kernels over a
  // balanced partition of the key pairs ("stream").  Automatic: the partition
  // pays when the one-kernel grid would leave SMs idle (n_sm / 2 .. 2 n_sm
  // units) and units are long enough (>= 24 pairs on average) for a piece
  // boundary's Q reload and epilogue.
  bool stream = false;
  if (!decode && h->use_umma) {
    if (h->n_sm == 0) H2O_CUDA(h, cudaDeviceGetAttribute(&h->n_sm, cudaDevAttrMultiProcessorCount, h->device),
                               "device attribute");
    const int mode = attn_mode();
    if (mode != 1 && (!a.inject_timeout || mode == 2) && h2o::attn_stream_plan(a, h->n_sm, &r->pl))
      stream = mode == 2 || (2 * r->pl.units >= h->n_sm && r->pl.units <= 2 * h->n_sm &&
                             r->pl.total_pairs >= 24 * (int64_t)r->pl.units);
  }
  H2O_CUDA(h, ensure(h->freed, (size_t)BH * S * sizeof(int32_t)), "scratch alloc");
  H2O_CUDA(h, ensure(h->evicted, (size_t)BH * S * sizeof(int32_t)), "scratch alloc");
  if (stream) {
    H2O_CUDA(h, ensure(h->ws_ml, r->pl.ml_bytes), "scratch alloc");
    if (r->pl.o_bytes) H2O_CUDA(h, ensure(h->ws_o, r->pl.o_bytes), "scratch alloc");
    H2O_CUDA(h, ensure(h->ws_count, r->pl.count_bytes), "scratch alloc");
  }
  if (S != h->tail_S) {
    h->tail_cs = split_tail() ? 0 : h2o::tail_cluster_size(h->M, S, BH);
    h->tail_S = S;
  }
  if (h->tail_cs == 0) H2O_CUDA(h, ensure(h->newscore, (size_t)BH * S * sizeof(float)), "scratch alloc");

  r->h = h;
  r->S = S;
  r->need = need;
  r->q_bytes = q_bytes;
  r->dq = dq;
  r->dk = dk;
  r->dv = dv;
  r->dout = dout;
  r->out = out;
  r->hout = hout;
  r->host_in = hq || hk || hv;
  r->decode = decode;
  r->stream = stream;
  r->fx_shift = fx_shift;
  r->launches = 0;
  return H2O_OK;
}

// The attention launch(es) of one prepared chunk.
int launch_attention(ChunkRun& r, cudaStream_t st) {
  h2o_ctx* h = r.h;
  const int BH = h->B * h->Hkv;
  if (fault_injected("launch")) return fail(h, H2O_ECUDA, "injected launch failure");
  cudaError_t e = cudaSuccess;
  if (r.decode) {
    h2o::DecodeArgs da;
    da.q = r.dq;
    da.k = r.dk;
    da.v = r.dv;
    da.out = r.dout;
    da.kcache = h->kc;
    da.vcache = h->vc;
    da.colacc = h->colacc;
    da.err = h->err;
    da.B = h->B;
    da.Hq = h->Hq;
    da.Hkv = h->Hkv;
    da.G = h->G;
    da.d = h->d;
    da.S = r.S;
    da.M = h->M;
    da.n_valid = h->n_valid;
    da.acc_stride = h->acc_stride;
    da.scale_log2 = r.a.scale * 1.4426950408889634f;
    da.fx_scale = h2o::fx_scale_of(r.fx_shift);
    e = h2o::launch_decode(da, h->dtype, BH, true, st);
    r.launches += 1;
  } else if (h->use_umma) {
    if (r.stream) {
      e = h2o::launch_attn_stream(r.a, r.pl, h->ws_ml.p, h->ws_o.p, static_cast<int*>(h->ws_count.p),
                                  true, st);
      r.launches += 2;
    } else {
      e = h2o::launch_attn_umma(r.a, true, st);
      r.launches += 1;
    }
  } else {
    e = h2o::launch_attn_simt(r.a, h->dtype, true, st);
    r.launches += 1;
  }
  if (e != cudaSuccess) return cuda_fail(h, e, "attention launch");
  return H2O_OK;
}

h2o::TailArgs tail_args(const ChunkRun& r) {
  const h2o_ctx* h = r.h;
  h2o::TailArgs t;
  t.colacc = h->colacc;
  t.scores = h->scores;
  t.pos = h->pos;
  t.k = static_cast<const uint4*>(r.dk);
  t.v = static_cast<const uint4*>(r.dv);
  t.kc = static_cast<uint4*>(h->kc);
  t.vc = static_cast<uint4*>(h->vc);
  t.freed = static_cast<int32_t*>(h->freed.p);
  t.evicted = static_cast<int32_t*>(h->evicted.p);
  t.err = h->err;
  t.M = h->M;
  t.S = r.S;
  t.n_valid = h->n_valid;
  t.t0 = h->t0;
  t.R = h->R;
  t.need = r.need;
  t.acc_stride = h->acc_stride;
  t.fx_inv = h2o::fx_inv_of(r.fx_shift);
  t.recency = h->policy == H2O_POLICY_LR ? 1 : 0;
  t.row_vecs = (int)(h->d * elem_size(h->dtype) / 16);
  t.per = t.per_s = 0;
  return t;
}

// Score accumulate + select + scatter of one prepared chunk.
int launch_tail(ChunkRun& r, cudaStream_t st) {
  h2o_ctx* h = r.h;
  const int BH = h->B * h->Hkv;
  cudaError_t e = cudaSuccess;
  if (h->tail_cs > 0) {
    e = h2o::launch_tail(tail_args(r), BH, h->tail_cs, true, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "tail launch");
    r.launches += 1;
  } else {
    e = h2o::launch_score_reduce(h->colacc, h->acc_stride, h2o::fx_inv_of(r.fx_shift), h->scores,
                                 static_cast<float*>(h->newscore.p), BH, r.S, h->M, h->n_valid, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "score reduce launch");
    e = h2o::launch_select(h->scores, h->pos, BH, h->M, h->t0, h->R, r.need, h->n_valid, r.S,
                           static_cast<int32_t*>(h->freed.p), r.S, h->err, st,
                           h->policy == H2O_POLICY_LR ? 1 : 0);
    if (e != cudaSuccess) return cuda_fail(h, e, "select launch");
    e = h2o::launch_scatter(r.dk, r.dv, h->kc, h->vc, h->scores, h->pos,
                            static_cast<int32_t*>(h->freed.p), static_cast<float*>(h->newscore.p),
                            static_cast<int32_t*>(h->evicted.p), BH, r.S, h->M, h->d,
                            (int)elem_size(h->dtype), h->t0, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "scatter launch");
    r.launches += 3;
  }
  return H2O_OK;
}

// After the launches: the output copy for host buffers, the staging set's
// release, the error event, the counters; with H2O_SYNC_CHECK=1 the step's own
// device error is waited for and reported.
int finish_chunk(ChunkRun& r, cudaStream_t st) {
  h2o_ctx* h = r.h;
  if (r.host_in) {
    const int set = h->st_set;
    H2O_CUDA(h, cudaEventRecord(h->ev_free[set], st), "event");
    h->st_used[set] = true;
    h->st_set = set ^ 1;
  }
  if (r.hout && !r.out_copied)
    H2O_CUDA(h, cudaMemcpyAsync(r.out, r.dout, r.q_bytes, cudaMemcpyDefault, st), "copy out");
  // the error word is read once this event has completed (by the next call)
  H2O_CUDA(h, cudaEventRecord(h->err_ev, st), "event");
  h->err_pending = true;
  h->t0 += r.S;
  h->n_valid = h->n_valid + r.S < h->M ? h->n_valid + r.S : h->M;
  h->last_S = r.S;
  h->last_launches = r.launches;
  if (sync_check_enabled()) return check_device_error(h, true);
  return H2O_OK;
}

// Runs one chunk of S tokens (prefill when the cache is empty).
int run_chunk(h2o_ctx* h, const void* q, const void* k, const void* v, void* out, int64_t S,
              cudaStream_t st) {
  ChunkRun r;
  int rc = prepare_chunk(h, q, k, v, out, S, st, &r);
  if (rc != H2O_OK) return rc;
  cudaEvent_t* evs = h->ev[h->prof_steps % h2o_ctx::kProfRing];
  if (h->prof) H2O_CUDA(h, cudaEventRecord(evs[0], st), "event");
  if ((rc = launch_attention(r, st)) != H2O_OK) return rc;
  if (h->prof) H2O_CUDA(h, cudaEventRecord(evs[1], st), "event");
  if ((rc = launch_tail(r, st)) != H2O_OK) return rc;
  if (h->prof) {
    H2O_CUDA(h, cudaEventRecord(evs[2], st), "event");
    ++h->prof_steps;
  }
  return finish_chunk(r, st);
}

// Several layers' chunk steps.  Layers of identical sizes on the one-kernel
// tensor-core path share one attention grid and one tail grid (in groups of up
// to the kernels' maximum); any other layer runs its own step.
int run_layers(h2o_ctx** hs, int n, const void* const* q, const void* const* k,
               const void* const* v, void* const* out, int64_t S, cudaStream_t st) {
  std::vector<ChunkRun> runs((size_t)n);
  for (int l = 0; l < n; ++l) {
    int rc = prepare_chunk(hs[l], q[l], k[l], v[l], out ? out[l] : nullptr, S, st, &runs[(size_t)l]);
    if (rc != H2O_OK) {
      // the layers before l are staged but not launched: nothing changed yet
      if (l > 0) fail(hs[0], rc, "layer %d: %s", l, hs[l]->msg.c_str());
      return rc;
    }
  }
  h2o_ctx* h0 = hs[0];
  auto groupable = [&](const ChunkRun& r) {
    const h2o_ctx* h = r.h;
    return h->use_umma && !r.decode && !r.stream && h->tail_cs > 0 && h->device == h0->device &&
           h->B == h0->B && h->Hq == h0->Hq && h->Hkv == h0->Hkv && h->d == h0->d &&
           h->M == h0->M && h->R == h0->R && h->t0 == h0->t0 && h->n_valid == h0->n_valid &&
           h->tail_cs == h0->tail_cs && h->policy == h0->policy && r.a.split == runs[0].a.split &&
           r.a.inject_timeout == runs[0].a.inject_timeout;
  };
  bool all = true;
  for (int l = 0; l < n; ++l) all = all && groupable(runs[(size_t)l]);
  cudaEvent_t* evs = h0->ev[h0->prof_steps % h2o_ctx::kProfRing];
  const bool prof = h0->prof;
  if (prof) H2O_CUDA(h0, cudaEventRecord(evs[0], st), "event");
  int rc = H2O_OK;
  if (!all) {
    // layer after layer, each with its own launches
    for (int l = 0; l < n && rc == H2O_OK; ++l) rc = launch_attention(runs[(size_t)l], st);
    if (prof && rc == H2O_OK) H2O_CUDA(h0, cudaEventRecord(evs[1], st), "event");
    for (int l = 0; l < n && rc == H2O_OK; ++l) rc = launch_tail(runs[(size_t)l], st);
  } else {
    if (fault_injected("launch")) return fail(h0, H2O_ECUDA, "injected launch failure");
    const int BH = h0->B * h0->Hkv;
    const int ga = h2o::attn_umma_max_group(), gt = h2o::tail_max_group();
    std::vector<h2o::AttnArgs> aa((size_t)n);
    std::vector<h2o::TailArgs> ta((size_t)n);
    for (int l = 0; l < n; ++l) {
      aa[(size_t)l] = runs[(size_t)l].a;
      ta[(size_t)l] = tail_args(runs[(size_t)l]);
    }
    // With host outputs (and no per-kernel profiling, whose events need one
    // attention and one tail stretch) the layers run in sub-groups of
    // kOutLayers consecutive layers, each its attention then its tail
    // launches, and each sub-group's outputs go to the host on d2h_st while
    // the later sub-groups compute; the caller's stream then waits for the
    // copies, so the outputs are in host memory once it has passed the step.
    bool any_hout = false;
    for (int l = 0; l < n; ++l) any_hout = any_hout || runs[(size_t)l].hout;
    const int per_sub = (any_hout && !prof && n >= 2 * h2o_ctx::kOutLayers) ? h2o_ctx::kOutLayers : n;
    const int n_sub = (n + per_sub - 1) / per_sub;
    if (n_sub > 1 && !h0->d2h_st) {
      H2O_CUDA(h0, cudaStreamCreateWithFlags(&h0->d2h_st, cudaStreamNonBlocking), "copy stream");
      H2O_CUDA(h0, cudaEventCreateWithFlags(&h0->ev_sub, cudaEventDisableTiming), "event");
      H2O_CUDA(h0, cudaEventCreateWithFlags(&h0->ev_d2h, cudaEventDisableTiming), "event");
    }
    // the tail's cluster size for grouped launches of per_sub layers
    if (h0->grp_tail_S != S || h0->grp_tail_n != per_sub) {
      const int m = per_sub < gt ? per_sub : gt;
      h0->grp_tail_cs = m > 1 ? h2o::tail_cluster_size(h0->M, S, m * BH, true) : h0->tail_cs;
      h0->grp_tail_S = S;
      h0->grp_tail_n = per_sub;
    }
    for (int g = 0; g < n_sub; ++g) {
      const int s0 = g * per_sub, s1 = s0 + per_sub < n ? s0 + per_sub : n;
      if (s0 >= s1) break;
      for (int l0 = s0; l0 < s1; l0 += ga) {
        const int m = s1 - l0 < ga ? s1 - l0 : ga;
        cudaError_t e = h2o::launch_attn_umma_group(aa.data() + l0, m, true, st);
        if (e != cudaSuccess) return cuda_fail(h0, e, "grouped attention launch");
        runs[(size_t)l0].launches += 1;
      }
      if (prof) H2O_CUDA(h0, cudaEventRecord(evs[1], st), "event");
      for (int l0 = s0; l0 < s1; l0 += gt) {
        const int m = s1 - l0 < gt ? s1 - l0 : gt;
        const int cs = m > 1 ? h0->grp_tail_cs : h0->tail_cs;
        if (cs < 1) return fail(h0, H2O_ECUDA, "grouped tail: no cluster size fits");
        cudaError_t e = h2o::launch_tail_group(ta.data() + l0, m, BH, cs, true, st);
        if (e != cudaSuccess) return cuda_fail(h0, e, "grouped tail launch");
        runs[(size_t)l0].launches += 1;
      }
      if (n_sub > 1) {
        // (the wait takes the event's latest record: one event serves every sub-group)
        H2O_CUDA(h0, cudaEventRecord(h0->ev_sub, st), "event");
        H2O_CUDA(h0, cudaStreamWaitEvent(h0->d2h_st, h0->ev_sub, 0), "event wait");
        for (int l = s0; l < s1; ++l) {
          ChunkRun& r = runs[(size_t)l];
          if (!r.hout) continue;
          H2O_CUDA(h0, cudaMemcpyAsync(r.out, r.dout, r.q_bytes, cudaMemcpyDefault, h0->d2h_st), "copy out");
          r.out_copied = true;
        }
      }
    }
    if (n_sub > 1) {
      H2O_CUDA(h0, cudaEventRecord(h0->ev_d2h, h0->d2h_st), "event");
      H2O_CUDA(h0, cudaStreamWaitEvent(st, h0->ev_d2h, 0), "event wait");
    }
  }
  if (rc != H2O_OK) return rc;
  if (prof) {
    H2O_CUDA(h0, cudaEventRecord(evs[2], st), "event");
    ++h0->prof_steps;
  }
  for (int l = 0; l < n; ++l) {
    const int r2 = finish_chunk(runs[(size_t)l], st);
    if (r2 != H2O_OK && rc == H2O_OK) rc = r2;
  }
  return rc;
}

// Frees the per-handle device state (cache, scores, positions, error word,
// events); pointers are reset so the handle can be destroyed or prefilled again.
void release_state(h2o_ctx* h) {
  cudaFree(h->kc);
  cudaFree(h->vc);
  cudaFree(h->scores);
  cudaFree(h->pos);
  cudaFree(h->colacc);
  if (h->err) cudaFreeHost(h->err);
  if (h->err_ev) cudaEventDestroy(h->err_ev);
  for (auto& set : h->ev)
    for (auto& ev : set) {
      if (ev) cudaEventDestroy(ev);
      ev = nullptr;
    }
  h->kc = h->vc = nullptr;
  h->scores = nullptr;
  h->pos = nullptr;
  h->colacc = nullptr;
  h->err = nullptr;
  h->err_ev = nullptr;
  h->device = -1;
  cudaGetLastError();
}

int alloc_state_impl(h2o_ctx* h, int B) {
  const size_t es = elem_size(h->dtype);
  const size_t slots = (size_t)B * h->Hkv * h->M;
  // the cache first: an injected allocation failure (H2O_FAULT=alloc) is
  // reported before any other CUDA call
  H2O_CUDA(h, dev_alloc(&h->kc, slots * h->d * es), "cache alloc");
  H2O_CUDA(h, cudaGetDevice(&h->device), "cudaGetDevice");
  H2O_CUDA(h, dev_alloc(&h->vc, slots * h->d * es), "cache alloc");
  H2O_CUDA(h, dev_alloc((void**)&h->scores, slots * sizeof(float)), "state alloc");
  H2O_CUDA(h, dev_alloc((void**)&h->pos, slots * sizeof(int32_t)), "state alloc");
  h->acc_stride = (2 * h->M + 3) & ~(int64_t)3;
  const size_t acc_bytes = (size_t)B * h->Hkv * h->acc_stride * sizeof(unsigned long long);
  H2O_CUDA(h, dev_alloc((void**)&h->colacc, acc_bytes), "state alloc");
  {
    void* hp = nullptr;
    H2O_CUDA(h, cudaHostAlloc(&hp, sizeof(int), cudaHostAllocMapped), "pinned alloc");
    h->err = static_cast<int*>(hp);
    *h->err = 0;
  }
  H2O_CUDA(h, cudaMemset(h->kc, 0, slots * h->d * es), "memset");
  H2O_CUDA(h, cudaMemset(h->vc, 0, slots * h->d * es), "memset");
  H2O_CUDA(h, cudaMemset(h->scores, 0, slots * sizeof(float)), "memset");
  H2O_CUDA(h, cudaMemset(h->pos, 0xFF, slots * sizeof(int32_t)), "memset");
  H2O_CUDA(h, cudaMemset(h->colacc, 0, acc_bytes), "memset");
  H2O_CUDA(h, cudaEventCreateWithFlags(&h->err_ev, cudaEventDisableTiming), "event");
  for (auto& set : h->ev)
    for (auto& ev : set) H2O_CUDA(h, cudaEventCreate(&ev), "event");
  H2O_CUDA(h, cudaDeviceSynchronize(), "state init");
  h->B = B;
  return H2O_OK;
}

// On failure nothing stays allocated: the handle is as before the call.
int alloc_state(h2o_ctx* h, int B) {
  const int rc = alloc_state_impl(h, B);
  if (rc != H2O_OK) release_state(h);
  return rc;
}

}  // namespace

extern "C" {

int h2o_create(int64_t M, int64_t R, int Hq, int Hkv, int d, int dtype, h2o_t* out) {
  return h2o_create_policy(M, R, Hq, Hkv, d, dtype, H2O_POLICY_H2O, out);
}

int h2o_create_policy(int64_t M, int64_t R, int Hq, int Hkv, int d, int dtype, int policy,
                      h2o_t* out) {
  if (!out) return fail(nullptr, H2O_EINVAL, "h2o_create: out is NULL");
  if (policy != H2O_POLICY_H2O && policy != H2O_POLICY_LR) {
    *out = nullptr;
    return fail(nullptr, H2O_EINVAL, "h2o_create: unknown policy %d", policy);
  }
  *out = nullptr;
  if (M < 1 || R < 0 || R >= M)
    return fail(nullptr, H2O_EINVAL, "h2o_create: need M >= 1 and 0 <= R < M (M=%lld R=%lld)",
                (long long)M, (long long)R);
  if (M > (int64_t)1 << 30)
    return fail(nullptr, H2O_EINVAL, "h2o_create: M=%lld too large", (long long)M);
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
    return fail(nullptr, H2O_EINVAL, "h2o_create: need Hq %% Hkv == 0 (Hq=%d Hkv=%d)", Hq, Hkv);
  if (d != 64 && d != 128) return fail(nullptr, H2O_EINVAL, "h2o_create: d must be 64 or 128 (d=%d)", d);
  if (dtype != H2O_F32 && dtype != H2O_BF16)
    return fail(nullptr, H2O_EINVAL, "h2o_create: dtype must be H2O_F32 or H2O_BF16");
  h2o_ctx* h = new (std::nothrow) h2o_ctx();
  if (!h) return fail(nullptr, H2O_ENOMEM, "h2o_create: out of host memory");
  h->M = M;
  h->R = R;
  h->Hq = Hq;
  h->Hkv = Hkv;
  h->G = Hq / Hkv;
  h->d = d;
  h->dtype = dtype;
  h->policy = policy;
  h->esize = (int)elem_size(dtype);
  h->use_umma = h2o::attn_umma_supported(dtype, d);
  h->row_tile = h->use_umma ? h2o::kUmmaRowTile : h2o::kSimtRowTile;
  *out = h;
  return H2O_OK;
}

int h2o_prefill(h2o_t h, const void* q, const void* k, const void* v, void* out, int B, int64_t P,
                void* stream) {
  if (!h) return fail(nullptr, H2O_EINVAL, "h2o_prefill: NULL handle");
  if (h->prefilled) return fail(h, H2O_ESTATE, "h2o_prefill: handle already prefilled");
  if (!q || !k || !v) return fail(h, H2O_EINVAL, "h2o_prefill: q, k and v must not be NULL");
  if (B < 1 || P < 1) return fail(h, H2O_EINVAL, "h2o_prefill: need B >= 1 and P >= 1");
  if (P > h->M)
    return fail(h, H2O_ESHAPE, "h2o_prefill: P=%lld exceeds the cache capacity M=%lld",
                (long long)P, (long long)h->M);
  int rc = alloc_state(h, B);
  if (rc != H2O_OK) return rc;
  h->prefilled = true;
  return run_chunk(h, q, k, v, out, P, static_cast<cudaStream_t>(stream));
}

int h2o_step(h2o_t h, const void* q, const void* k, const void* v, void* out, int64_t S,
             void* stream) {
  if (!h) return fail(nullptr, H2O_EINVAL, "h2o_step: NULL handle");
  if (!h->prefilled) return fail(h, H2O_ESTATE, "h2o_step: called before h2o_prefill");
  if (!q || !k || !v) return fail(h, H2O_EINVAL, "h2o_step: q, k and v must not be NULL");
  if (S < 1) return fail(h, H2O_EINVAL, "h2o_step: need S >= 1");
  if (S > h->M)
    return fail(h, H2O_ESHAPE, "h2o_step: S=%lld exceeds the cache capacity M=%lld",
                (long long)S, (long long)h->M);
  return run_chunk(h, q, k, v, out, S, static_cast<cudaStream_t>(stream));
}

int h2o_step_layers(h2o_t* hs, int n, const void* const* q, const void* const* k,
                    const void* const* v, void* const* out, int64_t S, void* stream) {
  if (!hs || n < 1) return fail(nullptr, H2O_EINVAL, "h2o_step_layers: need n >= 1 handles");
  if (!q || !k || !v) return fail(nullptr, H2O_EINVAL, "h2o_step_layers: q, k and v arrays must not be NULL");
  for (int l = 0; l < n; ++l) {
    h2o_ctx* h = hs[l];
    if (!h) return fail(nullptr, H2O_EINVAL, "h2o_step_layers: handle %d is NULL", l);
    for (int j = 0; j < l; ++j)
      if (hs[j] == h) return fail(h, H2O_EINVAL, "h2o_step_layers: handle %d repeats handle %d", l, j);
    if (!h->prefilled) return fail(h, H2O_ESTATE, "h2o_step_layers: handle %d not prefilled", l);
    if (!q[l] || !k[l] || !v[l])
      return fail(h, H2O_EINVAL, "h2o_step_layers: q, k and v of layer %d must not be NULL", l);
    if (S < 1) return fail(h, H2O_EINVAL, "h2o_step_layers: need S >= 1");
    if (S > h->M)
      return fail(h, H2O_ESHAPE, "h2o_step_layers: S=%lld exceeds the cache capacity M=%lld of layer %d",
                  (long long)S, (long long)h->M, l);
  }
  return run_layers(hs, n, q, k, v, out, S, static_cast<cudaStream_t>(stream));
}

int h2o_read_state(h2o_t h, int32_t* slots, float* scores, int32_t* positions, void* stream) {
  if (!h) return fail(nullptr, H2O_EINVAL, "h2o_read_state: NULL handle");
  if (!h->prefilled) return fail(h, H2O_ESTATE, "h2o_read_state: called before h2o_prefill");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t slots_n = (size_t)h->B * h->Hkv * h->M;
  if (slots)
    H2O_CUDA(h, cudaMemcpyAsync(slots, h->freed.p, (size_t)h->B * h->Hkv * h->last_S * sizeof(int32_t),
                                cudaMemcpyDefault, st), "copy slots");
  if (scores)
    H2O_CUDA(h, cudaMemcpyAsync(scores, h->scores, slots_n * sizeof(float), cudaMemcpyDefault, st),
             "copy scores");
  if (positions)
    H2O_CUDA(h, cudaMemcpyAsync(positions, h->pos, slots_n * sizeof(int32_t), cudaMemcpyDefault, st),
             "copy positions");
  if ((slots && !is_device_ptr(slots)) || (scores && !is_device_ptr(scores)) ||
      (positions && !is_device_ptr(positions))) {
    H2O_CUDA(h, cudaStreamSynchronize(st), "read_state sync");
    return check_device_error(h, true);
  }
  return check_device_error(h, false);
}

int h2o_read_delta(h2o_t h, int32_t* slots, int32_t* evicted_positions, void* stream) {
  if (!h) return fail(nullptr, H2O_EINVAL, "h2o_read_delta: NULL handle");
  if (!h->prefilled) return fail(h, H2O_ESTATE, "h2o_read_delta: called before h2o_prefill");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)h->B * h->Hkv * h->last_S * sizeof(int32_t);
  if (slots) H2O_CUDA(h, cudaMemcpyAsync(slots, h->freed.p, bytes, cudaMemcpyDefault, st), "copy slots");
  if (evicted_positions)
    H2O_CUDA(h, cudaMemcpyAsync(evicted_positions, h->evicted.p, bytes, cudaMemcpyDefault, st),
             "copy evicted positions");
  if ((slots && !is_device_ptr(slots)) || (evicted_positions && !is_device_ptr(evicted_positions))) {
    H2O_CUDA(h, cudaStreamSynchronize(st), "read_delta sync");
    return check_device_error(h, true);
  }
  return check_device_error(h, false);
}

int h2o_read_kv(h2o_t h, void* k_cache, void* v_cache, void* stream) {
  if (!h) return fail(nullptr, H2O_EINVAL, "h2o_read_kv: NULL handle");
  if (!h->prefilled) return fail(h, H2O_ESTATE, "h2o_read_kv: called before h2o_prefill");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)h->B * h->Hkv * h->M * h->d * h->esize;
  if (k_cache) H2O_CUDA(h, cudaMemcpyAsync(k_cache, h->kc, bytes, cudaMemcpyDefault, st), "copy k");
  if (v_cache) H2O_CUDA(h, cudaMemcpyAsync(v_cache, h->vc, bytes, cudaMemcpyDefault, st), "copy v");
  if ((k_cache && !is_device_ptr(k_cache)) || (v_cache && !is_device_ptr(v_cache)))
    H2O_CUDA(h, cudaStreamSynchronize(st), "read_kv sync");
  return H2O_OK;
}

int h2o_info(h2o_t h, int64_t out[5]) {
  if (!h || !out) return fail(h, H2O_EINVAL, "h2o_info: NULL argument");
  out[0] = h->B;
  out[1] = h->t0;
  out[2] = h->n_valid;
  out[3] = h->last_S;
  out[4] = h->last_launches;
  return H2O_OK;
}

int h2o_set_profiling(h2o_t h, int on) {
  if (!h) return fail(nullptr, H2O_EINVAL, "h2o_set_profiling: NULL handle");
  if (on && !h->prefilled) return fail(h, H2O_ESTATE, "h2o_set_profiling: prefill first");
  if (on < 0 || on > 2) return fail(h, H2O_EINVAL, "h2o_set_profiling: on must be 0, 1 or 2");
  h->prof = on != 0;
  if (on == 1) h->prof_steps = 0;
  return H2O_OK;
}

int h2o_step_timings(h2o_t h, int age, float* ms, int n) {
  if (!h || (!ms && n > 0)) return fail(h, H2O_EINVAL, "h2o_step_timings: NULL argument");
  if (age < 0 || age >= h2o_ctx::kProfRing || age >= h->prof_steps)
    return fail(h, H2O_ESTATE, "h2o_step_timings: no profiled step of age %d", age);
  cudaEvent_t* evs = h->ev[(h->prof_steps - 1 - age) % h2o_ctx::kProfRing];
  H2O_CUDA(h, cudaEventSynchronize(evs[2]), "event sync");
  int w = 0;
  for (int i = 0; i < 2 && w < n; ++i, ++w)
    H2O_CUDA(h, cudaEventElapsedTime(&ms[i], evs[i], evs[i + 1]), "event time");
  return w;
}

int h2o_last_timings(h2o_t h, float* ms, int n) {
  if (!h || (!ms && n > 0)) return fail(h, H2O_EINVAL, "h2o_last_timings: NULL argument");
  if (h->prof_steps == 0) return fail(h, H2O_ESTATE, "h2o_last_timings: no profiled step");
  return h2o_step_timings(h, 0, ms, n);
}

int h2o_destroy(h2o_t h) {
  if (!h) return H2O_OK;
  if (h->device >= 0) {
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
  }
  for (DevBuf* b : {&h->newscore, &h->freed, &h->evicted, &h->ws_ml, &h->ws_o,
                    &h->ws_count, &h->st_q[0], &h->st_k[0], &h->st_v[0], &h->st_q[1], &h->st_k[1],
                    &h->st_v[1], &h->st_out})
    cudaFree(b->p);
  for (int i = 0; i < 2; ++i) {
    if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
    if (h->ev_free[i]) cudaEventDestroy(h->ev_free[i]);
  }
  if (h->copy_st) cudaStreamDestroy(h->copy_st);
  if (h->ev_sub) cudaEventDestroy(h->ev_sub);
  if (h->ev_d2h) cudaEventDestroy(h->ev_d2h);
  if (h->d2h_st) cudaStreamDestroy(h->d2h_st);
  release_state(h);
  delete h;
  return H2O_OK;
}

const char* h2o_last_error(h2o_t h) { return h ? h->msg.c_str() : g_thread_err.c_str(); }

int h2o_select(const float* scores, const int32_t* positions, int n_heads, int64_t M, int64_t t0,
               int64_t R, int64_t need, int32_t* evicted, void* stream) {
  if (!scores || !positions || (!evicted && need > 0))
    return fail(nullptr, H2O_EINVAL, "h2o_select: NULL argument");
  if (n_heads < 1 || M < 1 || need < 0 || need > M || R < 0)
    return fail(nullptr, H2O_EINVAL, "h2o_select: bad sizes");
  if (need == 0) return H2O_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* derr = nullptr;
  cudaError_t e = cudaMallocAsync((void**)&derr, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "h2o_select: alloc");
  cudaMemsetAsync(derr, 0, sizeof(int), st);
  // the kernel writes `need` evictions then S - need "empty" slots; S = need here
  e = h2o::launch_select(scores, positions, n_heads, M, t0, R, need, M, need, evicted, need, derr, st);
  int hv = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&hv, derr, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaFreeAsync(derr, st);
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "h2o_select");
  if (hv & h2o::kErrSelect) return fail(nullptr, H2O_ESHAPE, "h2o_select: fewer eligible slots than need");
  return H2O_OK;
}

}  // extern "C"
