// Host side of libkda.so: the C ABI declared in include/kda.h.
//
// Every entry point validates its arguments on the host and returns an error
// code before launching anything; it allocates no device memory (scratch is
// the caller's workspace) and never synchronises except in
// kda_get_device_status().
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "kda_internal.cuh"

namespace kda {

// Per-device status word.  Kernels OR STATUS_* bits into it; the host reads
// and clears it in kda_get_device_status().
__device__ unsigned int g_device_status;

namespace {

constexpr int kMaxDevices = 64;

// Longer request lists run in index order (no workspace).  The allocation-free
// entry point's scratch holds exactly one order of this many requests.
constexpr int kMaxScheduledRequests = KDA_NOALLOC_MAX_REQUESTS;
static_assert(kMaxScheduledRequests == KDA_NOALLOC_MAX_REQUESTS,
              "the allocation-free scratch must hold every order the workspace path writes");

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool env_flag(const char *name) {
  const char *v = std::getenv(name);
  return v && v[0] && std::strcmp(v, "0") != 0;
}

// Limit of the bounded waits inside the tensor-core kernels, in ns; 0 keeps the
// kernels' 2 s.  KDA_TEST_WAIT_LIMIT_NS exists for tests that make a wait run out
// on purpose (to exercise the timeout path); nothing else should set it.
unsigned long long wait_limit_ns() {
  const char *v = std::getenv("KDA_TEST_WAIT_LIMIT_NS");
  if (!v || !v[0]) return 0ull;
  return std::strtoull(v, nullptr, 10);
}

bool valid_dtype(kda_dtype d) { return d == KDA_BF16 || d == KDA_F32; }
size_t dsize(kda_dtype d) { return d == KDA_BF16 ? 2 : 4; }

struct Range {
  const char *lo, *hi;
};
Range span(const void *p, size_t bytes) {
  const char *c = static_cast<const char *>(p);
  return {c, c + bytes};
}
bool overlap(Range a, Range b) {
  return a.lo && b.lo && a.lo < b.hi && b.lo < a.hi;
}

bool head_dims_supported(int dk, int dv) { return dk == dv && (dk == 64 || dk == 128); }

// The gate is given as exactly one of g (fp32 log alpha) and g_logits (bf16 logits of
// the fused activation); n = elements.
bool gate_given(const void *g, const void *g_logits) { return (g != nullptr) != (g_logits != nullptr); }
Range gate_span(const void *g, const void *g_logits, size_t n) {
  return g ? span(g, n * 4) : span(g_logits, n * 2);
}

kda_status check_prefill(const kda_prefill_args *a) {
  if (!a) return KDA_ERR_INVALID_ARG;
  if (a->n_req < 0 || a->total_tokens < 0 || a->H <= 0 || a->dk <= 0 || a->dv <= 0)
    return KDA_ERR_INVALID_ARG;
  if (!valid_dtype(a->in_dtype) || !valid_dtype(a->out_dtype)) return KDA_ERR_INVALID_ARG;
  if (!head_dims_supported(a->dk, a->dv)) return KDA_ERR_UNSUPPORTED;
  if (a->snapshot_stride < 0 || a->snapshot_stride % KDA_CHUNK != 0) return KDA_ERR_INVALID_ARG;
  if (a->n_req == 0) return KDA_OK;
  if (!a->cu_seqlens) return KDA_ERR_INVALID_ARG;
  if (a->g && a->g_logits) return KDA_ERR_INVALID_ARG;
  if (a->total_tokens > 0 &&
      (!a->q || !a->k || !a->v || !gate_given(a->g, a->g_logits) || !a->beta || !a->o))
    return KDA_ERR_INVALID_ARG;
  if (a->snapshot_stride > 0 && (!a->cu_snapshots || !a->snapshots)) return KDA_ERR_INVALID_ARG;
  const void *ptrs[] = {a->q, a->k, a->v, a->g, a->g_logits, a->beta, a->cu_seqlens,
                        a->initial_state, a->o, a->final_state, a->cu_snapshots, a->snapshots};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
  if (a->cu_seqlens_host) {
    const int32_t *cu = a->cu_seqlens_host;
    if (cu[0] != 0) return KDA_ERR_INVALID_ARG;
    for (int r = 0; r < a->n_req; ++r)
      if (cu[r + 1] < cu[r]) return KDA_ERR_INVALID_ARG;
    if (cu[a->n_req] != a->total_tokens) return KDA_ERR_INVALID_ARG;
  }
  // outputs must not overlap inputs (final_state may alias initial_state exactly)
  const size_t T = (size_t)a->total_tokens, H = (size_t)a->H, dk = (size_t)a->dk,
               dv = (size_t)a->dv, n = (size_t)a->n_req;
  const size_t st = n * H * dk * dv * 4;
  Range in[] = {span(a->q, T * H * dk * dsize(a->in_dtype)),
                span(a->k, T * H * dk * dsize(a->in_dtype)),
                span(a->v, T * H * dv * dsize(a->in_dtype)),
                gate_span(a->g, a->g_logits, T * H * dk), span(a->beta, T * H * 4),
                span(a->cu_seqlens, (n + 1) * 4)};
  Range o = span(a->o, T * H * dv * dsize(a->out_dtype));
  Range fs = span(a->final_state, st);
  Range is = span(a->initial_state, st);
  for (Range r : in) {
    if (overlap(o, r) || overlap(fs, r)) return KDA_ERR_INVALID_ARG;
  }
  if (overlap(o, fs) || overlap(o, is)) return KDA_ERR_INVALID_ARG;
  if (a->final_state && a->initial_state && a->final_state != a->initial_state &&
      overlap(fs, is))
    return KDA_ERR_INVALID_ARG;
  return KDA_OK;
}

size_t prefill_ws(int n_req) {
  if (n_req <= 1 || n_req > kMaxScheduledRequests) return 0;
  return align256((size_t)n_req * sizeof(int32_t));
}

// ---------------------------------------------------------------------------
// Context-parallel split of long requests when few chains are live.
//
// A (request, head) chain is one CTA of the tensor-core kernel, and its chunks run
// in order, so a call with fewer chains than SMs leaves most of the GPU idle.  Such a
// call is run as KDA context parallelism inside one device ("Kimi K3 开源日来了",
// Infra section, first layer): long requests are cut into segments.  Pass 1 runs
// each split request's first segment from its initial state on a second stream,
// beside a local-state pass that gives every middle segment its zero-start state S_loc
// and transition M (one CTA per segment and head, all in one wave); an exact combine
// per request then recovers the other segments' start states from the first
// segment's final state; and pass 2 runs every other segment from its start state,
// writing o, the snapshots and (through the last segment) the final state.  The
// results equal the unsplit call's up to rounding.
// ---------------------------------------------------------------------------
struct SplitPlan {
  int n_seg = 0;                    // segments over all requests; 0: no split
  std::vector<int32_t> seg_cu;      // [n_seg + 1] token bounds of the segments
  std::vector<int32_t> first_seg;   // [n_req + 1] first segment of each request
  std::vector<int32_t> pass1;       // local states: middle segments of split requests
  std::vector<int32_t> first;       // first segments of split requests (prefilled in pass 1)
  std::vector<int32_t> pass2;       // the other segments (and unsplit requests)
  std::vector<int32_t> seg_snap;    // [n_seg + 1] snapshot rows before each segment
  // workspace layout (byte offsets, 256-aligned)
  size_t off_cu = 0, off_p1 = 0, off_first = 0, off_p2 = 0, off_snap = 0, off_sloc = 0, off_m = 0,
         off_sin = 0, bytes = 0;
};

// SMs of the current device.  KDA_TEST_SM_COUNT overrides it, so that host tests
// (which may run without a GPU) can check the split plan; nothing else should set it.
int device_sm_count() {
  if (const char *v = std::getenv("KDA_TEST_SM_COUNT"))
    if (v[0]) return std::atoi(v);
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();  // no device here: never split
    return 0;
  }
  return n;
}

// Plans the split from the host lengths; false (no split) unless it pays:
//   - the tensor-core kernel runs, the host lengths are given, KDA_NO_SPLIT is unset;
//   - the chains fill at most half of the SMs;
//   - every segment holds at least 1,024 tokens and starts on a multiple of 32 (of
//     the snapshot stride when snapshots are taken), so that snapshots tile it;
//   - each pass fits in one wave: pass 1 runs, per head, the first segment of every
//     split request (a prefill from the request's initial state) beside the local
//     states of its middle segments; pass 2 runs every other segment;
//   - the estimated time, in tokens of one chain, drops by 15 % or more: the longest
//     first segment (it bounds pass 1: a middle segment's local state costs 0.9 of
//     a prefill chunk, measured 4.25 against 4.7 us per chunk), plus the longest
//     pass-2 segment, plus 256 for the extra launches and the combine, against the
//     longest request unsplit.  (So a two-way split never pays.)
// Extra segments go, one at a time, to the request whose longest segment is longest.
bool plan_split(const kda_prefill_args *a, SplitPlan *pl) {
  if (!a->cu_seqlens_host || a->n_req <= 0 || a->total_tokens <= 0) return false;
  if (!prefill_tc_supported(a->dk, a->dv, a->in_dtype) || env_flag("KDA_FORCE_SIMT") ||
      env_flag("KDA_NO_SPLIT"))
    return false;
  const int sms = device_sm_count();
  const long chains = (long)a->n_req * a->H;
  if (sms <= 0 || 2 * chains > sms) return false;
  const int max_total = sms / a->H, max_extra = max_total;
  const int align = a->snapshot_stride > 0 ? a->snapshot_stride : 32;  // stride % 64 == 0
  const int min_len = align > 1024 ? align : 1024;
  const int32_t *cu = a->cu_seqlens_host;
  std::vector<int> parts(a->n_req, 1);
  // segment length of request r cut in s parts (the last one takes the rest)
  auto piece = [&](int r, int s) -> long {
    const long len = cu[r + 1] - cu[r];
    const long p = (len + s - 1) / s;
    return (p + align - 1) / align * align;
  };
  // the next part count of request r with every segment but the last at least
  // min_len tokens and a non-empty last one (alignment may skip a count); 0 if none
  auto next_parts = [&](int r) -> int {
    const long len = cu[r + 1] - cu[r];
    for (int s = parts[r] + 1; s <= parts[r] + max_extra; ++s) {
      const long p = piece(r, s);
      if (p < min_len) return 0;
      if ((s - 1) * p < len) return s;
    }
    return 0;
  };
  // segments per head in each pass: pass 1 = sum over split requests of parts - 1
  // (the first segment and the middle ones), pass 2 = every segment but the first
  // segments of split requests
  int total = a->n_req, extra = 0, pass2 = a->n_req;
  auto in_pass2 = [](int n_parts) { return n_parts > 1 ? n_parts - 1 : 1; };
  for (;;) {
    int best = -1, best_parts = 0;
    long best_len = 0;
    for (int r = 0; r < a->n_req; ++r) {
      const int s = next_parts(r);
      if (s == 0 || pass2 + in_pass2(s) - in_pass2(parts[r]) > max_total ||
          extra + (s - parts[r]) > max_extra)
        continue;
      const long len = cu[r + 1] - cu[r];
      const long longest = parts[r] == 1 ? len : piece(r, parts[r]);
      if (longest > best_len) {
        best_len = longest;
        best = r;
        best_parts = s;
      }
    }
    if (best < 0) break;
    total += best_parts - parts[best];
    extra += best_parts - parts[best];
    pass2 += in_pass2(best_parts) - in_pass2(parts[best]);
    parts[best] = best_parts;
  }
  if (extra == 0) return false;
  long longest = 0, longest_p1 = 0, longest_p2 = 0;
  for (int r = 0; r < a->n_req; ++r) {
    const long len = cu[r + 1] - cu[r];
    longest = len > longest ? len : longest;
    const long p = parts[r] > 1 ? piece(r, parts[r]) : len;
    const long last = len - (parts[r] - 1) * p;
    if (parts[r] > 1) longest_p1 = std::max(longest_p1, p);
    longest_p2 = std::max(longest_p2, std::max(parts[r] > 2 ? p : 0L, last));
  }
  if ((double)longest_p1 + longest_p2 + 256.0 > 0.85 * longest) return false;

  pl->n_seg = total;
  pl->seg_cu.assign(1, 0);
  pl->first_seg.assign(1, 0);
  pl->pass1.clear();
  pl->first.clear();
  pl->pass2.clear();
  pl->seg_snap.assign(1, 0);
  int32_t snaps_before = 0;
  for (int r = 0; r < a->n_req; ++r) {
    const int32_t bos = cu[r], eos = cu[r + 1];
    const long p = parts[r] > 1 ? piece(r, parts[r]) : (long)(eos - bos);
    for (int k = 0; k < parts[r]; ++k) {
      const int32_t end = k + 1 < parts[r] ? bos + (int32_t)((k + 1) * p) : eos;
      const int32_t seg = (int32_t)pl->seg_cu.size() - 1;
      if (parts[r] > 1 && k == 0)
        pl->first.push_back(seg);
      else
        pl->pass2.push_back(seg);
      if (k > 0 && k + 1 < parts[r]) pl->pass1.push_back(seg);
      pl->seg_cu.push_back(end);
      if (a->snapshot_stride > 0)
        pl->seg_snap.push_back(snaps_before + (end - bos) / a->snapshot_stride);
    }
    pl->first_seg.push_back((int32_t)pl->seg_cu.size() - 1);
    if (a->snapshot_stride > 0) snaps_before += (eos - bos) / a->snapshot_stride;
  }
  const size_t n = (size_t)pl->n_seg, state = (size_t)a->H * a->dk * a->dv * sizeof(float);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  pl->off_cu = take((n + 1) * sizeof(int32_t));
  pl->off_p1 = take(pl->pass1.size() * sizeof(int32_t));
  pl->off_first = take(pl->first.size() * sizeof(int32_t));
  pl->off_p2 = take(pl->pass2.size() * sizeof(int32_t));
  pl->off_snap = take((n + 1) * sizeof(int32_t));
  pl->off_sloc = take(n * state);
  pl->off_m = take(n * (size_t)a->H * a->dk * a->dk * sizeof(float));
  pl->off_sin = take(n * state);
  pl->bytes = off;
  return true;
}

// A failed CUDA call becomes KDA_ERR_CUDA; with KDA_VERBOSE=1 its message goes to stderr.
kda_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return KDA_OK;
  if (env_flag("KDA_VERBOSE")) std::fprintf(stderr, "libkda: CUDA error: %s\n", cudaGetErrorString(e));
  return KDA_ERR_CUDA;
}

CUcontext current_context();

// A second stream of the current context, created once and kept: the split call runs
// the first segments' prefill on it beside the local-state pass.  Calls that share it
// stay correct (each joins through its own events); they only queue behind each other.
cudaStream_t side_stream() {
  static std::mutex mu;
  static std::vector<std::pair<CUcontext, cudaStream_t>> streams;
  const CUcontext ctx = current_context();
  if (!ctx) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto &e : streams)
    if (e.first == ctx) return e.second;
  cudaStream_t st = nullptr;
  if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
  streams.emplace_back(ctx, st);
  return st;
}

// The split call (see plan_split), in two passes:
//   1. on a second stream, the first segment of every split request from the request's
//      initial state (o, snapshots; its final state into that segment's S_loc slot),
//      and on the call's stream the local states and transitions of the middle
//      segments;
//   2. after both, the combine per split request from the first segment's final state,
//      then every other segment from its start state; the final states are copied out.
kda_status run_split(const kda_prefill_args *a, const SplitPlan &pl, char *ws,
                     const PrefillParams &base, cudaStream_t s) {
  int32_t *seg_cu = reinterpret_cast<int32_t *>(ws + pl.off_cu);
  int32_t *p1 = reinterpret_cast<int32_t *>(ws + pl.off_p1);
  int32_t *first = reinterpret_cast<int32_t *>(ws + pl.off_first);
  int32_t *p2 = reinterpret_cast<int32_t *>(ws + pl.off_p2);
  int32_t *seg_snap = reinterpret_cast<int32_t *>(ws + pl.off_snap);
  float *sloc = reinterpret_cast<float *>(ws + pl.off_sloc);
  float *m = reinterpret_cast<float *>(ws + pl.off_m);
  float *s_start = reinterpret_cast<float *>(ws + pl.off_sin);
  const size_t state = (size_t)a->H * a->dk * a->dv, trans = (size_t)a->H * a->dk * a->dk;
  // the plan's small tables (pageable host memory: each copy has left the host
  // buffer when it returns)
  cudaError_t e = cudaSuccess;
  auto put = [&](int32_t *dst, const std::vector<int32_t> &v) {
    if (e == cudaSuccess && !v.empty())
      e = cudaMemcpyAsync(dst, v.data(), v.size() * sizeof(int32_t), cudaMemcpyHostToDevice, s);
  };
  put(seg_cu, pl.seg_cu);
  put(p1, pl.pass1);
  put(first, pl.first);
  put(p2, pl.pass2);
  if (a->snapshot_stride > 0) put(seg_snap, pl.seg_snap);
  // every request's first segment starts from its initial state
  for (int r = 0; r < a->n_req && e == cudaSuccess; ++r) {
    const int row0 = pl.first_seg[r];
    const float *s_init = a->initial_state ? a->initial_state + (size_t)r * state : nullptr;
    e = s_init ? cudaMemcpyAsync(s_start + row0 * state, s_init, state * sizeof(float),
                                 cudaMemcpyDeviceToDevice, s)
               : cudaMemsetAsync(s_start + row0 * state, 0, state * sizeof(float), s);
  }
  if (e != cudaSuccess) return from_cuda(e);

  // pass 1: the first segments on the second stream, forked from and joined to s (on
  // s itself, one kernel after the other, if no second stream can be had)
  cudaStream_t side = side_stream();
  cudaEvent_t fork = nullptr, join = nullptr;
  if (side && cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess)
    side = nullptr;
  if (side && cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
    cudaEventDestroy(fork);
    side = nullptr;
  }
  if (!side) {
    (void)cudaGetLastError();  // a failed event or stream creation is not the call's error
    fork = join = nullptr;
  }
  PrefillParams fp = base;
  fp.cu_seqlens = seg_cu;
  fp.n_req = (int)pl.first.size();
  fp.order = first;
  fp.initial_state = s_start;
  fp.final_state = sloc;  // the first segment has no local state of its own
  fp.cu_snapshots = a->snapshot_stride > 0 ? seg_snap : nullptr;
  if (side) {
    e = cudaEventRecord(fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
    if (e == cudaSuccess) e = launch_prefill_tc(fp, a->in_dtype, a->out_dtype, side);
    if (e == cudaSuccess) e = cudaEventRecord(join, side);
  } else {
    e = launch_prefill_tc(fp, a->in_dtype, a->out_dtype, s);
  }
  if (e == cudaSuccess) {
    // local states and transitions of the middle segments
    PrefillParams lp = base;
    lp.q = nullptr;
    lp.o = nullptr;
    lp.initial_state = nullptr;
    lp.final_state = nullptr;
    lp.snapshot_stride = 0;
    lp.cu_snapshots = nullptr;
    lp.snapshots = nullptr;
    lp.cu_seqlens = seg_cu;
    lp.n_req = (int)pl.pass1.size();
    lp.order = p1;
    lp.local_mode = 1;
    lp.s_loc = sloc;
    lp.m = m;
    e = launch_prefill_tc(lp, a->in_dtype, KDA_F32, s);
  }
  if (side) {
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, join, 0);
    cudaEventDestroy(fork);  // released once recorded work completes
    cudaEventDestroy(join);
  }
  if (e != cudaSuccess) return from_cuda(e);

  // start states of the other segments of split requests: S_in[1] is the first
  // segment's final state, then S_in[k + 1] = M_k S_in[k] + S_loc_k
  for (int r = 0; r < a->n_req; ++r) {
    const int row0 = pl.first_seg[r], n = pl.first_seg[r + 1] - row0;
    if (n == 1) continue;
    e = launch_combine(sloc + (row0 + 1) * state, m + (row0 + 1) * trans, sloc + row0 * state,
                       n - 2, a->H, a->dk, a->dv, s_start + (row0 + 1) * state,
                       s_start + (row0 + n - 1) * state, s);
    if (e != cudaSuccess) return from_cuda(e);
  }

  // pass 2: every other segment from its start state; the final states land in place
  PrefillParams sp = base;
  sp.cu_seqlens = seg_cu;
  sp.n_req = (int)pl.pass2.size();
  sp.order = p2;
  sp.initial_state = s_start;
  sp.final_state = s_start;
  sp.cu_snapshots = a->snapshot_stride > 0 ? seg_snap : nullptr;
  if ((e = launch_prefill_tc(sp, a->in_dtype, a->out_dtype, s)) != cudaSuccess)
    return from_cuda(e);
  if (a->final_state)
    for (int r = 0; r < a->n_req; ++r) {
      const int last = pl.first_seg[r + 1] - 1;
      e = cudaMemcpyAsync(a->final_state + (size_t)r * state, s_start + last * state,
                          state * sizeof(float), cudaMemcpyDeviceToDevice, s);
      if (e != cudaSuccess) return from_cuda(e);
    }
  return KDA_OK;
}

// The current thread's CUDA context, through the driver entry point the
// runtime exposes (the library does not link libcuda).  NULL if unavailable.
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext *);
  static Fn fn = [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    return (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
               ? reinterpret_cast<Fn>(ptr)
               : nullptr;
  }();
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

}  // namespace

// Device addresses of this library's __device__ arrays, looked up with
// cudaGetSymbolAddress once per device and context: a device reset (or any
// new primary context) gives the module new addresses, so an entry is reused
// only while the context it was taken in is still current.  The lock makes a
// first call from two host threads at once safe.
SymbolAddressCache::SymbolAddressCache(const void *symbol) : symbol_(symbol) {}

void *SymbolAddressCache::get() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> hold(mu_);
  CUcontext ctx = current_context();
  if (ctx && ctx == ctx_[dev] && addr_[dev]) return addr_[dev];
  void *addr = nullptr;  // also makes the device's primary context current
  if (cudaGetSymbolAddress(&addr, symbol_) != cudaSuccess) return nullptr;
  ctx_[dev] = current_context();
  addr_[dev] = addr;
  return addr;
}

unsigned int *device_status_word() {
  static SymbolAddressCache cache(reinterpret_cast<const void *>(&g_device_status));
  return static_cast<unsigned int *>(cache.get());
}

}  // namespace kda

using namespace kda;

namespace kda {
// kda_prefill_chunked, with the context-parallel split allowed or not
kda_status prefill_call(const kda_prefill_args *a, void *workspace, size_t workspace_bytes,
                        void *stream, bool allow_split);
}  // namespace kda

extern "C" {

size_t kda_prefill_workspace_size(const kda_prefill_args *args) {
  if (check_prefill(args) != KDA_OK) return 0;
  kda::SplitPlan plan;
  if (kda::plan_split(args, &plan)) return plan.bytes;
  return prefill_ws(args->n_req);
}

int32_t kda_prefill_split_segments(const kda_prefill_args *args) {
  if (check_prefill(args) != KDA_OK) return 0;
  kda::SplitPlan plan;
  return kda::plan_split(args, &plan) ? plan.n_seg : 0;
}

kda_status kda_prefill_chunked(const kda_prefill_args *a, void *workspace,
                               size_t workspace_bytes, void *stream) {
  return kda::prefill_call(a, workspace, workspace_bytes, stream, true);
}

}  // extern "C"

namespace kda {

kda_status prefill_call(const kda_prefill_args *a, void *workspace, size_t workspace_bytes,
                        void *stream, bool allow_split) {
  kda_status st = check_prefill(a);
  if (st != KDA_OK) return st;
  if (a->n_req == 0) return KDA_OK;
  // the unsplit call's workspace (the split asks for more, and falls back to the
  // unsplit call when it does not get it)
  const size_t need = prefill_ws(a->n_req);
  if (need > 0 && (!workspace || workspace_bytes < need ||
                   (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
    return KDA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  PrefillParams p{};
  p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta;
  p.g_logits = static_cast<const __nv_bfloat16 *>(a->g_logits);
  p.cu_seqlens = a->cu_seqlens;
  p.initial_state = a->initial_state;
  p.o = a->o;
  p.final_state = a->final_state;
  p.cu_snapshots = a->cu_snapshots;
  p.snapshots = a->snapshots;
  p.n_req = a->n_req; p.total_tokens = a->total_tokens;
  p.H = a->H; p.dk = a->dk; p.dv = a->dv;
  p.snapshot_stride = a->snapshot_stride;
  p.validate = env_flag("KDA_VALIDATE");
  p.wait_ns = wait_limit_ns();
  p.status = device_status_word();
  if (!p.status) return KDA_ERR_CUDA;
  // the tensor-core kernel needs at least one token to build its TMA maps
  const bool use_tc = prefill_tc_supported(a->dk, a->dv, a->in_dtype) && a->total_tokens > 0 &&
                      !env_flag("KDA_FORCE_SIMT");
  // few chains: the context-parallel split, when the workspace holds it
  if (use_tc && allow_split && workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) == 0) {
    SplitPlan plan;
    if (plan_split(a, &plan) && workspace_bytes >= plan.bytes)
      return run_split(a, plan, static_cast<char *>(workspace), p, s);
  }
  if (need > 0) {
    int32_t *order = static_cast<int32_t *>(workspace);
    cudaError_t e = launch_schedule(a->cu_seqlens, a->n_req, order, s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    p.order = order;
  }
  if (use_tc) return from_cuda(launch_prefill_tc(p, a->in_dtype, a->out_dtype, s));
  p.n_slices = prefill_simt_slices(a->dk, a->dv, false);
  return from_cuda(launch_prefill_simt(p, a->in_dtype, a->out_dtype, s));
}

}  // namespace kda

extern "C" {

size_t kda_local_state_workspace_size(const kda_local_state_args *a) {
  (void)a;
  return 0;
}

kda_status kda_chunk_local_state(const kda_local_state_args *a, void *workspace,
                                 size_t workspace_bytes, void *stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (!a) return KDA_ERR_INVALID_ARG;
  if (a->n_seg <= 0 || a->total_tokens < 0 || a->H <= 0) return KDA_ERR_INVALID_ARG;
  if (!valid_dtype(a->in_dtype)) return KDA_ERR_INVALID_ARG;
  if (!head_dims_supported(a->dk, a->dv)) return KDA_ERR_UNSUPPORTED;
  if (!a->seg_cu || !a->s_loc || !a->m) return KDA_ERR_INVALID_ARG;
  if (a->g && a->g_logits) return KDA_ERR_INVALID_ARG;
  if (a->total_tokens > 0 && (!a->k || !a->v || !gate_given(a->g, a->g_logits) || !a->beta))
    return KDA_ERR_INVALID_ARG;
  const void *ptrs[] = {a->k, a->v, a->g, a->g_logits, a->beta, a->seg_cu, a->s_loc, a->m};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
  if (a->seg_cu_host) {
    if (a->seg_cu_host[0] != 0 || a->seg_cu_host[a->n_seg] != a->total_tokens)
      return KDA_ERR_INVALID_ARG;
    for (int s = 0; s < a->n_seg; ++s)
      if (a->seg_cu_host[s + 1] < a->seg_cu_host[s]) return KDA_ERR_INVALID_ARG;
  }
  const size_t T = (size_t)a->total_tokens, H = (size_t)a->H, dk = (size_t)a->dk,
               dv = (size_t)a->dv, n = (size_t)a->n_seg;
  Range outs[] = {span(a->s_loc, n * H * dk * dv * 4), span(a->m, n * H * dk * dk * 4)};
  Range ins[] = {span(a->k, T * H * dk * dsize(a->in_dtype)),
                 span(a->v, T * H * dv * dsize(a->in_dtype)),
                 gate_span(a->g, a->g_logits, T * H * dk), span(a->beta, T * H * 4),
                 span(a->seg_cu, (n + 1) * 4)};
  if (overlap(outs[0], outs[1])) return KDA_ERR_INVALID_ARG;
  for (Range o : outs)
    for (Range i : ins)
      if (overlap(o, i)) return KDA_ERR_INVALID_ARG;

  PrefillParams p{};
  p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta;
  p.g_logits = static_cast<const __nv_bfloat16 *>(a->g_logits);
  p.cu_seqlens = a->seg_cu;
  p.n_req = a->n_seg; p.total_tokens = a->total_tokens;
  p.H = a->H; p.dk = a->dk; p.dv = a->dv;
  p.local_mode = 1;
  p.s_loc = a->s_loc;
  p.m = a->m;
  p.validate = env_flag("KDA_VALIDATE");
  p.wait_ns = wait_limit_ns();
  p.status = device_status_word();
  if (!p.status) return KDA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (prefill_tc_supported(a->dk, a->dv, a->in_dtype) && a->total_tokens > 0 &&
      !env_flag("KDA_FORCE_SIMT"))
    return from_cuda(launch_prefill_tc(p, a->in_dtype, KDA_F32, s));
  p.n_slices = prefill_simt_slices(a->dk, a->dv, true);
  return from_cuda(launch_prefill_simt(p, a->in_dtype, KDA_F32, s));
}

kda_status kda_state_combine(const float *s_loc, const float *m, const float *s_init,
                             int32_t n_seg, int32_t H, int32_t dk, int32_t dv, float *s_in,
                             float *s_final, void *stream) {
  if (n_seg <= 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
  if (!head_dims_supported(dk, dv)) return KDA_ERR_UNSUPPORTED;
  if (!s_loc || !m) return KDA_ERR_INVALID_ARG;
  const void *ptrs[] = {s_loc, m, s_init, s_in, s_final};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
  const size_t n = n_seg, h = H, k = dk, v = dv;
  Range ins[] = {span(s_loc, n * h * k * v * 4), span(m, n * h * k * k * 4),
                 span(s_init, h * k * v * 4)};
  Range outs[] = {span(s_in, n * h * k * v * 4), span(s_final, h * k * v * 4)};
  if (overlap(outs[0], outs[1])) return KDA_ERR_INVALID_ARG;
  for (Range o : outs)
    for (Range i : ins)
      if (overlap(o, i)) return KDA_ERR_INVALID_ARG;
  return from_cuda(launch_combine(s_loc, m, s_init, n_seg, H, dk, dv, s_in, s_final,
                                  static_cast<cudaStream_t>(stream)));
}

kda_status kda_decode_step(const kda_decode_args *a, void *stream) {
  if (!a) return KDA_ERR_INVALID_ARG;
  if (a->n < 0 || a->H <= 0 || a->dk <= 0 || a->dv <= 0 || a->n_slots < 0)
    return KDA_ERR_INVALID_ARG;
  if (!valid_dtype(a->in_dtype) || !valid_dtype(a->out_dtype)) return KDA_ERR_INVALID_ARG;
  if (!head_dims_supported(a->dk, a->dv)) return KDA_ERR_UNSUPPORTED;
  if (a->n == 0) return KDA_OK;
  if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->state || !a->o)
    return KDA_ERR_INVALID_ARG;
  if (!a->slot && a->n_slots < a->n) return KDA_ERR_INVALID_ARG;
  const void *ptrs[] = {a->q, a->k, a->v, a->g, a->beta, a->state, a->slot, a->o};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
  const size_t n = a->n, H = a->H, dk = a->dk, dv = a->dv;
  Range st = span(a->state, (size_t)a->n_slots * H * dk * dv * 4);
  Range o = span(a->o, n * H * dv * dsize(a->out_dtype));
  Range ins[] = {span(a->q, n * H * dk * dsize(a->in_dtype)),
                 span(a->k, n * H * dk * dsize(a->in_dtype)),
                 span(a->v, n * H * dv * dsize(a->in_dtype)), span(a->g, n * H * dk * 4),
                 span(a->beta, n * H * 4), span(a->slot, a->slot ? n * 4 : 0)};
  if (overlap(o, st)) return KDA_ERR_INVALID_ARG;
  for (Range i : ins)
    if (overlap(o, i) || overlap(st, i)) return KDA_ERR_INVALID_ARG;
  DecodeParams p{};
  p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta;
  p.state = a->state; p.slot = a->slot; p.o = a->o;
  p.n = a->n; p.H = a->H; p.dk = a->dk; p.dv = a->dv; p.n_slots = a->n_slots;
  p.validate = env_flag("KDA_VALIDATE");
  p.status = device_status_word();
  if (!p.status) return KDA_ERR_CUDA;
  return from_cuda(launch_decode(p, a->in_dtype, a->out_dtype, static_cast<cudaStream_t>(stream)));
}

int32_t kda_snapshot_count(int32_t len, int32_t stride) {
  return (stride > 0 && len > 0) ? len / stride : 0;
}

kda_status kda_get_device_status(void *stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KDA_ERR_CUDA;
  unsigned int *addr = device_status_word();
  if (!addr) return KDA_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpy(&word, addr, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return KDA_ERR_CUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpy(addr, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return KDA_ERR_CUDA;
  }
  if (word & STATUS_TIMEOUT) return KDA_ERR_TIMEOUT;
  if (word & STATUS_GATE_RANGE) return KDA_ERR_GATE_RANGE;
  if (word & STATUS_BAD_SEQLENS) return KDA_ERR_INVALID_ARG;
  return KDA_OK;
}

const char *kda_status_string(kda_status status) {
  switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_GATE_RANGE: return "KDA_ERR_GATE_RANGE";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
  }
  return "KDA_ERR_UNKNOWN";
}

int32_t kda_version(void) { return KDA_VERSION; }

int32_t kda_prefill_uses_tensor_cores(int32_t dk, int32_t dv, kda_dtype in_dtype) {
  return (prefill_tc_supported(dk, dv, in_dtype) && !env_flag("KDA_FORCE_SIMT")) ? 1 : 0;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free prefill: the workspace of kda_prefill_chunked (the
// longest-first request order) comes from a fixed array in this library.
// ---------------------------------------------------------------------------

namespace kda {
namespace {

// Scratch of kda_prefill_chunked_noalloc.  Host code must not use this name
// as a device address: it is a host-side stand-in.  The device address comes
// from cudaGetSymbolAddress, looked up on the first call with a device (and
// context) current and reused after that.
static __device__ __align__(256) int32_t g_noalloc_order[KDA_NOALLOC_MAX_REQUESTS];

int32_t *noalloc_scratch() {
  static SymbolAddressCache cache(reinterpret_cast<const void *>(&g_noalloc_order));
  return static_cast<int32_t *>(cache.get());
}

}  // namespace
}  // namespace kda

extern "C" kda_status kda_prefill_chunked_noalloc(const kda_prefill_args *args, void *stream) {
  if (!args) return KDA_ERR_INVALID_ARG;
  if (args->n_req > KDA_NOALLOC_MAX_REQUESTS) return KDA_ERR_WORKSPACE;
  int32_t *scratch = kda::noalloc_scratch();
  if (!scratch) return KDA_ERR_CUDA;
  // no context-parallel split: its states would need more than the fixed scratch
  return kda::prefill_call(args, scratch, sizeof(kda::g_noalloc_order), stream, false);
}

// ---------------------------------------------------------------------------
// Backward of the prefill: argument checks, the chunk table, the forward pass
// that leaves the chunk-start states in the workspace, then the backward
// kernels (kda_backward.cu).
// ---------------------------------------------------------------------------

namespace kda {
namespace {

struct BwdShape {
  int n_chunks = 0, n_snap = 0;
};

kda_status check_backward(const kda_backward_args *a, BwdShape *sh) {
  if (!a) return KDA_ERR_INVALID_ARG;
  if (a->n_req < 0 || a->total_tokens < 0 || a->H <= 0 || a->dk <= 0 || a->dv <= 0)
    return KDA_ERR_INVALID_ARG;
  if (!valid_dtype(a->in_dtype)) return KDA_ERR_INVALID_ARG;
  if (!head_dims_supported(a->dk, a->dv)) return KDA_ERR_UNSUPPORTED;
  *sh = BwdShape{};
  if (a->n_req == 0) return KDA_OK;
  if (!a->cu_seqlens || !a->cu_seqlens_host) return KDA_ERR_INVALID_ARG;
  const int32_t *cu = a->cu_seqlens_host;
  if (cu[0] != 0 || cu[a->n_req] != a->total_tokens) return KDA_ERR_INVALID_ARG;
  long long n_chunks = 0, n_snap = 0;
  for (int r = 0; r < a->n_req; ++r) {
    const long long len = (long long)cu[r + 1] - cu[r];
    if (len < 0) return KDA_ERR_INVALID_ARG;
    n_chunks += (len + KDA_CHUNK - 1) / KDA_CHUNK;
    n_snap += len / KDA_CHUNK;
  }
  if (n_chunks * a->H > 0x7fffffffLL || (long long)a->n_req * a->H > 0x7fffffffLL)
    return KDA_ERR_UNSUPPORTED;
  if (a->g && a->g_logits) return KDA_ERR_INVALID_ARG;
  if (a->total_tokens > 0 &&
      (!a->q || !a->k || !a->v || !gate_given(a->g, a->g_logits) || !a->beta || !a->d_q ||
       !a->d_k || !a->d_v || !a->d_g || !a->d_beta))
    return KDA_ERR_INVALID_ARG;
  const void *ptrs[] = {a->q, a->k, a->v, a->g, a->g_logits, a->beta, a->cu_seqlens,
                        a->initial_state, a->d_o, a->d_final, a->d_q, a->d_k, a->d_v, a->d_g,
                        a->d_beta, a->d_initial};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
  const size_t T = (size_t)a->total_tokens, H = (size_t)a->H, dk = (size_t)a->dk,
               dv = (size_t)a->dv, n = (size_t)a->n_req;
  Range ins[] = {span(a->q, T * H * dk * dsize(a->in_dtype)),
                 span(a->k, T * H * dk * dsize(a->in_dtype)),
                 span(a->v, T * H * dv * dsize(a->in_dtype)),
                 gate_span(a->g, a->g_logits, T * H * dk), span(a->beta, T * H * 4),
                 span(a->cu_seqlens, (n + 1) * 4),
                 span(a->initial_state, n * H * dk * dv * 4), span(a->d_o, T * H * dv * 4),
                 span(a->d_final, n * H * dk * dv * 4)};
  Range outs[] = {span(a->d_q, T * H * dk * 4), span(a->d_k, T * H * dk * 4),
                  span(a->d_v, T * H * dv * 4), span(a->d_g, T * H * dk * 4),
                  span(a->d_beta, T * H * 4), span(a->d_initial, n * H * dk * dv * 4)};
  for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
    for (Range in : ins)
      if (overlap(outs[i], in)) return KDA_ERR_INVALID_ARG;
    for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
      if (overlap(outs[i], outs[j])) return KDA_ERR_INVALID_ARG;
  }
  sh->n_chunks = (int)n_chunks;
  sh->n_snap = (int)n_snap;
  return KDA_OK;
}

}  // namespace
}  // namespace kda

extern "C" size_t kda_prefill_backward_workspace_size(const kda_backward_args *a) {
  kda::BwdShape sh;
  if (kda::check_backward(a, &sh) != KDA_OK || a->n_req == 0) return 0;
  return kda::backward_workspace_bytes(a->n_req, sh.n_chunks, sh.n_snap, a->H, a->dk);
}

extern "C" kda_status kda_prefill_backward(const kda_backward_args *a, void *workspace,
                                           size_t workspace_bytes, void *stream) {
  using namespace kda;
  BwdShape sh;
  kda_status st = check_backward(a, &sh);
  if (st != KDA_OK) return st;
  if (a->n_req == 0) return KDA_OK;
  const int D = a->dk, H = a->H, n_req = a->n_req;
  const size_t need = backward_workspace_bytes(n_req, sh.n_chunks, sh.n_snap, H, D);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return KDA_ERR_WORKSPACE;
  {  // outputs must not overlap the workspace
    const size_t T = (size_t)a->total_tokens, n = (size_t)n_req;
    Range ws = span(workspace, need);
    Range outs[] = {span(a->d_q, T * H * D * 4), span(a->d_k, T * H * D * 4),
                    span(a->d_v, T * H * D * 4), span(a->d_g, T * H * D * 4),
                    span(a->d_beta, T * H * 4), span(a->d_initial, n * H * D * D * 4)};
    for (Range o : outs)
      if (overlap(o, ws)) return KDA_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  size_t o_chunks, o_cu_chunks, o_cu_snap, o_snaps, o_zero;
  backward_offsets(n_req, sh.n_chunks, sh.n_snap, H, D, &o_chunks, &o_cu_chunks, &o_cu_snap,
                   &o_snaps, &o_zero);
  char *ws = static_cast<char *>(workspace);

  // chunk table (request, chunk index, first token, rows), chunk and snapshot offsets
  std::vector<unsigned char> host(o_snaps, 0);
  int32_t *chunks = reinterpret_cast<int32_t *>(host.data() + o_chunks);
  int32_t *cu_chunks = reinterpret_cast<int32_t *>(host.data() + o_cu_chunks);
  int32_t *cu_snap = reinterpret_cast<int32_t *>(host.data() + o_cu_snap);
  const int32_t *cu = a->cu_seqlens_host;
  int jc = 0;
  cu_chunks[0] = 0;
  cu_snap[0] = 0;
  for (int r = 0; r < n_req; ++r) {
    const int len = cu[r + 1] - cu[r];
    for (int c = 0; c * KDA_CHUNK < len; ++c, ++jc) {
      chunks[4 * jc + 0] = r;
      chunks[4 * jc + 1] = c;
      chunks[4 * jc + 2] = cu[r] + c * KDA_CHUNK;
      chunks[4 * jc + 3] = len - c * KDA_CHUNK < KDA_CHUNK ? len - c * KDA_CHUNK : KDA_CHUNK;
    }
    cu_chunks[r + 1] = jc;
    cu_snap[r + 1] = cu_snap[r] + len / KDA_CHUNK;
  }
  cudaError_t e = cudaMemcpyAsync(ws, host.data(), o_snaps, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws + o_zero, 0, (size_t)D * D * sizeof(float), s);
  if (e != cudaSuccess) return from_cuda(e);

  // forward pass: the state at every 64-token boundary is a chunk's start state
  if (sh.n_chunks > 0) {
    PrefillParams p{};
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta;
    p.g_logits = static_cast<const __nv_bfloat16 *>(a->g_logits);
    p.cu_seqlens = a->cu_seqlens;
    p.initial_state = a->initial_state;
    p.cu_snapshots = reinterpret_cast<const int32_t *>(ws + o_cu_snap);
    p.snapshots = reinterpret_cast<float *>(ws + o_snaps);
    p.n_req = n_req; p.total_tokens = a->total_tokens;
    p.H = H; p.dk = D; p.dv = D;
    p.snapshot_stride = KDA_CHUNK;
    p.validate = env_flag("KDA_VALIDATE");
    p.status = device_status_word();
    if (!p.status) return KDA_ERR_CUDA;
    if (prefill_tc_supported(D, D, a->in_dtype) && !env_flag("KDA_FORCE_SIMT")) {
      e = launch_prefill_tc(p, a->in_dtype, KDA_F32, s);
    } else {
      p.n_slices = prefill_simt_slices(D, D, false);
      e = launch_prefill_simt(p, a->in_dtype, KDA_F32, s);
    }
    if (e != cudaSuccess) return from_cuda(e);
  }
  BackwardLaunch b{};
  b.q = a->q; b.k = a->k; b.v = a->v; b.g = a->g; b.beta = a->beta;
  b.g_logits = static_cast<const __nv_bfloat16 *>(a->g_logits);
  b.initial_state = a->initial_state; b.d_o = a->d_o; b.d_final = a->d_final;
  b.dq = a->d_q; b.dk = a->d_k; b.dv = a->d_v; b.dg = a->d_g; b.dbeta = a->d_beta;
  b.d_initial = a->d_initial;
  b.workspace = workspace;
  b.n_req = n_req; b.n_chunks = sh.n_chunks; b.n_snap = sh.n_snap; b.H = H; b.D = D;
  b.in_dtype = a->in_dtype;
  return from_cuda(launch_backward(b, s));
}
