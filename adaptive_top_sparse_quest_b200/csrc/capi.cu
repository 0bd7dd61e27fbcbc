// C ABI of the Twilight decode path (declared in include/twilight.h): host-side
// argument checks, workspace carving and kernel launches.  Nothing here
// allocates device memory, synchronises, or reads device results.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "twilight.h"
#include "tw_kernels.h"
#include "tw_label.h"

namespace {

thread_local int g_last_cuda = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda = (int)e;
  return TW_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Per-device cache: 0 = unknown, -1 = unsupported, >0 = SM count.
std::atomic<int> g_dev_sms[128];

int device_check(int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 128) return TW_ERR_UNSUPPORTED;
  int v = g_dev_sms[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e);
    v = (major == 10 && minor == 0 && sms > 0) ? sms : -1;
    g_dev_sms[dev].store(v, std::memory_order_relaxed);
  }
  if (v < 0) return TW_ERR_UNSUPPORTED;
  if (num_sms) *num_sms = v;
  return TW_OK;
}

int check_kv(const tw_kv* kv, bool need_k, bool need_v, tw::Layout* L) {
  if (!kv) return TW_ERR_INVALID_ARG;
  if (kv->head_dim != tw::kHeadDim || kv->page_size != tw::kPage) return TW_ERR_UNSUPPORTED;
  if (kv->batch < 0 || kv->num_kv_heads < 1 || kv->max_seq_len < 0) return TW_ERR_INVALID_ARG;
  if (kv->key_bits != 0 && kv->key_bits != 4 && kv->key_bits != 2) return TW_ERR_UNSUPPORTED;
  if (need_k && (!kv->k || !aligned(kv->k, 16))) return TW_ERR_INVALID_ARG;
  if (need_v && (!kv->v || !aligned(kv->v, 16))) return TW_ERR_INVALID_ARG;
  if (kv->seq_lens && !aligned(kv->seq_lens, 4)) return TW_ERR_INVALID_ARG;
  if (kv->page_table) {
    if (!aligned(kv->page_table, 4) || kv->max_pages_per_seq < 1 || kv->num_pool_pages < 1 ||
        (int64_t)kv->max_seq_len != (int64_t)kv->max_pages_per_seq * tw::kPage)
      return TW_ERR_INVALID_ARG;
  }
  // physical rows are 32-bit indices (row lists between the kernels)
  const int64_t nrows = kv->page_table ? (int64_t)kv->num_pool_pages * kv->num_kv_heads * tw::kPage
                                       : (int64_t)kv->batch * kv->num_kv_heads * kv->max_seq_len;
  if (nrows >= (int64_t)tw::kNoRow) return TW_ERR_UNSUPPORTED;
  L->B = kv->batch;
  L->Hk = kv->num_kv_heads;
  L->N = kv->max_seq_len;
  L->seq_lens = kv->seq_lens;
  L->page_table = kv->page_table;
  L->max_pages = kv->page_table ? kv->max_pages_per_seq : (kv->max_seq_len + tw::kPage - 1) / tw::kPage;
  L->pool_pages = kv->page_table ? kv->num_pool_pages : 0;
  L->kbits = kv->key_bits == 2 ? 2 : 4;
  return TW_OK;
}

int check_heads(int Hq, int Hk) {
  if (Hq < 1 || Hq % Hk != 0) return TW_ERR_INVALID_ARG;
  const int G = Hq / Hk;
  if (G != 1 && G != 2 && G != 4 && G != 8) return TW_ERR_UNSUPPORTED;
  return TW_OK;
}

// Workspace regions, in order: status word | logits of the selection sets
// that exceed shared memory | score keys of caches too long for shared memory
// | physical rows of the kept tokens | per-set completion counters |
// attention partial records.  The status word collects device-side error bits
// (a bounded wait that gave up); the caller zeroes it once after allocating.
// tw_topp_prune uses the regions up to topp_end, tw_select_pages up to
// scores_end.
struct Plan {
  size_t status_off, logits_off, keys_off, rows_off, done_off, part_off;
  size_t topp_end, scores_end, total;
  int lcap;
};

Plan make_plan(int B, int Hq, int Hk, int N, int cap) {
  Plan p;
  const int G = Hq / Hk;
  const int64_t pmax = (N + tw::kPage - 1) / tw::kPage;
  p.lcap = (int)(((int64_t)cap + 63) / 64 * 64);
  p.status_off = 0;
  p.logits_off = 256;
  p.topp_end = p.logits_off + align256((size_t)B * Hk * G * (size_t)p.lcap * sizeof(float));
  p.keys_off = p.topp_end;
  p.scores_end = p.keys_off + align256((size_t)B * Hk * pmax * sizeof(uint32_t));
  const size_t nsets = (size_t)B * (Hq > Hk ? Hq : Hk);
  p.rows_off = p.scores_end;
  p.done_off = p.rows_off + align256(nsets * (size_t)cap * sizeof(uint32_t));
  p.part_off = p.done_off + align256(nsets * sizeof(int32_t));
  p.total = p.part_off + align256(tw::decode_part_floats(B, Hq, Hk) * sizeof(float));
  return p;
}

char* wsp(void* ws, size_t off) { return static_cast<char*>(ws) + off; }

struct Marker {
  void* const* ev;
  int n;
  cudaStream_t st;
  int next = 0;
  cudaError_t mark() {
    if (!ev) return cudaSuccess;
    if (next >= n) return cudaErrorInvalidValue;
    return cudaEventRecord(static_cast<cudaEvent_t>(ev[next++]), st);
  }
};

int check_launch() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TW_OK : cuda_fail(e);
}

#define TW_TRY(x)               \
  do {                          \
    const int _s = (x);         \
    if (_s != TW_OK) return _s; \
  } while (0)

// ---------------------------------------------------------------------------
// Argument checks shared by the single calls and the fused step.

int check_select(const uint16_t* q, int Hq, const tw::Layout& L, const uint16_t* meta,
                 int budget, const int32_t* cand, int cand_stride, const int32_t* ncand) {
  TW_TRY(check_heads(Hq, L.Hk));
  if (!q || !aligned(q, 16) || !meta || !aligned(meta, 16)) return TW_ERR_INVALID_ARG;
  if (budget < tw::kPage) return TW_ERR_INVALID_ARG;
  if (!cand || !aligned(cand, 4) || !ncand || !aligned(ncand, 4)) return TW_ERR_INVALID_ARG;
  const int kp = budget / tw::kPage < L.max_pages ? budget / tw::kPage : L.max_pages;
  if (cand_stride < kp || cand_stride < 1) return TW_ERR_CAPACITY;
  return TW_OK;
}

int candidates_max(const tw::Layout& L, const int32_t* cand, int cand_stride) {
  if (!cand) return L.N;
  const int rows = cand_stride < L.max_pages ? cand_stride : L.max_pages;
  return rows * tw::kPage;
}

int check_topp(const uint16_t* q, int Hq, const tw::Layout& L, const uint8_t* codes,
               const uint16_t* scales, const uint16_t* zeros, const int32_t* cand,
               int cand_stride, const int32_t* ncand, double p, int group_mode, int32_t* idx,
               int capacity, int32_t* count) {
  TW_TRY(check_heads(Hq, L.Hk));
  if (!q || !aligned(q, 16)) return TW_ERR_INVALID_ARG;
  if (!codes || !aligned(codes, 16) || !scales || !aligned(scales, 16) || !zeros ||
      !aligned(zeros, 16))
    return TW_ERR_INVALID_ARG;
  if (cand && (!aligned(cand, 4) || !ncand || !aligned(ncand, 4) || cand_stride < 1))
    return TW_ERR_INVALID_ARG;
  if (!(p > 0.0) || !(p <= 1.0)) return TW_ERR_INVALID_ARG;
  if (group_mode != 0 && group_mode != 1) return TW_ERR_INVALID_ARG;
  if (!idx || !aligned(idx, 4) || !count || !aligned(count, 4) || capacity < 1)
    return TW_ERR_INVALID_ARG;
  const int cmax = candidates_max(L, cand, cand_stride);
  if (capacity < cmax) return TW_ERR_CAPACITY;
  if (cmax > tw::kMaxSetCandidates) return TW_ERR_UNSUPPORTED;
  return TW_OK;
}

int check_decode(const uint16_t* q, int Hq, const tw::Layout& L, const int32_t* idx,
                 int capacity, const int32_t* count, int group_mode, uint16_t* out,
                 float* lse) {
  TW_TRY(check_heads(Hq, L.Hk));
  if (!q || !aligned(q, 16) || !idx || !aligned(idx, 4) || !count || !aligned(count, 4))
    return TW_ERR_INVALID_ARG;
  if (capacity < 1 || (group_mode != 0 && group_mode != 1)) return TW_ERR_INVALID_ARG;
  if (!out || !aligned(out, 16) || (lse && !aligned(lse, 4))) return TW_ERR_INVALID_ARG;
  return TW_OK;
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return TW_OK;
  if (!ws || !aligned(ws, 256)) return TW_ERR_INVALID_ARG;
  if (ws_bytes < need) return TW_ERR_CAPACITY;
  return TW_OK;
}

int group_sets_of(int Hq, int Hk, int group_mode) { return (group_mode || Hq == Hk) ? 1 : 0; }

// Selection-stage arguments shared by every call: layout, query and the
// workspace status word.
tw::SpArgs sp_args(const tw::Layout& L, const uint16_t* q, int Hq, void* ws, const Plan& plan) {
  tw::SpArgs a;
  std::memset(&a, 0, sizeof(a));
  a.L = L;
  a.q = reinterpret_cast<const __half*>(q);
  a.Hq = Hq;
  a.status = reinterpret_cast<int*>(wsp(ws, plan.status_off));
  return a;
}

void set_prune(tw::SpArgs* a, const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros,
               int group_sets, double p, int32_t* idx, uint32_t* rows, int icap, int32_t* count,
               int32_t* done) {
  a->codes = codes;
  a->scales = reinterpret_cast<const __half*>(scales);
  a->zeros = reinterpret_cast<const __half*>(zeros);
  a->group_sets = group_sets;
  a->p = p;
  a->idx = idx;
  a->rows = rows;
  a->icap = icap;
  a->count = count;
  a->done = done;
}

// Candidate pages per unit at most: the Quest budget, the caller's list
// stride, or every page.
int selection_pages(const tw::SpArgs& a) {
  const int mp = a.L.max_pages;
  if (a.meta) return a.budget_pages < mp ? a.budget_pages : mp;
  if (a.cand) return a.cand_stride < mp ? a.cand_stride : mp;
  return mp;
}

// Launch the selection stages on one cluster per unit, with the keys and
// logits in the workspace when they exceed shared memory.
int run_select_prune(tw::SpArgs* a, void* ws, const Plan& plan, int sms, cudaStream_t st,
                     bool pdl) {
  const int sel = selection_pages(*a);
  if (sel > tw::select_prune_max_pages()) return TW_ERR_UNSUPPORTED;
  a->gkeys = reinterpret_cast<uint32_t*>(wsp(ws, plan.keys_off));
  a->glogits = reinterpret_cast<float*>(wsp(ws, plan.logits_off));
  a->lcap = plan.lcap;
  const cudaError_t e = tw::launch_select_prune(*a, sel, sms, st, pdl);
  return e == cudaSuccess ? TW_OK : cuda_fail(e);
}

// Device address of the page-locked host memory at p (allocated or registered
// page-locked and mapped into the device's address space); nullptr for
// pageable, device or unknown memory.
const void* host_mapped(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

// The fused step, optionally recording an event before the first kernel and
// after each kernel, and optionally staging q in from and out back to
// page-locked host memory with copy kernels in the same launch chain.
int decode_step_impl(const tw_step* s, void* const* events, int n_events, cudaStream_t st,
                     const uint16_t* q_host = nullptr, uint16_t* out_host = nullptr) {
  if (!s) return TW_ERR_INVALID_ARG;
  tw::Layout L;
  TW_TRY(check_kv(&s->kv, true, true, &L));
  const int Hq = s->num_q_heads;
  const bool use_select = s->budget_tokens > 0;
  if (use_select)
    TW_TRY(check_select(s->q, Hq, L, s->meta, s->budget_tokens, s->cand_pages, s->cand_stride,
                        s->ncand));
  const int32_t* cand = use_select ? s->cand_pages : nullptr;
  TW_TRY(check_topp(s->q, Hq, L, s->codes, s->scales, s->zeros, cand, s->cand_stride, s->ncand,
                    s->p, s->group_mode, s->idx, s->capacity, s->count));
  TW_TRY(check_decode(s->q, Hq, L, s->idx, s->capacity, s->count, s->group_mode, s->out, s->lse));
  const void* q_in = nullptr;
  void* out_back = nullptr;
  if (q_host || out_host) {
    if (!q_host || !out_host || !aligned(q_host, 16) || !aligned(out_host, 16))
      return TW_ERR_INVALID_ARG;
    if (L.B > 0) {
      q_in = host_mapped(q_host);
      out_back = const_cast<void*>(host_mapped(out_host));
      if (!q_in || !out_back) return TW_ERR_INVALID_ARG;
    }
  }
  if (L.B == 0) return TW_OK;
  const Plan plan = make_plan(L.B, Hq, L.Hk, L.N, s->capacity);
  TW_TRY(check_ws(s->ws, s->ws_bytes, plan.total));
  int sms = 0;
  TW_TRY(device_check(&sms));
  const int64_t qo_bytes = (int64_t)L.B * Hq * tw::kHeadDim * 2;
  const int gs = group_sets_of(Hq, L.Hk, s->group_mode);
  const auto* q = reinterpret_cast<const __half*>(s->q);
  // programmatic dependent launch overlaps each kernel's launch with its
  // predecessor's tail; the profiled variant runs them strictly in order so
  // that each event pair brackets exactly one kernel
  const bool pdl = events == nullptr;
  Marker mk{events, n_events, st};
  cudaError_t e;
  if ((e = mk.mark()) != cudaSuccess) return cuda_fail(e);
  if (q_in) {   // the query comes in from host memory first
    e = tw::launch_copy16(q_in, const_cast<uint16_t*>(s->q), qo_bytes, true, st, pdl);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (s->append_keys) {   // the newest token of every sequence joins the int4 cache and metadata
    e = tw::launch_append_keys(L, reinterpret_cast<const __half*>(s->kv.k),
                               const_cast<uint8_t*>(s->codes),
                               reinterpret_cast<__half*>(const_cast<uint16_t*>(s->scales)),
                               reinterpret_cast<__half*>(const_cast<uint16_t*>(s->zeros)),
                               use_select ? reinterpret_cast<__half*>(const_cast<uint16_t*>(s->meta))
                                          : nullptr,
                               st, sms, pdl);
    if (e != cudaSuccess || (e = mk.mark()) != cudaSuccess) return cuda_fail(e);
  }
  uint32_t* rows = reinterpret_cast<uint32_t*>(wsp(s->ws, plan.rows_off));
  int32_t* done = reinterpret_cast<int32_t*>(wsp(s->ws, plan.done_off));
  tw::SpArgs a = sp_args(L, s->q, Hq, s->ws, plan);
  if (use_select) {
    a.meta = reinterpret_cast<const __half*>(s->meta);
    a.budget_pages = s->budget_tokens / tw::kPage;
    a.cand = s->cand_pages;
    a.cand_stride = s->cand_stride;
    a.ncand = s->ncand;
  }
  set_prune(&a, s->codes, s->scales, s->zeros, gs, s->p, s->idx, rows, s->capacity, s->count,
            done);
  TW_TRY(run_select_prune(&a, s->ws, plan, sms, st, pdl));
  if ((e = mk.mark()) != cudaSuccess) return cuda_fail(e);
  float* part = reinterpret_cast<float*>(wsp(s->ws, plan.part_off));
  const auto* K = reinterpret_cast<const __half*>(s->kv.k);
  const auto* V = reinterpret_cast<const __half*>(s->kv.v);
  auto* out = reinterpret_cast<__half*>(s->out);
  e = tw::launch_sparse_decode(L, q, Hq, gs, K, V, rows, s->capacity, s->count, part, done, out,
                               s->lse, st, pdl);
  if (e != cudaSuccess || (e = mk.mark()) != cudaSuccess) return cuda_fail(e);
  if (out_back) {   // and the attention output goes back to host memory last
    e = tw::launch_copy16(out, out_back, qo_bytes, false, st, pdl);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return check_launch();
}

// Workspace of tw_topp_prune_tokens: the pruner's own regions for the
// contiguous cache of candidate rows (B * Hk one-head sequences of cand_stride
// rows, G query heads each), then that cache's codes, scales and zeros.
struct TokenPlan {
  Plan topp;
  size_t vcodes_off, vscales_off, vzeros_off, total;
};

TokenPlan make_token_plan(int B, int Hq, int Hk, int cand_stride, int capacity, int kbits) {
  TokenPlan t;
  t.topp = make_plan(B * Hk, Hq / Hk, 1, cand_stride, capacity);
  const size_t rows = (size_t)B * Hk * cand_stride;
  t.vcodes_off = align256(t.topp.scores_end);
  t.vscales_off = t.vcodes_off + align256(rows * (size_t)(tw::kHeadDim * kbits / 8));
  t.vzeros_off = t.vscales_off + align256(rows * tw::kGroups * sizeof(uint16_t));
  t.total = t.vzeros_off + align256(rows * tw::kGroups * sizeof(uint16_t));
  return t;
}

size_t label_scores_bytes(int B, int Hk, int N) {
  return align256((size_t)B * Hk * N * sizeof(float));
}

}  // namespace

extern "C" {

const char* tw_status_string(int status) {
  switch (status) {
    case TW_OK: return "TW_OK";
    case TW_ERR_INVALID_ARG: return "TW_ERR_INVALID_ARG: null/misaligned pointer or bad parameter";
    case TW_ERR_UNSUPPORTED: return "TW_ERR_UNSUPPORTED: shape or device not supported";
    case TW_ERR_CAPACITY: return "TW_ERR_CAPACITY: output or workspace buffer too small";
    case TW_ERR_CUDA: return "TW_ERR_CUDA: a CUDA call failed";
    case TW_ERR_TIMEOUT: return "TW_ERR_TIMEOUT: a bounded device wait gave up";
    default: return "unknown tw_status";
  }
}

int tw_last_cuda_error(void) { return g_last_cuda; }

int tw_version(void) { return 101; }

int tw_selftest_bounded_wait(int32_t* status, void* stream) {
  if (!status || (reinterpret_cast<uintptr_t>(status) & 3)) return TW_ERR_INVALID_ARG;
  const cudaError_t e = tw::launch_wait_selftest(status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TW_OK : cuda_fail(e);
}

int tw_quantize_keys(const tw_kv* kv, uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                     void* stream) {
  tw::Layout L;
  TW_TRY(check_kv(kv, true, false, &L));
  if (!codes || !aligned(codes, 16) || !scales || !aligned(scales, 16) || !zeros ||
      !aligned(zeros, 16))
    return TW_ERR_INVALID_ARG;
  if ((int64_t)L.B * L.N == 0) return TW_OK;
  int sms = 0;
  TW_TRY(device_check(&sms));
  tw::launch_quantize_keys(L, reinterpret_cast<const __half*>(kv->k), codes,
                           reinterpret_cast<__half*>(scales), reinterpret_cast<__half*>(zeros),
                           static_cast<cudaStream_t>(stream), sms);
  return check_launch();
}

int tw_page_meta(const tw_kv* kv, uint16_t* meta, void* stream) {
  tw::Layout L;
  TW_TRY(check_kv(kv, true, false, &L));
  if (!meta || !aligned(meta, 16)) return TW_ERR_INVALID_ARG;
  if ((int64_t)L.B * L.N == 0) return TW_OK;
  int sms = 0;
  TW_TRY(device_check(&sms));
  tw::launch_page_meta(L, reinterpret_cast<const __half*>(kv->k), reinterpret_cast<__half*>(meta),
                       static_cast<cudaStream_t>(stream), sms);
  return check_launch();
}

int tw_append_keys(const tw_kv* kv, uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                   uint16_t* meta, void* stream) {
  tw::Layout L;
  TW_TRY(check_kv(kv, true, false, &L));
  if (!codes != !scales || !codes != !zeros) return TW_ERR_INVALID_ARG;
  if ((codes && (!aligned(codes, 16) || !aligned(scales, 16) || !aligned(zeros, 16))) ||
      (meta && !aligned(meta, 16)))
    return TW_ERR_INVALID_ARG;
  if ((int64_t)L.B * L.N == 0 || (!codes && !meta)) return TW_OK;
  int sms = 0;
  TW_TRY(device_check(&sms));
  const cudaError_t e = tw::launch_append_keys(
      L, reinterpret_cast<const __half*>(kv->k), codes, reinterpret_cast<__half*>(scales),
      reinterpret_cast<__half*>(zeros), reinterpret_cast<__half*>(meta),
      static_cast<cudaStream_t>(stream), sms, false);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch();
}

int tw_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                      int32_t max_seq_len, int32_t capacity, size_t* bytes) {
  if (!bytes || batch < 0 || num_kv_heads < 1 || max_seq_len < 0 || capacity < 1)
    return TW_ERR_INVALID_ARG;
  TW_TRY(check_heads(num_q_heads, num_kv_heads));
  *bytes = make_plan(batch, num_q_heads, num_kv_heads, max_seq_len, capacity).total;
  return TW_OK;
}

int tw_select_pages(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                    const uint16_t* meta, int32_t budget_tokens, int32_t* cand_pages,
                    int32_t cand_stride, int32_t* ncand, void* ws, size_t ws_bytes,
                    void* stream) {
  tw::Layout L;
  TW_TRY(check_kv(kv, false, false, &L));
  TW_TRY(check_select(q, num_q_heads, L, meta, budget_tokens, cand_pages, cand_stride, ncand));
  if (L.B == 0) return TW_OK;
  const Plan plan = make_plan(L.B, num_q_heads, L.Hk, L.N, 1);
  TW_TRY(check_ws(ws, ws_bytes, plan.scores_end));
  int sms = 0;
  TW_TRY(device_check(&sms));
  tw::SpArgs a = sp_args(L, q, num_q_heads, ws, plan);
  a.meta = reinterpret_cast<const __half*>(meta);
  a.budget_pages = budget_tokens / tw::kPage;
  a.cand = cand_pages;
  a.cand_stride = cand_stride;
  a.ncand = ncand;
  TW_TRY(run_select_prune(&a, ws, plan, sms, static_cast<cudaStream_t>(stream), false));
  return check_launch();
}

int tw_topp_prune(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                  const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros,
                  const int32_t* cand_pages, int32_t cand_stride, const int32_t* ncand,
                  double p, int32_t group_mode, int32_t* idx, int32_t capacity, int32_t* count,
                  void* ws, size_t ws_bytes, void* stream) {
  tw::Layout L;
  TW_TRY(check_kv(kv, false, false, &L));
  TW_TRY(check_topp(q, num_q_heads, L, codes, scales, zeros, cand_pages, cand_stride, ncand, p,
                    group_mode, idx, capacity, count));
  if (L.B == 0) return TW_OK;
  const Plan plan = make_plan(L.B, num_q_heads, L.Hk, L.N, capacity);
  TW_TRY(check_ws(ws, ws_bytes, plan.topp_end));
  int sms = 0;
  TW_TRY(device_check(&sms));
  tw::SpArgs a = sp_args(L, q, num_q_heads, ws, plan);
  a.cand = const_cast<int32_t*>(cand_pages);
  a.cand_stride = cand_stride;
  a.ncand = const_cast<int32_t*>(ncand);
  set_prune(&a, codes, scales, zeros, group_sets_of(num_q_heads, L.Hk, group_mode), p, idx,
            nullptr, capacity, count, nullptr);
  TW_TRY(run_select_prune(&a, ws, plan, sms, static_cast<cudaStream_t>(stream), false));
  return check_launch();
}

int tw_sparse_decode(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                     const int32_t* idx, int32_t capacity, const int32_t* count,
                     int32_t group_mode, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                     void* stream) {
  tw::Layout L;
  TW_TRY(check_kv(kv, true, true, &L));
  TW_TRY(check_decode(q, num_q_heads, L, idx, capacity, count, group_mode, out, lse));
  if (L.B == 0) return TW_OK;
  const Plan plan = make_plan(L.B, num_q_heads, L.Hk, L.N, capacity);
  TW_TRY(check_ws(ws, ws_bytes, plan.total));
  TW_TRY(device_check(nullptr));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* part = reinterpret_cast<float*>(wsp(ws, plan.part_off));
  int32_t* done = reinterpret_cast<int32_t*>(wsp(ws, plan.done_off));
  const int gs = group_sets_of(num_q_heads, L.Hk, group_mode);
  const int nsets = gs ? L.B * L.Hk : L.B * num_q_heads;
  const auto* K = reinterpret_cast<const __half*>(kv->k);
  const auto* V = reinterpret_cast<const __half*>(kv->v);
  uint32_t* rows = reinterpret_cast<uint32_t*>(wsp(ws, plan.rows_off));
  cudaError_t e = cudaMemsetAsync(done, 0, (size_t)nsets * sizeof(int32_t), st);
  if (e == cudaSuccess)   // caller-given token ids: map them to physical rows first
    e = tw::launch_resolve_rows(L, num_q_heads, gs, idx, capacity, count, rows, st, false);
  if (e == cudaSuccess)
    e = tw::launch_sparse_decode(L, reinterpret_cast<const __half*>(q), num_q_heads, gs, K, V,
                                 rows, capacity, count, part, done,
                                 reinterpret_cast<__half*>(out), lse, st, false);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch();
}

int tw_label_cache(const tw_kv* kv, const int32_t* channels, int32_t r, uint16_t* labels,
                   void* stream) {
  tw::Layout L;
  TW_TRY(check_kv(kv, true, false, &L));
  if (!channels || !aligned(channels, 4) || !labels || !aligned(labels, 2))
    return TW_ERR_INVALID_ARG;
  if (r < 1 || r > tw::kMaxLabelChannels) return TW_ERR_UNSUPPORTED;
  if ((int64_t)L.B * L.N == 0) return TW_OK;
  int sms = 0;
  TW_TRY(device_check(&sms));
  const cudaError_t e =
      tw::launch_label_cache(L, reinterpret_cast<const __half*>(kv->k), channels, r,
                             reinterpret_cast<__half*>(labels), static_cast<cudaStream_t>(stream),
                             sms);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch();
}

int tw_token_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t max_seq_len, int32_t cand_stride, int32_t capacity,
                            int32_t key_bits, size_t* bytes) {
  if (!bytes || batch < 0 || num_kv_heads < 1 || max_seq_len < 0 || cand_stride < 1 ||
      capacity < cand_stride)
    return TW_ERR_INVALID_ARG;
  if (key_bits != 0 && key_bits != 2 && key_bits != 4) return TW_ERR_UNSUPPORTED;
  TW_TRY(check_heads(num_q_heads, num_kv_heads));
  const size_t a = label_scores_bytes(batch, num_kv_heads, max_seq_len);
  const size_t b = make_token_plan(batch, num_q_heads, num_kv_heads, cand_stride, capacity,
                                   key_bits == 2 ? 2 : 4).total;
  *bytes = a > b ? a : b;
  return TW_OK;
}

int tw_select_tokens(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                     const uint16_t* labels, const int32_t* channels, int32_t r,
                     int32_t budget_tokens, int32_t* cand_tokens, int32_t cand_stride,
                     int32_t* ncand, void* ws, size_t ws_bytes, void* stream) {
  tw::Layout L;
  TW_TRY(check_kv(kv, false, false, &L));
  TW_TRY(check_heads(num_q_heads, L.Hk));
  if (!q || !aligned(q, 16) || !labels || !aligned(labels, 2) || !channels ||
      !aligned(channels, 4) || !cand_tokens || !aligned(cand_tokens, 4) || !ncand ||
      !aligned(ncand, 4))
    return TW_ERR_INVALID_ARG;
  if (r < 1 || r > tw::kMaxLabelChannels) return TW_ERR_UNSUPPORTED;
  if (budget_tokens < 1) return TW_ERR_INVALID_ARG;
  const int keep = budget_tokens < L.N ? budget_tokens : L.N;
  if (cand_stride < keep || cand_stride < 1) return TW_ERR_CAPACITY;
  if ((int64_t)L.B * L.Hk > 65535) return TW_ERR_UNSUPPORTED;
  if (L.B == 0) return TW_OK;
  TW_TRY(check_ws(ws, ws_bytes, label_scores_bytes(L.B, L.Hk, L.N)));
  TW_TRY(device_check(nullptr));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* scores = reinterpret_cast<float*>(ws);
  cudaError_t e = tw::launch_label_scores(L, reinterpret_cast<const __half*>(q), num_q_heads,
                                          reinterpret_cast<const __half*>(labels), channels, r,
                                          scores, st);
  if (e == cudaSuccess)
    e = tw::launch_token_topk(L, scores, budget_tokens, cand_tokens, cand_stride, ncand, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch();
}

int tw_topp_prune_tokens(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                         const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros,
                         const int32_t* cand_tokens, int32_t cand_stride, const int32_t* ncand,
                         double p, int32_t group_mode, int32_t* idx, int32_t capacity,
                         int32_t* count, void* ws, size_t ws_bytes, void* stream) {
  tw::Layout L;
  TW_TRY(check_kv(kv, false, false, &L));
  TW_TRY(check_heads(num_q_heads, L.Hk));
  if (!cand_tokens || !aligned(cand_tokens, 4) || !ncand || !aligned(ncand, 4) ||
      cand_stride < 1)
    return TW_ERR_INVALID_ARG;
  if ((int64_t)L.B * L.Hk * cand_stride >= (int64_t)tw::kNoRow) return TW_ERR_UNSUPPORTED;
  // the candidate rows form a contiguous cache of B * Hk one-head sequences
  // (lengths ncand) of cand_stride rows, on which the page-free pruner runs
  const int G = num_q_heads / L.Hk;
  tw::Layout Lv;
  Lv.B = L.B * L.Hk;
  Lv.Hk = 1;
  Lv.N = cand_stride;
  Lv.seq_lens = ncand;
  Lv.page_table = nullptr;
  Lv.max_pages = (cand_stride + tw::kPage - 1) / tw::kPage;
  Lv.pool_pages = 0;
  Lv.kbits = L.kbits;
  TW_TRY(check_topp(q, G, Lv, codes, scales, zeros, nullptr, 0, nullptr, p, group_mode, idx,
                    capacity, count));
  if (L.B == 0) return TW_OK;
  const TokenPlan plan = make_token_plan(L.B, num_q_heads, L.Hk, cand_stride, capacity, L.kbits);
  TW_TRY(check_ws(ws, ws_bytes, plan.total));
  int sms = 0;
  TW_TRY(device_check(&sms));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* vcodes = reinterpret_cast<uint8_t*>(wsp(ws, plan.vcodes_off));
  auto* vscales = reinterpret_cast<__half*>(wsp(ws, plan.vscales_off));
  auto* vzeros = reinterpret_cast<__half*>(wsp(ws, plan.vzeros_off));
  const int gs = group_sets_of(num_q_heads, L.Hk, group_mode);
  const int nsets = gs ? L.B * L.Hk : L.B * num_q_heads;
  cudaError_t e = tw::launch_gather_keys(L, cand_tokens, cand_stride, ncand, codes,
                                         reinterpret_cast<const __half*>(scales),
                                         reinterpret_cast<const __half*>(zeros), vcodes, vscales,
                                         vzeros, st, sms);
  if (e != cudaSuccess) return cuda_fail(e);
  tw::SpArgs a = sp_args(Lv, q, G, ws, plan.topp);
  set_prune(&a, vcodes, reinterpret_cast<const uint16_t*>(vscales),
            reinterpret_cast<const uint16_t*>(vzeros), gs, p, idx, nullptr, capacity, count,
            nullptr);
  TW_TRY(run_select_prune(&a, ws, plan.topp, sms, st, false));
  e = tw::launch_map_tokens(nsets, G, gs, cand_tokens, cand_stride, idx, capacity, count, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch();
}

int tw_decode_step(const tw_step* step, void* stream) {
  return decode_step_impl(step, nullptr, 0, static_cast<cudaStream_t>(stream));
}

int tw_decode_step_host(const tw_step* step, const uint16_t* q_host, uint16_t* out_host,
                        void* stream) {
  if (!q_host || !out_host) return TW_ERR_INVALID_ARG;
  return decode_step_impl(step, nullptr, 0, static_cast<cudaStream_t>(stream), q_host, out_host);
}

int tw_decode_step_num_kernels(const tw_step* step) {
  if (!step) return -TW_ERR_INVALID_ARG;
  return 2 + (step->append_keys ? 1 : 0);
}

const char* tw_decode_step_kernel_name(const tw_step* step, int32_t i) {
  if (!step) return nullptr;
  if (step->append_keys) {
    if (i == 0) return "append_keys";
    --i;
  }
  if (i == 0) return step->budget_tokens > 0 ? "select_prune" : "prune";
  return i == 1 ? "sparse_decode" : nullptr;
}

int tw_decode_step_profiled(const tw_step* step, void* const* events, int32_t n_events,
                            void* stream) {
  if (!events || n_events < tw_decode_step_num_kernels(step) + 1) return TW_ERR_INVALID_ARG;
  return decode_step_impl(step, events, n_events, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
