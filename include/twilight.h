/*
 * twilight.h -- C ABI of the B200 (sm_100a) decode path of Twilight's
 * hierarchical top-p attention pruning.
 *
 * Method: "Twilight: Adaptive Attention Sparsity with Hierarchical Top-p
 * Pruning" (arXiv 2502.02770).  A base sparse-attention selector (here Quest:
 * pages ranked by a per-page key min/max bound) pre-selects candidate tokens;
 * top-p (nucleus) thresholding over the candidates' attention weights, which
 * are estimated from a 4-bit key cache, prunes them further; exact attention
 * then runs over the survivors only (atlas.scime.ai summary, "Approach";
 * group-wise budgets under GQA: "Limitations").  A 2-bit key cache, the width
 * the quantisation ablation compares 4-bit against (table of measured
 * effects), is selected with tw_kv.key_bits = 2.
 *
 * Conventions shared by every call
 *   - Every function returns a tw_status (0 = TW_OK).  Host-side argument
 *     checks run before anything is launched; on an error nothing is launched
 *     and no output is touched.  TW_ERR_CUDA keeps the CUDA error code, read it
 *     with tw_last_cuda_error() (per host thread).
 *   - All data pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned.  The library allocates no memory; scratch comes from a caller
 *     workspace sized by tw_workspace_size().
 *   - The first 4 bytes of a workspace are a device status word.  Zero it
 *     once after allocating; the kernels only set bits in it.  Bit 0: a
 *     bounded wait of the selection kernel (0.2 s on one pipeline stage) gave
 *     up, and that call's outputs are invalid; a caller that reads the word
 *     after synchronising reports it as TW_ERR_TIMEOUT.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     only enqueue work and return; they never synchronise and never read
 *     device results on the host.
 *   - fp16 data is passed as uint16_t (IEEE binary16 bit patterns).
 *   - head_dim must be 128 and page_size 16 (TW_ERR_UNSUPPORTED otherwise);
 *     the device must be compute capability 10.0 (sm_100a).
 *   - Inputs must be finite; NaN or Inf in q, K or V gives unspecified results.
 *
 * Layouts (element = fp16 unless stated; b = sequence, h = KV head,
 * t = token, pg = logical page = t / 16, N = max_seq_len)
 *   contiguous (page_table == NULL):
 *     K, V        [B][Hk][N][128]
 *     codes (u8)  [B][Hk][N][64]   channel 2i in the low nibble of byte i
                                 (key_bits 2: [B][Hk][N][32], channel 4i + j in
                                 bits 2j, 2j + 1 of byte i)
 *     scales      [B][Hk][N][4]    one per group of 32 channels
 *     zeros       [B][Hk][N][4]
 *     meta        [B][Hk][ceil(N/16)][2][128]   row 0 = min, row 1 = max
 *   paged (page_table != NULL), pool page P = page_table[b][pg]:
 *     K, V        [num_pool_pages][Hk][16][128]
 *     codes       [num_pool_pages][Hk][16][64]   (key_bits 2: [..][32])
 *     scales      [num_pool_pages][Hk][16][4]
 *     zeros       [num_pool_pages][Hk][16][4]
 *     meta        [num_pool_pages][Hk][2][128]
 *   q      [B][Hq][128];  out [B][Hq][128];  lse (fp32) [B][Hq]
 *   Hq is a multiple of Hk; G = Hq / Hk query heads share a KV head
 *   (G in {1, 2, 4, 8}).
 *
 * Selection sets.  With group_mode = 1 (or G = 1) one top-p set is formed per
 * (b, KV head): "selection unit" u = b * Hk + h.  With group_mode = 0 and
 * G > 1 each query head has its own set: u = b * Hq + hq.  idx / count are
 * indexed by u.
 */
#ifndef TWILIGHT_H
#define TWILIGHT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tw_status {
  TW_OK = 0,
  TW_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or parameter */
  TW_ERR_UNSUPPORTED = 2,   /* head_dim != 128, page_size != 16, G not in {1,2,4,8},
                               candidates per set > 131072, device not sm_100 */
  TW_ERR_CAPACITY = 3,      /* an output or workspace buffer is too small */
  TW_ERR_CUDA = 4,          /* a CUDA call failed; see tw_last_cuda_error() */
  TW_ERR_TIMEOUT = 5        /* a bounded device wait gave up (workspace status word) */
} tw_status;

/* KV-cache descriptor (see "Layouts" above).  Used by every call. */
typedef struct tw_kv {
  const void* k;              /* fp16 keys (device); required by quantize/meta/decode */
  const void* v;              /* fp16 values (device); required by sparse_decode only */
  int32_t batch;              /* B >= 0 */
  int32_t num_kv_heads;       /* Hk >= 1 */
  int32_t max_seq_len;        /* N: contiguous: tokens allocated per sequence;
                                 paged: must equal max_pages_per_seq * 16 */
  const int32_t* seq_lens;    /* device [B] valid lengths in [0, N]; NULL = all N */
  const int32_t* page_table;  /* device [B][max_pages_per_seq]; NULL = contiguous.
                                 Entries for pages past a sequence's end are never read. */
  int32_t max_pages_per_seq;  /* row stride of page_table (paged only) */
  int32_t num_pool_pages;     /* pages in the pool (paged only) */
  int32_t page_size;          /* must be 16 */
  int32_t head_dim;           /* must be 128 */
  int32_t key_bits;           /* width of the quantised key cache: 4 (or 0, read as 4)
                                 or 2; any other value gives TW_ERR_UNSUPPORTED */
} tw_kv;

/* Name of a status code (static string). */
const char* tw_status_string(int status);

/* The cudaError_t of the last TW_ERR_CUDA returned on this host thread. */
int tw_last_cuda_error(void);

/*
 * Diagnostic: runs one device wait that nothing completes, bounded as the
 * selection kernel's ring waits are (0.2 s).  The wait gives up, sets bit 0
 * of *status (a device int32 the caller zeroed) and the kernel returns
 * normally; bit 1 would mean the wait did not give up.  The CUDA context stays
 * usable.  Enqueues on `stream` and returns; read *status after
 * synchronising.
 */
int tw_selftest_bounded_wait(int32_t* status, void* stream);

/* Library ABI version (major * 100 + minor). */
int tw_version(void);

/*
 * Build the quantised key cache (prefill-time, once per token).
 * Source: the 4-bit key cache used to estimate attention weights
 * (atlas.scime.ai summary, "Approach"; 4-bit preferred to 2-bit, table of
 * measured effects; about 1/8 extra KV memory, "Limitations").
 * Per token and group of 32 channels, in IEEE fp32 round-to-nearest, with
 * n = 15 (kv->key_bits 4) or 3 (kv->key_bits 2):
 *   mn, mx = exact fp16 min / max (totalOrder: -0 < +0)
 *   scale = fp16_rn((mx - mn) / n),  zero = mn,
 *   code  = clamp(round_half_even((x - mn) / scale), 0, n), 0 if scale == 0.
 * codes are packed as "Layouts" states for the width.
 * Reads kv->k for tokens t < seq_lens[b]; writes codes/scales/zeros at the same
 * positions (other positions are left untouched).  Bit-exact with the CPU
 * definition.
 */
int tw_quantize_keys(const tw_kv* kv, uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                     void* stream);

/*
 * Build Quest page metadata: for each page of 16 tokens with at least one
 * valid token, the channel-wise exact fp16 min and max of K over its valid
 * tokens (Quest's per-page layout, atlas.scime.ai summary, "Surprising
 * findings").  Writes meta for pages pg < ceil(seq_lens[b] / 16).
 */
int tw_page_meta(const tw_kv* kv, uint16_t* meta, void* stream);

/*
 * Incremental decode append: after the caller has written the newest token's
 * K (and V) row at position t = seq_lens[b] - 1 of every sequence b and KV
 * head (and raised seq_lens), quantise that key row into codes / scales /
 * zeros exactly as tw_quantize_keys does, and fold it into the metadata of its
 * page (a page whose first row is t holds only t).  The int4 cache supplies
 * the weight estimate for every cached token (atlas.scime.ai summary,
 * "Approach"); keeping it current one token per step is this library's
 * reading of how a decoder maintains it.  If codes / meta were current for the
 * lengths minus one, the result equals tw_quantize_keys + tw_page_meta for
 * the new lengths bit for bit.  Sequences with seq_lens[b] == 0 are skipped.
 * codes, scales and zeros are all NULL or all set (16-byte aligned); meta may
 * be NULL (metadata not maintained).
 */
int tw_append_keys(const tw_kv* kv, uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                   uint16_t* meta, void* stream);

/*
 * Workspace bytes needed by tw_select_pages / tw_topp_prune / tw_sparse_decode
 * and tw_decode_step for these sizes (the maximum over the calls).
 * capacity: the idx row length that will be passed (>= candidates per set).
 */
int tw_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                      int32_t max_seq_len, int32_t capacity, size_t* bytes);

/*
 * Quest pre-selection (the base selector).  Twilight prunes on top of a base
 * selector, and Quest is one of the two it builds on; Quest ranks 16-token
 * pages by a bound computed from the page's per-channel key min / max (its
 * max-pooled page layout is why Twilight's pruning is hierarchical:
 * atlas.scime.ai summary, "Surprising findings"; "Builds on").  The pages give
 * no formula; the bound below is Quest's published criterion.
 * For each (b, KV head):
 *   score[pg] = sum over the G query heads of the group, in head order, of
 *               sum_j max(q_j * min_j, q_j * max_j)      (fp32, fixed order:
 *               16 chunks of 8 channels summed left to right, then chunk c
 *               added to c+8, then +4, +2, +1)
 *   keep K_p = min(budget_tokens / 16, ceil(len / 16)) pages with the largest
 *   score, ties to the lower page index, written ascending.
 * cand_pages: [B][Hk][cand_stride] int32 logical page ids; ncand: [B][Hk].
 * cand_stride >= min(budget_tokens / 16, ceil(N / 16)); budget_tokens >= 16.
 * Bit-exact page ids with the CPU definition.
 */
int tw_select_pages(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                    const uint16_t* meta, int32_t budget_tokens, int32_t* cand_pages,
                    int32_t cand_stride, int32_t* ncand, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * Twilight's top-p pruner (atlas.scime.ai summary, "Approach"; group-wise
 * under GQA, "Limitations").  Candidates of (b, KV head) are the valid tokens
 * of its cand_pages (ascending), or every token t < len when cand_pages is NULL
 * (base = full attention).  For each candidate i and query head h, with the
 * codes of the cache width kv->key_bits:
 *   l[i,h] = q_h . (zero + scale * code_i) / sqrt(128)          (fp32)
 *   w_h[i] = exp(l[i,h] - max_i l) / sum_i exp(l[i,h] - max_i l)
 * The set's weight is w_h (per-head sets) or the mean of w_h over the G heads
 * (group sets).  The threshold theta is the largest weight value whose
 * retained mass sum_{w >= theta} w reaches p (searched on the fp32 bit pattern
 * of the weights, a few bits per step, with exact integer mass sums at 2^-40
 * resolution); all weights > theta are kept plus the lowest-position ties
 * needed to reach p.  p >= 1 keeps every candidate.
 * idx: [U][capacity] int32 token ids (ascending), count: [U] int32, U as in
 * "Selection sets".  capacity >= candidates per set; p in (0, 1].
 * Candidates per set must be <= 131072.
 */
int tw_topp_prune(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                  const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros,
                  const int32_t* cand_pages, int32_t cand_stride, const int32_t* ncand,
                  double p, int32_t group_mode, int32_t* idx, int32_t capacity, int32_t* count,
                  void* ws, size_t ws_bytes, void* stream);

/*
 * Exact attention over the selected tokens' fp16 K/V (split-K flash decoding
 * with a log-sum-exp merge).  After the base selector and the top-p pruner,
 * attention runs over the surviving tokens only (atlas.scime.ai summary,
 * "Approach": select, then prune, then sparse attention; the authors' kernels
 * build on FlashInfer's sparse attention, "Experimental setup").  For query
 * head hq of sequence b, with S its selection set:
 *   out = sum_{i in S} softmax(q . k_i / sqrt(128)) v_i
 * (fp32 accumulation, fp16 result); lse[b][hq] = log sum exp (natural log).
 * An empty set gives out = 0 and lse = -inf.  lse may be NULL.
 */
int tw_sparse_decode(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                     const int32_t* idx, int32_t capacity, const int32_t* count,
                     int32_t group_mode, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * tw_topp_prune without a workspace, for callers that cannot allocate device
 * memory (a runtime recording the step into a CUDA graph with allocation
 * forbidden, a plugin whose enqueue hook may not allocate, a server that fixes
 * its device memory at start-up).  The paper has no counterpart to this call:
 * it exists only for that calling constraint.
 * Same inputs, outputs and results as tw_topp_prune; the scratch is one fixed
 * array of TW_NOALLOC_SCRATCH_BYTES (8 MiB) compiled into the library, resident
 * on every GPU that loads it until the process exits.  A call needs
 *   256 + align256(B * Hk * G * lcap * 4) bytes of it,
 * lcap = capacity rounded up to a multiple of 64 and align256 rounding up to a
 * multiple of 256 (a status word, then room for the selection sets' logits);
 * a call that needs more returns TW_ERR_CAPACITY before any device work.  The
 * first call on a device looks up the array's device address (TW_ERR_CUDA if
 * that fails) and keeps it for later calls on that device, so make it before
 * any stream capture; the address stays valid for the life of the device's
 * primary context (no cudaDeviceReset between calls).  Every call shares the
 * array: calls that overlap on the GPU race.  Nothing in it needs to start at
 * zero.
 */
#define TW_NOALLOC_SCRATCH_BYTES (8u << 20)
int tw_topp_prune_noalloc(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                          const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros,
                          const int32_t* cand_pages, int32_t cand_stride, const int32_t* ncand,
                          double p, int32_t group_mode, int32_t* idx, int32_t capacity,
                          int32_t* count, void* stream);

/*
 * Token-level label-channel base selector: a synthetic stand-in for Double
 * Sparsity, the other base selector Twilight builds on (atlas.scime.ai
 * summary, "Builds on", "Key results"; the pages give no mechanism, so this
 * follows Double Sparsity's published idea).  Per KV head h, r label channels
 * channels[h][0 .. r) (device int32 [Hk][r], values in [0, 128); out-of-range
 * values are clamped) stand in for offline calibration on trained weights.
 * Use: tw_label_cache once per token (prefill), then per decode step
 * tw_select_tokens -> tw_topp_prune_tokens -> tw_sparse_decode.
 */

/* labels[row][j] = K[row][channels[h][j]] (fp16, r per row, rows addressed
 * like codes: [B][Hk][N][r] contiguous, [num_pool_pages][Hk][16][r] paged) for
 * every valid token.  1 <= r <= 32. */
int tw_label_cache(const tw_kv* kv, const int32_t* channels, int32_t r, uint16_t* labels,
                   void* stream);

/* Workspace bytes for tw_select_tokens and tw_topp_prune_tokens (the maximum
 * of the two) with these sizes; key_bits as in tw_kv. */
int tw_token_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t max_seq_len, int32_t cand_stride, int32_t capacity,
                            int32_t key_bits, size_t* bytes);

/* For each (b, KV head h): score[t] = sum over the G query heads of the group,
 * in head order, of sum_{j = 0 .. r-1, in order} q_hq[c_j] * labels[t][j]
 * (fp32, products exact, each sum rounded), and the min(budget_tokens,
 * len_b) tokens with the largest score (ties to the lower token index)
 * written ascending to cand_tokens[b][h][0 ..), their number to ncand[b][h].
 * cand_stride >= min(budget_tokens, N); budget_tokens >= 1; B * Hk <= 65535.
 * Bit-exact token ids with the CPU definition. */
int tw_select_tokens(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                     const uint16_t* labels, const int32_t* channels, int32_t r,
                     int32_t budget_tokens, int32_t* cand_tokens, int32_t cand_stride,
                     int32_t* ncand, void* ws, size_t ws_bytes, void* stream);

/* tw_topp_prune over token candidates: cand_tokens[b][h][0 .. ncand[b][h])
 * (ascending valid token ids, ncand <= cand_stride) instead of pages.  The
 * same estimate, threshold and tie rule as tw_topp_prune; idx holds token ids
 * (ascending), count the kept numbers.  capacity >= cand_stride; workspace
 * from tw_token_workspace_size.  Token ids outside [0, len) give unspecified
 * results (they read a clamped row, never outside the cache). */
int tw_topp_prune_tokens(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                         const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros,
                         const int32_t* cand_tokens, int32_t cand_stride, const int32_t* ncand,
                         double p, int32_t group_mode, int32_t* idx, int32_t capacity,
                         int32_t* count, void* ws, size_t ws_bytes, void* stream);

/* One decode step: [tw_append_keys when append_keys != 0] -> tw_select_pages
 * (skipped when budget_tokens <= 0, every token is then a candidate) ->
 * tw_topp_prune -> tw_sparse_decode, enqueued back to back on one stream with
 * no host synchronisation.  With append_keys set, codes / scales / zeros (and
 * meta when budget_tokens > 0) must be writable: the step updates them first. */
typedef struct tw_step {
  const uint16_t* q;          /* [B][Hq][128] */
  int32_t num_q_heads;        /* Hq */
  tw_kv kv;
  const uint8_t* codes;       /* int4 key cache (tw_quantize_keys) */
  const uint16_t* scales;
  const uint16_t* zeros;
  const uint16_t* meta;       /* page metadata (tw_page_meta); unused if budget_tokens <= 0 */
  int32_t budget_tokens;      /* Quest budget in tokens; <= 0: base = full attention */
  double p;                   /* top-p, in (0, 1] */
  int32_t group_mode;         /* 1: one set per KV group, 0: per query head */
  int32_t* cand_pages;        /* [B][Hk][cand_stride] (unused if budget_tokens <= 0) */
  int32_t cand_stride;
  int32_t* ncand;             /* [B][Hk] */
  int32_t* idx;               /* [U][capacity] */
  int32_t capacity;
  int32_t* count;             /* [U] */
  uint16_t* out;              /* [B][Hq][128] */
  float* lse;                 /* [B][Hq] or NULL */
  void* ws;
  size_t ws_bytes;
  int32_t append_keys;        /* nonzero: run tw_append_keys on the cache first */
} tw_step;

int tw_decode_step(const tw_step* step, void* stream);

/* tw_decode_step with the query read from, and the attention output written
 * to, page-locked host memory: q_host [B][Hq][128] fp16 is copied into
 * step->q, the step runs, and step->out is copied to out_host [B][Hq][128],
 * all enqueued on `stream` as kernels of one launch chain (a step moves only
 * a few KB each way, less than a copy engine's fixed cost).  step->q and
 * step->out stay the device staging buffers; lse stays on the device.
 * q_host and out_host must be 16-byte aligned and lie in page-locked host
 * memory mapped into the device's address space (cudaHostAlloc /
 * cudaMallocHost, or cudaHostRegister with cudaHostRegisterMapped);
 * pageable memory gives TW_ERR_INVALID_ARG before anything is launched.  As
 * with cudaMemcpyAsync, q_host is read and out_host written when the stream
 * reaches the call: do not write q_host or read out_host until the stream
 * has passed it. */
int tw_decode_step_host(const tw_step* step, const uint16_t* q_host, uint16_t* out_host,
                        void* stream);

/* Profiling variant of tw_decode_step: records events[0] before the first
 * kernel and events[i + 1] after kernel i on `stream` (events are
 * cudaEvent_t, n_events >= tw_decode_step_num_kernels(step) + 1). */
int tw_decode_step_num_kernels(const tw_step* step);
const char* tw_decode_step_kernel_name(const tw_step* step, int32_t i);
int tw_decode_step_profiled(const tw_step* step, void* const* events, int32_t n_events,
                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TWILIGHT_H */
