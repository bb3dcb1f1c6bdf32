/*
 * pagedattn — single-token decode attention over a paged KV cache, for
 * NVIDIA B200 (sm_100a).  C ABI of libpagedattn.so.
 *
 * The method (citations name the web pages by title and section):
 *  - "KV-Cache Optimization Techniques", section "PagedAttention (vLLM)":
 *    the cache is kept in fixed-size pages of P tokens in one physical pool;
 *    each request has a page table mapping its logical KV positions to
 *    physical pages; pages are allocated on demand. Eq. (1): attention for
 *    the current query token is softmax(q [K_page1; ...; K_pagen]^T / sqrt(d_k))
 *    times [V_page1; ...; V_pagen], i.e. ordinary attention over the
 *    gathered pages.
 *  - same page, section "Multi-Query and Grouped-Query Caching", Eq. (7):
 *    H query heads share G groups of K/V; here query head hq reads KV head
 *    hq / (Hq / Hkv).
 *  - same page, section "KV-Cache Quantization", Eq. (3): per-token INT8
 *    codes with one scale/zero-point per row of K or V.
 *  - same page, section "Prefix Caching": requests that share a prefix point
 *    their tables at the same physical pages; results must not depend on
 *    which physical pages a table names ("Understanding KV-Cache Optimization
 *    in Modern LLM Serving", section "PagedAttention Solution": paging does
 *    not change the model's output).
 *
 * Conventions for every entry point
 *  - Pointers marked (device) are CUDA device pointers owned by the caller;
 *    the library allocates nothing, keeps no mutable global state and never
 *    synchronises a stream. `stream` is a cudaStream_t passed as void*
 *    (NULL = legacy default stream). Calls are asynchronous on that stream.
 *  - Host-side checks run before any launch; a failed check returns an error
 *    status and launches nothing. pa_last_error() then gives a message
 *    (per host thread).
 *  - Device-side checks never trap: a kernel that meets a table entry outside
 *    the pool, an out-of-range context length, sequence index or position
 *    skips that data (it is neither read nor written) and ORs a PA_DERR_*
 *    bit into *d_err when d_err is not NULL.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_ABI_VERSION 2

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, mismatched shapes  */
  PA_ERR_UNSUPPORTED = 2,  /* shape outside the compiled set (D, P, G, dtype)  */
  PA_ERR_WORKSPACE = 3,    /* workspace too small or misaligned                */
  PA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed             */
  PA_ERR_BAD_TABLE = 5,    /* a device error word reports bad tables, context
                              lengths, sequence indices or positions
                              (pa_derr_status)                                 */
  PA_ERR_TIMEOUT = 6       /* a device error word reports an expired bounded
                              wait (pa_derr_status)                            */
} pa_status_t;

/* Bits a kernel ORs into *d_err (device int32) when it skips bad input. */
#define PA_DERR_BAD_PAGE 1 /* a needed table entry is outside [0, num_pages)  */
#define PA_DERR_BAD_CTX 2  /* context_len < 0 or > max_pages * page_size       */
#define PA_DERR_BAD_SEQ 4  /* append: seq_idx outside [0, num_seqs)            */
#define PA_DERR_BAD_POS 8  /* append: pos < 0 or pos / page_size >= max_pages  */
#define PA_DERR_TIMEOUT 32 /* a bounded wait on the kernel's own tensor-core
                              work ran out (not expected; outputs invalid)    */

/*
 * pa_derr_status — the status a device error word stands for, once the
 * caller has read *d_err back to the host (host only, no device access):
 * 0 -> PA_OK; PA_DERR_TIMEOUT set -> PA_ERR_TIMEOUT (it wins over the
 * others: outputs are invalid); any of PA_DERR_BAD_PAGE, _BAD_CTX, _BAD_SEQ,
 * _BAD_POS -> PA_ERR_BAD_TABLE; any other bit -> PA_ERR_INVALID_ARG.
 */
pa_status_t pa_derr_status(int32_t derr);

typedef enum {
  PA_KV_BF16 = 0,          /* K/V stored as bf16                               */
  PA_KV_U8_PER_TOKEN = 1,  /* Eq. (3): uint8 codes + fp32 (scale, zero) per row */
  PA_KV_FP8_PER_TOKEN = 2, /* E4M3 codes + fp32 (scale, 0) per row; x = s * e4m3 */
  PA_KV_U4_PER_TOKEN = 3   /* Eq. (3) with 16 levels: two 4-bit codes per byte
                              (element 2i in the low nibble) + fp32 (scale, zero) */
} pa_kv_dtype_t;

/*
 * The physical page pool ("PagedAttention (vLLM)", "Architecture").
 * Layout of one tensor (K or V): [num_pages][num_kv_heads][page_size][head_dim],
 * row-major, so the page_size x head_dim block of one (page, KV head) is
 * contiguous. bf16 pools hold 2-byte elements; INT8 and FP8 pools hold 1-byte
 * codes and INT4 pools half-byte codes (rows of head_dim / 2 bytes), all three
 * plus k_sz / v_sz = fp32 [num_pages][num_kv_heads][page_size][2] holding
 * (scale, zero) of each row (zero is 0 for FP8). Every pointer must be
 * 16-byte aligned.
 * Supported: page_size in {16, 32}; head_dim in {64, 128}.
 */
typedef struct {
  int32_t num_pages;
  int32_t page_size;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t dtype;      /* pa_kv_dtype_t */
  void *k_pool;       /* (device) */
  void *v_pool;       /* (device) */
  float *k_sz;        /* (device) INT8, FP8 and INT4 pools, else NULL */
  float *v_sz;        /* (device) INT8, FP8 and INT4 pools, else NULL */
} pa_kv_pool_t;

/*
 * pa_kv_append — write new tokens' K/V rows into their page slots.
 * ("PagedAttention (vLLM)", "Architecture": logical position -> physical page
 * through the request's page table; pages are allocated by the caller on
 * demand. For an INT8 pool each row is quantised on the way in by Eq. (3):
 * z = min of the row, s = (max - min) / 255, code = round-half-even((x - z)/s)
 * clamped to [0, 255], all in IEEE fp32; a constant row stores s = 0, codes 0.
 * For an FP8 pool (the pages name FP8 KV caches without fixing the encoding;
 * this library uses OCP E4M3 with a per-row absmax scale): s = max|x| / 448,
 * code = E4M3(x / s) rounded to nearest even and saturated at +-448, zero 0;
 * an all-zero row stores s = 0, codes 0. An INT4 pool uses Eq. (3) with
 * s = (max - min) / 15 and codes in [0, 15], in the same fp32 order as INT8.
 * Input rows must be finite; -0 is stored as +0.)
 *
 *   k_new, v_new : (device) bf16 [num_tokens][num_kv_heads][head_dim]
 *   seq_idx, pos : (device) int32 [num_tokens]; token i is position pos[i]
 *                  (0-based) of sequence seq_idx[i]
 *   block_tables : (device) int32 [num_seqs][max_pages]
 * Row i goes to page block_tables[seq_idx[i]][pos[i] / P], slot pos[i] % P.
 * Two tokens that name the same slot race (the caller must not do that);
 * writing into a page shared by several tables changes all of them
 * (copy-on-write is the caller's job). num_tokens == 0 is a no-op.
 */
pa_status_t pa_kv_append(const pa_kv_pool_t *pool, const void *k_new,
                         const void *v_new, const int32_t *seq_idx,
                         const int32_t *pos, int32_t num_tokens,
                         const int32_t *block_tables, int32_t num_seqs,
                         int32_t max_pages, int32_t *d_err, void *stream);

/*
 * pa_decode_append_lens — pa_decode_append with the context lengths also given
 * in host memory (host_context_lens: int32 [num_seqs], the values in
 * context_lens as the host knows them, e.g. from a serving scheduler; may be
 * NULL, which is pa_decode_append). With num_splits == 0 and num_seqs <= 256
 * the split count comes from pa_decode_plan_lens: a ragged batch that needs
 * several waves of CTAs runs one CTA per (sequence, KV head), launched
 * longest context first, and then needs no workspace. Host values that
 * differ from the device ones change only the schedule: the result is
 * always Eq. 1 over the device's context_lens. Other arguments, layouts and
 * errors as for pa_decode_append; a workspace sized as for pa_decode_append
 * (pa_decode_workspace_bytes with pa_decode_num_splits' count) always
 * suffices (the split count here is 1 or that count).
 */
pa_status_t pa_decode_append_lens(const pa_kv_pool_t *pool, const void *q,
                                  const void *k_new, const void *v_new,
                                  int32_t num_seqs, int32_t num_q_heads,
                                  const int32_t *block_tables, int32_t max_pages,
                                  const int32_t *context_lens,
                                  const int32_t *host_context_lens, float scale,
                                  float *out, void *workspace,
                                  size_t workspace_bytes, int32_t num_splits,
                                  int32_t *d_err, void *stream);

/*
 * pa_decode_num_splits_lens — the split count pa_decode_append_lens uses
 * (pa_decode_plan_lens with this device's SM count and decode occupancy);
 * pa_decode_num_splits when host_context_lens is NULL, requested > 0 or
 * num_seqs > 256. Returns <= 0 on invalid arguments.
 */
int32_t pa_decode_num_splits_lens(const pa_kv_pool_t *pool, int32_t num_seqs,
                                  int32_t max_pages,
                                  const int32_t *host_context_lens,
                                  int32_t requested);

/*
 * pa_decode_plan_lens — host only: the split count pa_decode_append_lens
 * uses for num_seqs sequences of host_context_lens tokens (values clamped to
 * [0, max_pages * page_size]) over num_kv_heads KV heads, on num_sms SMs
 * holding ctas_per_sm decode CTAs each, and in order[0 .. num_seqs) the
 * sequences longest first (ties by index). Returns 1 when the (sequence, KV
 * head) units fill more than one wave of the planner's slots (num_sms x
 * min(ctas_per_sm, 3)), the longest context is at least 1.3 x the mean and
 * max_pages <= 2048; otherwise pa_decode_plan_splits' automatic count.
 * Returns <= 0 on invalid arguments (num_seqs outside 1..256 included).
 */
int32_t pa_decode_plan_lens(const int32_t *host_context_lens, int32_t num_seqs,
                            int32_t num_kv_heads, int32_t max_pages,
                            int32_t page_size, int32_t num_sms,
                            int32_t ctas_per_sm, uint16_t *order);

/*
 * pa_decode_num_splits — the split-KV partition count S pa_decode uses for
 * this pool shape, table width and request. requested == 0 picks S from the
 * number of (sequence, KV head) units, the table width and how many decode
 * CTAs fit on the current device: with fewer units than resident CTA slots,
 * the fewest splits that give about 1.7 CTAs per SM in one wave; otherwise a
 * wave model of the CTAs' lengths. requested > 0 is honoured as far as the
 * limits allow. Either way S is then clamped to [1, min(max_pages, 256)],
 * raised to at least ceil(max_pages / 2048) (a split stages at most 2048
 * table entries), and reduced so no split is empty by construction:
 * with C = ceil(max_pages / S), split s covers logical pages [s*C, (s+1)*C)
 * and S = ceil(max_pages / C). Only pool->num_kv_heads, page_size,
 * head_dim and dtype are read. Returns <= 0 on invalid arguments.
 */
int32_t pa_decode_num_splits(const pa_kv_pool_t *pool, int32_t num_seqs,
                             int32_t max_pages, int32_t requested);

/*
 * pa_decode_plan_splits — the planning rule of pa_decode_num_splits as a pure
 * host function (no device access), for num_units (sequence, KV head) units,
 * a table of max_pages pages of page_size tokens, and a device with num_sms
 * SMs holding ctas_per_sm decode CTAs each. requested as for
 * pa_decode_num_splits (0 = automatic). Returns <= 0 on invalid arguments.
 */
int32_t pa_decode_plan_splits(int64_t num_units, int32_t max_pages, int32_t page_size,
                              int32_t num_sms, int32_t ctas_per_sm, int32_t requested);

/*
 * pa_decode_auto_splits — the split count pa_decode picks with
 * num_splits == 0 for a batch of num_seqs sequences whose longest context is
 * max_ctx tokens, in a bf16 pool of head_dim 128 with num_kv_heads heads and
 * pages of page_size tokens, on the current device: the same as
 * pa_decode_num_splits with such a pool and ceil(max_ctx / page_size) table
 * columns. (A shape-only form for planners that hold no pool yet; use
 * pa_decode_num_splits for other dtypes and head sizes.) Returns <= 0 on
 * invalid arguments.
 */
int32_t pa_decode_auto_splits(int32_t num_seqs, int32_t num_kv_heads, int32_t max_ctx,
                              int32_t page_size);

/*
 * pa_decode_workspace_bytes — device scratch pa_decode needs for
 * num_splits (already resolved, >= 1): 0 when num_splits == 1, else room for
 * the partial outputs fp32 [num_seqs][num_q_heads][num_splits][head_dim] and
 * their log-sum-exps fp32 [num_seqs][num_q_heads][num_splits] (each 256-byte
 * aligned) plus the split counters.
 * Workspace layout, for every entry point that takes one: bytes
 * [0, C) with C = 256 * floor(workspace_bytes / 32768) hold int32 split
 * counters, one per (sequence, KV head); the partials follow from byte C.
 * C depends on the workspace's size only, so calls of any shape and entry
 * point that share a workspace use the same counters, and nothing else is
 * ever written there. The counters must be zero before a workspace's first
 * use (allocate it zero-filled); every completed call leaves them zero, so a
 * workspace zero-filled once serves any later call it is large enough for.
 */
size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                 int32_t head_dim, int32_t num_splits);

/*
 * pa_decode — Eq. (1) for one query token per sequence.
 *
 *   q            : (device) bf16 [num_seqs][num_q_heads][head_dim]
 *   block_tables : (device) int32 [num_seqs][max_pages]; entries at or past
 *                  ceil(context_lens[b] / P) are never read
 *   context_lens : (device) int32 [num_seqs]; tokens 0..ctx-1 are attended
 *                  (the token appended for this step included, no mask)
 *   scale        : multiplies q.k (1 / sqrt(head_dim) for Eq. (1))
 *   out          : (device) fp32 [num_seqs][num_q_heads][head_dim]
 *   workspace    : (device) >= pa_decode_workspace_bytes(...) bytes, 256-byte
 *                  aligned; may be NULL when that is 0
 *   num_splits   : 0 = automatic; the count actually used is always
 *                  pa_decode_num_splits(pool, num_seqs, max_pages, num_splits)
 * num_q_heads must be a multiple of pool->num_kv_heads with a ratio of 1..8.
 * A sequence with context length 0 gets out = 0. When a sequence spans more
 * than one split, each split writes a partial result and its log-sum-exp to
 * the workspace and the split that finishes last merges them (in split order,
 * the same arithmetic as pa_splitkv_reduce) — one kernel launch in all.
 * The kernel is launched as a programmatic dependent of the previous kernel
 * on the stream and waits for it before reading any input. Results are
 * deterministic and do not depend on the physical page ids. Two calls that
 * share a workspace must not overlap on the GPU.
 */
pa_status_t pa_decode(const pa_kv_pool_t *pool, const void *q,
                      int32_t num_seqs, int32_t num_q_heads,
                      const int32_t *block_tables, int32_t max_pages,
                      const int32_t *context_lens, float scale, float *out,
                      void *workspace, size_t workspace_bytes,
                      int32_t num_splits, int32_t *d_err, void *stream);

/*
 * pa_decode_append — one decode step in one launch: the cache write of
 * pa_kv_append for each sequence's newest token, fused into pa_decode.
 *   k_new, v_new : (device) bf16 [num_seqs][num_kv_heads][head_dim], 16-byte
 *                  aligned: the K/V rows of token context_lens[b] - 1 of
 *                  sequence b (its page must already be in the table)
 * Every other argument is pa_decode's. The CTA whose split holds position
 * context_lens[b] - 1 stores that row (quantised for INT8/FP8/INT4 pools by
 * the same per-row quantiser as pa_kv_append, so the stored bits are
 * identical) before it reads
 * the page; then Eq. (1) runs over tokens 0 .. context_lens[b] - 1 as in
 * pa_decode. The result equals pa_kv_append(seq_idx = b, pos =
 * context_lens[b] - 1) followed by pa_decode, bit for bit, without the
 * append's launch. A sequence with context length 0 stores nothing. As with
 * pa_kv_append, the page receiving a sequence's new token must belong to
 * that sequence alone (copy-on-write is the caller's job): here another
 * sequence's CTAs could otherwise read that page while it is written.
 */
pa_status_t pa_decode_append(const pa_kv_pool_t *pool, const void *q,
                             const void *k_new, const void *v_new,
                             int32_t num_seqs, int32_t num_q_heads,
                             const int32_t *block_tables, int32_t max_pages,
                             const int32_t *context_lens, float scale, float *out,
                             void *workspace, size_t workspace_bytes,
                             int32_t num_splits, int32_t *d_err, void *stream);

/*
 * pa_decode_shared_prefix — cascade decode for a batch whose requests all
 * begin with the same prompt prefix stored once in shared pages
 * ("KV-Cache Optimization Techniques", section "Prefix Caching", Eq. 2).
 * Computes exactly what pa_decode computes when every request's logical pages
 * [0, prefix_len / P) are prefix_pages, in three launches: (1) attention of
 * all num_seqs * num_q_heads query rows over the prefix, as dense tcgen05
 * tensor-core tiles (accumulators in tensor memory) that read each prefix
 * K/V row once per 128 query rows instead of once per request; (2) the paged
 * decode over each request's own tokens [prefix_len, context_lens[b]),
 * writing its split partials; (3) the log-sum-exp merge of (2) and (1) per
 * row, in that order (deterministic). (1) and (2) run side by side, so the
 * prefix pass (tensor-core and L2 bound) overlaps the suffix decode (HBM
 * bound); the split count of (1) is pa_prefix_plan_splits'. Called eagerly,
 * all three run on `stream` as programmatic dependent launches ((1) lets (2)
 * start once the work before the call has finished; (3) starts after both).
 * While `stream` is being captured into a CUDA graph, (2) runs on a second
 * stream the library keeps per device, forked from `stream` before (1) and
 * joined back before (3) (the fork and join become graph edges; calls from
 * several host threads are serialised around the fork). Either way the call
 * is one unit of `stream`: all three complete before later work on it.
 *
 *   prefix_pages : (device) int32 [prefix_len / P] physical pages of the prefix
 *   prefix_len   : tokens in the prefix; a multiple of the page size (0 falls
 *                  back to pa_decode)
 *   block_tables : (device) int32 [num_seqs][max_pages]; entries for logical
 *                  pages < prefix_len / P are not read
 *   context_lens : (device) int32 [num_seqs], each >= prefix_len (a shorter
 *                  one is flagged PA_DERR_BAD_CTX and treated as prefix_len)
 *   workspace    : (device) >= pa_decode_shared_prefix_workspace_bytes(...)
 *                  bytes, 256-byte aligned, zero-filled before its first use
 * Other arguments as for pa_decode. bf16 pools only. Three kernel launches.
 */
size_t pa_decode_shared_prefix_workspace_bytes(const pa_kv_pool_t *pool,
                                               int32_t num_seqs,
                                               int32_t num_q_heads,
                                               int32_t max_pages,
                                               int32_t prefix_len,
                                               int32_t num_splits);

pa_status_t pa_decode_shared_prefix(const pa_kv_pool_t *pool, const void *q,
                                    int32_t num_seqs, int32_t num_q_heads,
                                    const int32_t *prefix_pages,
                                    int32_t prefix_len,
                                    const int32_t *block_tables,
                                    int32_t max_pages,
                                    const int32_t *context_lens, float scale,
                                    float *out, void *workspace,
                                    size_t workspace_bytes, int32_t num_splits,
                                    int32_t *d_err, void *stream);

/*
 * pa_prefix_plan_splits — host only (no device access): how many 64-token
 * tiles of the shared prefix each CTA of pa_decode_shared_prefix's prefix pass
 * takes, for `units` (128-row query tile, KV head) pairs, a prefix of `tiles`
 * 64-token tiles, a device of num_sms SMs holding decode_ctas_per_sm suffix
 * decode CTAs each, and an estimate of the bytes the suffix decode streams.
 * The pass runs beside the suffix decode, so the rule picks the split count
 * whose estimated finish, the later of the two, is earliest: the prefix pass
 * takes 4 us plus 1.6 us per tile with one of its CTAs on an SM (2.2 us with
 * two; more than two per SM run in waves), and the decode streams at 6.5 TB/s
 * while it keeps at least 2 * num_sms CTAs resident, slower in proportion
 * below that (an SM holding one prefix CTA keeps decode_ctas_per_sm - 2
 * decode CTAs, one holding two keeps none). Ties go to fewer CTAs. The
 * constants were measured on B200. The pass then has ceil(tiles / result)
 * splits. Returns <= 0 on invalid arguments.
 */
int32_t pa_prefix_plan_splits(int64_t units, int32_t tiles, int32_t num_sms,
                              int32_t decode_ctas_per_sm, double suffix_bytes);

/*
 * pa_decode_window — decode over the StreamingLLM token set: the first `sinks`
 * tokens (attention sinks) and the last `window` tokens of each sequence
 * ("KV-Cache Optimization Techniques", section "Token Eviction Strategies",
 * Eq. 5; sinks = 0 is the sliding-window cache of Eq. 6). Only the pages that
 * hold kept tokens are read: the sink pages and the last ceil(window / P) + 1
 * pages; table entries of evicted pages are never dereferenced, so a caller
 * may free those pages and leave any value in their entries.
 *   window : >= 0; 0 keeps every token (falls back to pa_decode)
 *   sinks  : >= 0; tokens [0, min(sinks, ctx)) are always kept
 *   workspace : >= pa_decode_window_workspace_bytes(...), zero-filled before
 *               its first use, 256-byte aligned (NULL if that is 0)
 * Other arguments and behaviour as for pa_decode (bf16, INT8, FP8 and INT4
 * pools). The sinks are a second token range of the first split, so one
 * split per (sequence, KV head) needs no workspace.
 */
size_t pa_decode_window_workspace_bytes(const pa_kv_pool_t *pool,
                                        int32_t num_seqs, int32_t num_q_heads,
                                        int32_t max_pages, int32_t sinks,
                                        int32_t window, int32_t num_splits);

pa_status_t pa_decode_window(const pa_kv_pool_t *pool, const void *q,
                             int32_t num_seqs, int32_t num_q_heads,
                             const int32_t *block_tables, int32_t max_pages,
                             const int32_t *context_lens, int32_t sinks,
                             int32_t window, float scale, float *out,
                             void *workspace, size_t workspace_bytes,
                             int32_t num_splits, int32_t *d_err, void *stream);

/*
 * pa_decode_noalloc — pa_decode for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point: it only changes where
 * pa_decode's split-KV scratch lives.
 *
 * Some callers have no way to obtain the workspace pa_decode asks for: a
 * plugin or C host that is handed only its input and output buffers, a
 * server that reserved all device memory up front for its own pool, or a
 * latency-critical loop that must not pay the implicit synchronisation of
 * cudaMalloc. This entry point takes the same arguments as pa_decode minus
 * the workspace, and keeps the partial results and their log-sum-exps in a
 * buffer that belongs to the library itself: a file-scope device array of
 * PA_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the library
 * holds until the process exits. It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 *   num_splits : 0 = automatic, lowered if needed until the partials fit the
 *                scratch; an explicit count whose partials
 *                (pa_decode_workspace_bytes) exceed PA_NOALLOC_SCRATCH_BYTES
 *                is rejected with PA_ERR_WORKSPACE before any launch.
 *
 * Set-up: the first call on each device (with that device current) looks up
 * the array's device address with cudaGetSymbolAddress; make that first call
 * before any stream capture. The address is cached per device under the id of
 * the CUDA context it was found in: after cudaDeviceReset (or anything else
 * that destroys and re-creates the context) the module is loaded anew, the
 * cached address is no longer valid, and the next call looks it up again —
 * that call is a first call again, with the same rule on stream capture.
 * A planner failure (e.g. an unsupported pool) is reported as pa_decode
 * reports it. Every call on a device shares the one array and
 * it keeps the last call's contents. The only part that must start at zero is
 * the split counters, which the array holds from load time and which every
 * completed call returns to zero. Calls that overlap on the GPU — on
 * different streams or from different host threads without ordering between
 * them — race on the array and must be serialised by the caller. Results
 * equal pa_decode's for the same split count.
 */
#define PA_NOALLOC_SCRATCH_BYTES (16u << 20)

pa_status_t pa_decode_noalloc(const pa_kv_pool_t *pool, const void *q,
                              int32_t num_seqs, int32_t num_q_heads,
                              const int32_t *block_tables, int32_t max_pages,
                              const int32_t *context_lens, float scale,
                              float *out, int32_t num_splits, int32_t *d_err,
                              void *stream);

/*
 * pa_decode_range — Eq. (1) restricted to a token range, returned as a
 * normalised partial and its log-sum-exp, for merging with other ranges
 * (e.g. the context-parallel decode of a sequence whose pages are spread over
 * several GPUs: each GPU decodes its range, the partials are all-gathered and
 * merged with pa_merge_partials).
 * Every sequence b attends tokens [tok_begin, min(context_lens[b], tok_end));
 * a sequence with no token there gets o = 0, lse = -inf (not an error).
 *   tok_begin, tok_end : tok_begin a multiple of the page size, tok_end >=
 *                        tok_begin; table entries outside the range's pages
 *                        are not read
 *   o_out   : (device) fp32 [num_seqs][num_q_heads][head_dim], the range's
 *             attention output normalised by the range's own softmax sum
 *   lse_out : (device) fp32 [num_seqs][num_q_heads], natural log of the sum
 *             of exp(scale * q.k) over the range
 *   workspace : >= pa_decode_range_workspace_bytes(...) bytes, 256-byte
 *               aligned, zero-filled before first use (NULL when that is 0)
 * Other arguments as for pa_decode (fixed split partition over the range's
 * pages); one launch, or two when the range is split.
 */
size_t pa_decode_range_workspace_bytes(const pa_kv_pool_t *pool, int32_t num_seqs,
                                       int32_t num_q_heads, int32_t max_pages,
                                       int32_t tok_begin, int32_t tok_end,
                                       int32_t num_splits);

pa_status_t pa_decode_range(const pa_kv_pool_t *pool, const void *q,
                            int32_t num_seqs, int32_t num_q_heads,
                            const int32_t *block_tables, int32_t max_pages,
                            const int32_t *context_lens, int32_t tok_begin,
                            int32_t tok_end, float scale, float *o_out,
                            float *lse_out, void *workspace,
                            size_t workspace_bytes, int32_t num_splits,
                            int32_t *d_err, void *stream);

/*
 * pa_merge_partials — merge num_parts partial results of disjoint token
 * ranges, laid out part-major (what an all-gather of pa_decode_range outputs
 * produces), with the same weights as pa_splitkv_reduce, in part order.
 *   o_parts   : (device) fp32; part p is [rows][head_dim] at
 *               o_parts + p * o_part_stride, normalised
 *   lse_parts : (device) fp32; part p is [rows] at
 *               lse_parts + p * lse_part_stride, natural log
 *   o_part_stride, lse_part_stride : floats between parts; 0 = dense
 *               (rows * head_dim, rows). One all-gathered buffer holding
 *               each rank's o and lse back to back is read in place with
 *               both strides set to that buffer's per-rank size. Parts must
 *               not overlap; o_part_stride a multiple of 4.
 *   out       : (device) fp32 [rows][head_dim]
 *   lse_out   : (device) fp32 [rows], the merged log-sum-exp, or NULL
 * head_dim a multiple of 4 and at most 512. One launch.
 */
pa_status_t pa_merge_partials(const float *o_parts, const float *lse_parts,
                              int32_t num_parts, int32_t rows, int32_t head_dim,
                              int64_t o_part_stride, int64_t lse_part_stride,
                              float *out, float *lse_out, void *stream);

/*
 * pa_splitkv_reduce — merge split-KV partial results.
 * (Not on the pages: the exact identity for softmax over disjoint token
 * ranges. With M = max_s lse_s and w_s = exp(lse_s - M):
 * out = sum_s w_s o_s / sum_s w_s; a split with lse = -inf has weight 0 and
 * if every split is empty out = 0.)
 *   o_part : (device) fp32 [num_seqs][num_q_heads][num_splits][head_dim],
 *            each o_s already normalised by its own softmax sum
 *   lse    : (device) fp32 [num_seqs][num_q_heads][num_splits], natural log
 *            of the split's sum of exp(scale * q.k)
 *   out    : (device) fp32 [num_seqs][num_q_heads][head_dim]
 * head_dim must be a multiple of 4 and at most 512; num_splits in [1, 256].
 */
pa_status_t pa_splitkv_reduce(const float *o_part, const float *lse,
                              int32_t num_seqs, int32_t num_q_heads,
                              int32_t num_splits, int32_t head_dim, float *out,
                              void *stream);

/*
 * pa_validate_tables — check the page tables a decode would read.
 * For each sequence: 0 <= context_lens[b] <= max_pages * page_size, and every
 * entry in [0, ceil(ctx / page_size)) lies in [0, num_pages). Violations set
 * PA_DERR_BAD_CTX / PA_DERR_BAD_PAGE in *d_err (device int32, required);
 * the word is OR-ed into, not cleared. Asynchronous like everything else.
 */
pa_status_t pa_validate_tables(const int32_t *block_tables, int32_t num_seqs,
                               int32_t max_pages, const int32_t *context_lens,
                               int32_t num_pages, int32_t page_size,
                               int32_t *d_err, void *stream);

/*
 * One decode step end to end from host memory: the step's inputs cross to the
 * device as ONE packet (one host-to-device copy), the new K/V rows are written
 * (pa_kv_append), Eq. (1) is decoded (pa_decode) and the output comes back
 * (one device-to-host copy), all in stream order on `stream`.
 *
 * Packet layout: seven sections in this order, each starting on a 256-byte
 * boundary of the packet:
 *   0 q            bf16  [num_seqs][num_q_heads][head_dim]
 *   1 k_new        bf16  [num_new][num_kv_heads][head_dim]
 *   2 v_new        bf16  [num_new][num_kv_heads][head_dim]
 *   3 seq_idx      int32 [num_new]
 *   4 pos          int32 [num_new]
 *   5 block_tables int32 [num_seqs][max_pages]
 *   6 context_lens int32 [num_seqs]
 * (the same meaning as the arguments of pa_kv_append and pa_decode).
 *
 * num_new == PA_STEP_NEWEST_PER_SEQ instead means one row per sequence, its
 * newest token (position context_lens[b] - 1): k_new and v_new are then
 * [num_seqs][num_kv_heads][head_dim], sections 3 and 4 are empty, and the
 * step runs pa_decode_append (cache write fused into the decode, one launch)
 * instead of pa_kv_append + pa_decode.
 *
 * pa_step_packet_layout — host only (no device access): writes the seven
 * section offsets in bytes to offsets[0..6] (when offsets is not NULL) and
 * returns the packet size in bytes, or 0 on invalid arguments.
 */
#define PA_STEP_NEWEST_PER_SEQ (-1)
size_t pa_step_packet_layout(const pa_kv_pool_t *pool, int32_t num_seqs,
                             int32_t num_q_heads, int32_t max_pages,
                             int32_t num_new, size_t *offsets);

/*
 * pa_decode_step_host — the step itself.
 *   packet_host : (host) packet_bytes bytes laid out as above; page-locked
 *                 memory makes the copy asynchronous (pageable memory works,
 *                 but the copy then blocks the calling thread)
 *   packet_dev  : (device) >= packet_bytes bytes, 256-byte aligned; the
 *                 library copies the packet here and reads every input from it
 *   packet_bytes: pa_step_packet_layout(...) for the same shape
 *   out_dev     : (device) fp32 [num_seqs][num_q_heads][head_dim]
 *   out_host    : (host) fp32, same shape; receives out_dev
 *   workspace, workspace_bytes, num_splits, d_err : as for pa_decode
 *   synchronize : nonzero = wait for the stream before returning, so that
 *                 out_host holds the result when the call returns
 * Errors: those of pa_kv_append and pa_decode, PA_ERR_INVALID_ARG for a
 * packet_bytes that does not match the shape, PA_ERR_CUDA for a failed copy.
 * The packet buffers may be reused by the next step once this one has
 * completed on the stream.
 */
pa_status_t pa_decode_step_host(const pa_kv_pool_t *pool, const void *packet_host,
                                void *packet_dev, size_t packet_bytes,
                                int32_t num_seqs, int32_t num_q_heads,
                                int32_t max_pages, int32_t num_new, float scale,
                                float *out_dev, float *out_host, void *workspace,
                                size_t workspace_bytes, int32_t num_splits,
                                int32_t *d_err, void *stream, int32_t synchronize);

/*
 * A pa_decode_step_host step captured once into a CUDA graph and replayed:
 * per step the host then makes one graph launch instead of one copy, one or
 * two kernel launches and a second copy. Every pointer and size is fixed at
 * creation; each launch copies whatever packet_host holds at that time, so
 * the caller refills the packet (and reads out_host) between launches.
 *
 * pa_step_graph_create — arguments as for pa_decode_step_host (minus stream
 *   and synchronize; packet_host and out_host must be page-locked, as graph
 *   copies require); plans the step, captures it on a private stream and
 *   instantiates the graph into *graph (caller-owned, released with
 *   pa_step_graph_destroy). Errors: those of pa_decode_step_host, or
 *   PA_ERR_CUDA when capture or instantiation fails; *graph is then NULL.
 * pa_step_graph_launch — launches the step on `stream`; synchronize != 0
 *   waits for it (out_host then holds the result).
 * pa_step_graph_destroy — releases the graph (NULL is ignored); no launch of
 *   it may still be pending.
 */
typedef struct pa_step_graph pa_step_graph_t;

pa_status_t pa_step_graph_create(const pa_kv_pool_t *pool, const void *packet_host,
                                 void *packet_dev, size_t packet_bytes,
                                 int32_t num_seqs, int32_t num_q_heads,
                                 int32_t max_pages, int32_t num_new, float scale,
                                 float *out_dev, float *out_host, void *workspace,
                                 size_t workspace_bytes, int32_t num_splits,
                                 int32_t *d_err, pa_step_graph_t **graph);
pa_status_t pa_step_graph_launch(pa_step_graph_t *graph, void *stream, int32_t synchronize);
void pa_step_graph_destroy(pa_step_graph_t *graph);

/*
 * pa_selftest_wait_timeout — exercises the failure path of the kernels'
 * bounded waits (the tcgen05 prefix pass waits on mbarriers for its tensor-
 * core work): one thread waits on an mbarrier that nothing arrives at, gives
 * up after limit_us microseconds of wall time and ORs PA_DERR_TIMEOUT into
 * *d_err (device int32, required). It neither faults nor hangs, and the
 * context stays usable. limit_us in [1, 1000000]. One launch.
 */
pa_status_t pa_selftest_wait_timeout(int32_t limit_us, int32_t *d_err, void *stream);

/* Static description of a status code. */
const char *pa_status_str(pa_status_t status);

/* Message describing the last failed call on this host thread ("" if none). */
const char *pa_last_error(void);

/* PA_ABI_VERSION of the loaded library. */
int32_t pa_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PAGEDATTN_H */
