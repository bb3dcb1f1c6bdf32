// extern "C" boundary of libpagedattn.so: argument checks, split-KV planning
// and kernel launches. See include/pagedattn.h for the contract of each call.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>

#include "pa_internal.h"

namespace pa {
namespace {

thread_local std::string g_last_error;

pa_status_t fail(pa_status_t st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

pa_status_t cuda_status(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return PA_OK;
  return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_ctas[kMaxDevices][2][2][4];  // [dev][D==128][P==32][dtype]

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

pa_status_t check_pool(const pa_kv_pool_t *pool) {
  if (pool == nullptr) return fail(PA_ERR_INVALID_ARG, "pool is NULL");
  if (pool->num_pages <= 0 || pool->num_kv_heads <= 0)
    return fail(PA_ERR_INVALID_ARG, "pool: num_pages=%d num_kv_heads=%d must be positive",
                pool->num_pages, pool->num_kv_heads);
  if (pool->page_size != 16 && pool->page_size != 32)
    return fail(PA_ERR_UNSUPPORTED, "pool: page_size=%d (supported: 16, 32)", pool->page_size);
  if (pool->head_dim != 64 && pool->head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "pool: head_dim=%d (supported: 64, 128)", pool->head_dim);
  if (pool->dtype < PA_KV_BF16 || pool->dtype > PA_KV_U4_PER_TOKEN)
    return fail(PA_ERR_UNSUPPORTED, "pool: dtype=%d", pool->dtype);
  if (pool->k_pool == nullptr || pool->v_pool == nullptr)
    return fail(PA_ERR_INVALID_ARG, "pool: k_pool/v_pool is NULL");
  if (!aligned(pool->k_pool, 16) || !aligned(pool->v_pool, 16))
    return fail(PA_ERR_INVALID_ARG, "pool: k_pool/v_pool must be 16-byte aligned");
  if (pool->dtype != PA_KV_BF16) {
    if (pool->k_sz == nullptr || pool->v_sz == nullptr)
      return fail(PA_ERR_INVALID_ARG, "pool: an INT8/FP8/INT4 pool needs k_sz and v_sz");
    if (!aligned(pool->k_sz, 16) || !aligned(pool->v_sz, 16))
      return fail(PA_ERR_INVALID_ARG, "pool: k_sz/v_sz must be 16-byte aligned");
  }
  const long long rows = (long long)pool->num_pages * pool->num_kv_heads * pool->page_size;
  if (rows > (1LL << 40)) return fail(PA_ERR_INVALID_ARG, "pool too large");
  return PA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Split counters. The CTA that finishes a (sequence, KV head) last is found
// with one atomic counter per unit, which that CTA re-arms to zero. The
// counters sit at the start of every workspace, in a region whose size
// depends on the workspace's size alone (1/128 of it, in whole 256-byte
// units), and partial results are written only after that region. Calls of
// any shape and any entry point that share a workspace therefore use the same
// counter region and never write anything else into it: a workspace
// zero-filled once stays valid for every later call.
size_t counter_region(size_t ws_bytes) { return (ws_bytes / 32768) * 256; }

bool workspace_fits(size_t ws_bytes, size_t rest, size_t counter_bytes) {
  const size_t c = counter_region(ws_bytes);
  return c >= counter_bytes && ws_bytes - c >= rest;
}

// Smallest workspace size (a multiple of 256) for `rest` bytes of partials
// and `counter_bytes` of counters, with 256 bytes to spare so that every
// larger size fits too (ws - counter_region(ws) dips by at most 255 bytes).
size_t workspace_for(size_t rest, size_t counter_bytes) {
  const size_t want = align256(rest) + 256;
  size_t ws = want + align256(counter_bytes);
  while (!workspace_fits(ws, want, counter_bytes)) {
    const size_t c = counter_region(ws);
    const size_t short_c = counter_bytes > c ? counter_bytes - c : 0;
    const size_t short_r = want > ws - c ? want - (ws - c) : 0;
    ws += align256(std::max<size_t>(std::max<size_t>(short_c * 128, short_r + short_r / 127),
                                    256));
  }
  return ws;
}

}  // namespace

void set_last_error_message(const char *msg) { g_last_error = msg; }

int device_sm_count() {
  const int dev = current_device();
  if (dev < 0) return 148;
  int v = g_sm_count[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

static int cached_ctas_per_sm(int D, int P, int dtype) {
  const int dev = current_device();
  if (dev < 0) return 1;
  std::atomic<int> &slot = g_ctas[dev][D == 128][P == 32][dtype];
  int v = slot.load(std::memory_order_relaxed);
  if (v > 0) return v;
  v = decode_ctas_per_sm(D, P, dtype);
  slot.store(v, std::memory_order_relaxed);
  return v;
}

}  // namespace pa

using namespace pa;

extern "C" {

const char *pa_status_str(pa_status_t s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PA_ERR_WORKSPACE: return "workspace too small or misaligned";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_BAD_TABLE: return "bad page table, context length, sequence index or position";
    case PA_ERR_TIMEOUT: return "a bounded device wait expired";
  }
  return "unknown status";
}

pa_status_t pa_derr_status(int32_t derr) {
  if (derr == 0) return PA_OK;
  if (derr & PA_DERR_TIMEOUT) return PA_ERR_TIMEOUT;
  if (derr & (PA_DERR_BAD_PAGE | PA_DERR_BAD_CTX | PA_DERR_BAD_SEQ | PA_DERR_BAD_POS))
    return PA_ERR_BAD_TABLE;
  return PA_ERR_INVALID_ARG;
}

const char *pa_last_error(void) { return g_last_error.c_str(); }

int32_t pa_abi_version(void) { return PA_ABI_VERSION; }

pa_status_t pa_kv_append(const pa_kv_pool_t *pool, const void *k_new, const void *v_new,
                         const int32_t *seq_idx, const int32_t *pos, int32_t num_tokens,
                         const int32_t *block_tables, int32_t num_seqs, int32_t max_pages,
                         int32_t *d_err, void *stream) {
  g_last_error.clear();
  pa_status_t st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_tokens < 0 || num_seqs < 0 || max_pages <= 0)
    return fail(PA_ERR_INVALID_ARG, "num_tokens=%d num_seqs=%d max_pages=%d", num_tokens,
                num_seqs, max_pages);
  if (num_tokens == 0) return PA_OK;
  if (!k_new || !v_new || !seq_idx || !pos || !block_tables)
    return fail(PA_ERR_INVALID_ARG, "k_new, v_new, seq_idx, pos and block_tables are required");
  if (!aligned(k_new, 16) || !aligned(v_new, 16))
    return fail(PA_ERR_INVALID_ARG, "k_new/v_new must be 16-byte aligned");
  return cuda_status(launch_kv_append(*pool, k_new, v_new, seq_idx, pos, num_tokens,
                                      block_tables, num_seqs, max_pages, d_err,
                                      static_cast<cudaStream_t>(stream)),
                     "pa_kv_append launch");
}

int32_t pa_prefix_plan_splits(int64_t units, int32_t tiles, int32_t num_sms,
                              int32_t decode_ctas_per_sm, double suffix_bytes) {
  if (units <= 0 || tiles <= 0 || num_sms <= 0 || decode_ctas_per_sm <= 0 ||
      !(suffix_bytes >= 0.0))
    return -1;
  // Measured on B200 (cascade steps of 32..256 requests, prefixes of 1024..8000
  // tokens, suffixes of up to 64..1024 tokens): a prefix CTA's set-up and
  // epilogue, one 64-token tile with one or two prefix CTAs on the SM, the
  // copy bandwidth, and the decode CTAs that keep HBM streaming.
  constexpr double kFixedUs = 4.0, kTile1Us = 1.6, kTile2Us = 2.2, kBytesPerUs = 6.5e6;
  const long long sms = num_sms;
  const long long need = 2 * sms;
  const double td0 = suffix_bytes / kBytesPerUs;
  const int with_prefix = decode_ctas_per_sm > 2 ? decode_ctas_per_sm - 2 : 0;
  double best = 0.0;
  bool have = false;
  int best_tp = tiles;
  int last_n = -1;
  for (int ns = 1; ns <= tiles && ns <= kMaxSplits; ++ns) {
    const int tp = (tiles + ns - 1) / ns;  // tiles per split
    const int n = (tiles + tp - 1) / tp;   // splits
    if (n == last_n) continue;
    last_n = n;
    const long long ctas = units * n;
    double tprefix;
    long long slots;
    if (ctas <= sms) {
      tprefix = kFixedUs + tp * kTile1Us;
      slots = (sms - ctas) * decode_ctas_per_sm + ctas * with_prefix;
    } else if (ctas <= 2 * sms) {
      tprefix = kFixedUs + tp * kTile2Us;
      slots = (2 * sms - ctas) * with_prefix;
    } else {
      const long long waves = (ctas + 2 * sms - 1) / (2 * sms);
      tprefix = kFixedUs + (double)waves * tp * kTile2Us;
      slots = 0;
    }
    const double tdecode =
        td0 * (slots >= need ? 1.0 : (double)need / (double)(slots > 0 ? slots : 1));
    const double cost = tprefix > tdecode ? tprefix : tdecode;
    if (!have || cost < best) {  // strictly better: ties keep fewer CTAs
      have = true;
      best = cost;
      best_tp = tp;
    }
  }
  return best_tp;
}

int32_t pa_decode_plan_splits(int64_t num_units, int32_t max_pages, int32_t page_size,
                              int32_t num_sms, int32_t ctas_per_sm, int32_t requested) {
  if (num_units < 0 || max_pages <= 0 || page_size <= 0 || num_sms <= 0 || ctas_per_sm <= 0 ||
      requested < 0)
    return -1;
  const int P = page_size;
  const int hi = max_pages < kMaxSplits ? max_pages : kMaxSplits;
  int S = requested;
  if (S == 0) {
    // R resident CTA slots; a unit is one (sequence, KV head).
    const long long units = num_units;
    const long long sms = num_sms;
    const long long R = sms * ctas_per_sm;
    // CTAs that stream at once and keep HBM saturated: measured on the
    // Llama-3-70B shapes (B = 8, 16, 32 x 8192 tokens), one wave of ~1.7
    // CTAs per SM read at 79-103 % of the copy peak, and it was the fastest
    // split count each time; more splits only added partial writes and a merge
    const long long kSaturate = (sms * 17 + 9) / 10;
    if (units == 0) {
      S = 1;
    } else if (units < R) {
      // one wave: the fewest splits that reach kSaturate CTAs, without
      // spilling into a second wave
      long long s1 = (kSaturate + units - 1) / units;
      if (s1 * units > R) s1 = R / units;
      S = (int)(s1 < 1 ? 1 : (s1 > hi ? hi : s1));
    } else {
      // Several waves. Wave model: CTAs of equal length run in waves of R; a
      // split count is worth its extra partial writes only if it shortens
      // (#waves x tokens per CTA); ties go to fewer splits.
      // CTA start-up, table staging and epilogue, in tokens of streaming
      // (measured: ~2,400 warp instructions plus two dependent loads per CTA;
      // on ragged Llama-3-8B-shaped batches 4 splits beat 6 by 2-7 %)
      const double kCtaOverheadTok = 256.0;
      const double kSplitCostTok = 16.0;     // partial write + merge per split, per unit
      double best = 1e300;
      for (int s = 1; s <= hi; ++s) {
        const long long chunk = (max_pages + s - 1) / s;
        const int s_eff = (int)((max_pages + chunk - 1) / chunk);
        if (s_eff != s) continue;
        const long long waves = (units * s + R - 1) / R;
        double cost = (double)waves * ((double)chunk * P + kCtaOverheadTok);
        if (s > 1) cost += kSplitCostTok * s * (double)units / (double)R + kCtaOverheadTok;
        if (cost < best * (1.0 - 1e-9)) {
          best = cost;
          S = s;
        }
      }
    }
  }
  if (S > hi) S = hi;
  const int lo = (max_pages + kMaxPagesPerSplit - 1) / kMaxPagesPerSplit;
  if (S < lo) S = lo;
  if (S < 1) S = 1;
  const int chunk = (max_pages + S - 1) / S;
  return (max_pages + chunk - 1) / chunk;
}

int32_t pa_decode_plan_lens(const int32_t *host_context_lens, int32_t num_seqs,
                            int32_t num_kv_heads, int32_t max_pages, int32_t page_size,
                            int32_t num_sms, int32_t ctas_per_sm, uint16_t *order) {
  if (host_context_lens == nullptr || order == nullptr || num_seqs <= 0 ||
      num_seqs > kMaxOrdered || num_kv_heads <= 0 || max_pages <= 0 || page_size <= 0 ||
      num_sms <= 0 || ctas_per_sm <= 0)
    return -1;
  // the planner's slot count (its constants were measured with three decode
  // CTAs per SM, see pa_decode_num_splits)
  const int cps = ctas_per_sm < 3 ? ctas_per_sm : 3;
  const long long units = (long long)num_seqs * num_kv_heads;
  const int S_plan = pa_decode_plan_splits(units, max_pages, page_size, num_sms, cps, 0);
  // longest context first, ties by index (a stable sort of the indices)
  const long long cap = (long long)max_pages * page_size;
  auto len = [&](int i) {
    const long long c = host_context_lens[i];
    return c < 0 ? 0LL : (c > cap ? cap : c);
  };
  for (int i = 0; i < num_seqs; ++i) order[i] = (uint16_t)i;
  std::stable_sort(order, order + num_seqs,
                   [&](uint16_t x, uint16_t y) { return len(x) > len(y); });
  long long sum = 0;
  for (int i = 0; i < num_seqs; ++i) sum += len(i);
  const long long longest = len(order[0]);
  // Several waves of a ragged batch: one CTA per (sequence, KV head),
  // launched longest first, so the short ones fill the last wave. Measured on
  // the ragged Llama-3-8B-shaped step (contexts 242..4095, longest / mean =
  // 1.9): INT8 63.7 us against 70.9 at four splits, FP8 64.3 / 72.0, INT4
  // 57.7 / 62.0, bf16 96.7 / 98.6. Uniform batches keep the planner's splits:
  // one split per unit just over one wave was 11-21 % slower there.
  const bool several_waves = units >= (long long)num_sms * cps;
  const bool ragged = longest * 10 * num_seqs >= sum * 13;  // longest >= 1.3 x mean
  if (several_waves && ragged && max_pages <= kMaxPagesPerSplit) return 1;
  return S_plan;
}

int32_t pa_decode_num_splits_lens(const pa_kv_pool_t *pool, int32_t num_seqs,
                                  int32_t max_pages, const int32_t *host_context_lens,
                                  int32_t requested) {
  if (host_context_lens == nullptr || requested != 0 || num_seqs <= 0 || num_seqs > kMaxOrdered ||
      pool == nullptr)
    return pa_decode_num_splits(pool, num_seqs, max_pages, requested);
  if (pa_decode_num_splits(pool, num_seqs, max_pages, 0) <= 0) return -1;  // argument checks
  uint16_t order[kMaxOrdered];
  return pa_decode_plan_lens(host_context_lens, num_seqs, pool->num_kv_heads, max_pages,
                             pool->page_size, device_sm_count(),
                             cached_ctas_per_sm(pool->head_dim, pool->page_size, pool->dtype),
                             order);
}

int32_t pa_decode_num_splits(const pa_kv_pool_t *pool, int32_t num_seqs, int32_t max_pages,
                             int32_t requested) {
  if (pool == nullptr || num_seqs < 0 || max_pages <= 0 || requested < 0) return -1;
  if ((pool->head_dim != 64 && pool->head_dim != 128) ||
      (pool->page_size != 16 && pool->page_size != 32) ||
      pool->dtype < PA_KV_BF16 || pool->dtype > PA_KV_U4_PER_TOKEN ||
      pool->num_kv_heads <= 0)
    return -1;
  const int64_t units = (int64_t)num_seqs * pool->num_kv_heads;
  if (requested > 0)  // no device query needed
    return pa_decode_plan_splits(units, max_pages, pool->page_size, 1, 1, requested);
  // The rule's regimes and constants were measured with three resident decode
  // CTAs per SM; a kernel that fits a fourth (INT4) is planned as if it had
  // three: with more slots the one-wave regime would hand a ragged batch one
  // CTA per (sequence, KV head), whose longest member then sets the time
  // (INT4, ragged Llama-3-8B shapes: 74.5 us at S = 1 vs 60.6 us at S = 4).
  const int cps = cached_ctas_per_sm(pool->head_dim, pool->page_size, pool->dtype);
  return pa_decode_plan_splits(units, max_pages, pool->page_size, device_sm_count(),
                               cps < 3 ? cps : 3, 0);
}

int32_t pa_decode_auto_splits(int32_t num_seqs, int32_t num_kv_heads, int32_t max_ctx,
                              int32_t page_size) {
  if (num_seqs < 0 || num_kv_heads <= 0 || max_ctx < 0 || page_size <= 0) return -1;
  pa_kv_pool_t shape = {};
  shape.page_size = page_size;
  shape.num_kv_heads = num_kv_heads;
  shape.head_dim = 128;
  shape.dtype = PA_KV_BF16;
  const int32_t max_pages = max_ctx > 0 ? (int32_t)((max_ctx + (int64_t)page_size - 1) / page_size)
                                        : 1;
  return pa_decode_num_splits(&shape, num_seqs, max_pages, 0);
}

size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                 int32_t num_splits) {
  if (num_splits <= 1 || num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0) return 0;
  const size_t rows = (size_t)num_seqs * num_q_heads;
  return workspace_for(align256(rows * num_splits * head_dim * sizeof(float)) +
                           align256(rows * num_splits * sizeof(float)),
                       rows * sizeof(int32_t));
}

namespace {

// pa_decode, optionally with the fused cache write of pa_decode_append
// (k_new / v_new non-null).
pa_status_t decode_impl(const pa_kv_pool_t *pool, const void *q, int32_t num_seqs,
                        int32_t num_q_heads, const int32_t *block_tables, int32_t max_pages,
                        const int32_t *context_lens, float scale, float *out, void *workspace,
                        size_t workspace_bytes, int32_t num_splits, int32_t *d_err,
                        void *stream, const void *k_new, const void *v_new,
                        const int32_t *host_lens = nullptr) {
  g_last_error.clear();
  pa_status_t st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || max_pages <= 0 || num_splits < 0)
    return fail(PA_ERR_INVALID_ARG, "num_seqs=%d num_q_heads=%d max_pages=%d num_splits=%d",
                num_seqs, num_q_heads, max_pages, num_splits);
  if (num_q_heads % pool->num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads=%d is not a multiple of num_kv_heads=%d",
                num_q_heads, pool->num_kv_heads);
  const int G = num_q_heads / pool->num_kv_heads;
  if (G > kMaxGroup)
    return fail(PA_ERR_UNSUPPORTED, "GQA group %d > %d query heads per KV head", G, kMaxGroup);
  if (num_seqs > 65535 || pool->num_kv_heads > 65535)
    return fail(PA_ERR_UNSUPPORTED, "num_seqs and num_kv_heads must be <= 65535");
  if ((long long)max_pages * pool->page_size > (1LL << 30))
    return fail(PA_ERR_UNSUPPORTED, "max_pages * page_size too large");
  if (!(scale == scale)) return fail(PA_ERR_INVALID_ARG, "scale is NaN");
  if (num_seqs == 0) return PA_OK;
  if (!q || !block_tables || !context_lens || !out)
    return fail(PA_ERR_INVALID_ARG, "q, block_tables, context_lens and out are required");
  if (!aligned(q, 16) || !aligned(out, 16))
    return fail(PA_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  // with host context lengths (and automatic splits) the lengths choose the
  // split count and, for one split, a longest-first launch order
  uint16_t order[kMaxOrdered];
  int S = 0;
  int ordered = 0;  // 1: longest first; 2: and the units fill several waves
  if (host_lens != nullptr && num_splits == 0 && num_seqs <= kMaxOrdered) {
    const int cps = cached_ctas_per_sm(pool->head_dim, pool->page_size, pool->dtype);
    S = pa_decode_plan_lens(host_lens, num_seqs, pool->num_kv_heads, max_pages, pool->page_size,
                            device_sm_count(), cps, order);
    if (S == 1)
      ordered = (long long)num_seqs * pool->num_kv_heads >=
                        (long long)device_sm_count() * (cps < 3 ? cps : 3)
                    ? 2
                    : 1;
  }
  if (S <= 0) S = pa_decode_num_splits(pool, num_seqs, max_pages, num_splits);
  if (S <= 0) return fail(PA_ERR_INVALID_ARG, "could not plan splits");
  const int chunk = (max_pages + S - 1) / S;
  const size_t rows = (size_t)num_seqs * num_q_heads;
  const size_t o_bytes = align256(rows * S * pool->head_dim * sizeof(float));
  const size_t l_bytes = align256(rows * S * sizeof(float));
  if (S > 1) {
    if (workspace == nullptr ||
        workspace_bytes < workspace_for(o_bytes + l_bytes, rows * sizeof(int32_t)) ||
        !workspace_fits(workspace_bytes, o_bytes + l_bytes, rows * sizeof(int32_t)))
      return fail(PA_ERR_WORKSPACE, "workspace: need %zu bytes for %d splits, got %zu",
                  pa_decode_workspace_bytes(num_seqs, num_q_heads, pool->head_dim, S), S,
                  workspace == nullptr ? (size_t)0 : workspace_bytes);
    if (!aligned(workspace, 256))
      return fail(PA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  }
  char *part_base = S > 1 ? static_cast<char *>(workspace) + counter_region(workspace_bytes)
                          : nullptr;
  DecodeArgs a;
  a.k_pool = pool->k_pool;
  a.v_pool = pool->v_pool;
  a.k_sz = pool->k_sz;
  a.v_sz = pool->v_sz;
  a.num_pages = pool->num_pages;
  a.hkv = pool->num_kv_heads;
  a.q = q;
  a.B = num_seqs;
  a.hq = num_q_heads;
  a.block_tables = block_tables;
  a.max_pages = max_pages;
  a.ctx = context_lens;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = out;
  a.o_part = S > 1 ? reinterpret_cast<float *>(part_base) : nullptr;
  a.lse = S > 1 ? reinterpret_cast<float *>(part_base + o_bytes) : nullptr;
  a.counters = S > 1 ? static_cast<int32_t *>(workspace) : nullptr;
  a.S = S;
  a.S_main = S;
  a.pages_per_split = chunk;
  a.tbl_cap = chunk;
  a.window = 0;
  a.sinks = 0;
  a.tok_begin = 0;
  a.prior_o = nullptr;
  a.prior_lse = nullptr;
  a.n_prior = 0;
  a.keep_partials = 0;
  a.tok_end = 0x7fffffff;
  a.range_mode = 0;
  a.d_err = d_err;
  a.k_new = static_cast<const unsigned char *>(k_new);
  a.v_new = static_cast<const unsigned char *>(v_new);
  a.ordered = ordered;
  if (ordered)
    for (int i = 0; i < num_seqs; ++i) a.order[i] = (uint8_t)order[i];
  return cuda_status(launch_decode(pool->head_dim, pool->page_size, pool->dtype, a,
                                   static_cast<cudaStream_t>(stream)),
                     k_new ? "pa_decode_append launch" : "pa_decode launch");
}

}  // namespace

pa_status_t pa_decode(const pa_kv_pool_t *pool, const void *q, int32_t num_seqs,
                      int32_t num_q_heads, const int32_t *block_tables, int32_t max_pages,
                      const int32_t *context_lens, float scale, float *out, void *workspace,
                      size_t workspace_bytes, int32_t num_splits, int32_t *d_err,
                      void *stream) {
  return decode_impl(pool, q, num_seqs, num_q_heads, block_tables, max_pages, context_lens,
                     scale, out, workspace, workspace_bytes, num_splits, d_err, stream, nullptr,
                     nullptr);
}

pa_status_t pa_decode_append(const pa_kv_pool_t *pool, const void *q, const void *k_new,
                             const void *v_new, int32_t num_seqs, int32_t num_q_heads,
                             const int32_t *block_tables, int32_t max_pages,
                             const int32_t *context_lens, float scale, float *out,
                             void *workspace, size_t workspace_bytes, int32_t num_splits,
                             int32_t *d_err, void *stream) {
  g_last_error.clear();
  if (num_seqs > 0 && (k_new == nullptr || v_new == nullptr))
    return fail(PA_ERR_INVALID_ARG, "k_new and v_new are required");
  if (!aligned(k_new, 16) || !aligned(v_new, 16))
    return fail(PA_ERR_INVALID_ARG, "k_new/v_new must be 16-byte aligned");
  return decode_impl(pool, q, num_seqs, num_q_heads, block_tables, max_pages, context_lens,
                     scale, out, workspace, workspace_bytes, num_splits, d_err, stream,
                     num_seqs > 0 ? k_new : nullptr, num_seqs > 0 ? v_new : nullptr);
}

pa_status_t pa_decode_append_lens(const pa_kv_pool_t *pool, const void *q, const void *k_new,
                                  const void *v_new, int32_t num_seqs, int32_t num_q_heads,
                                  const int32_t *block_tables, int32_t max_pages,
                                  const int32_t *context_lens,
                                  const int32_t *host_context_lens, float scale, float *out,
                                  void *workspace, size_t workspace_bytes, int32_t num_splits,
                                  int32_t *d_err, void *stream) {
  g_last_error.clear();
  if (num_seqs > 0 && (k_new == nullptr || v_new == nullptr))
    return fail(PA_ERR_INVALID_ARG, "k_new and v_new are required");
  if (!aligned(k_new, 16) || !aligned(v_new, 16))
    return fail(PA_ERR_INVALID_ARG, "k_new/v_new must be 16-byte aligned");
  return decode_impl(pool, q, num_seqs, num_q_heads, block_tables, max_pages, context_lens,
                     scale, out, workspace, workspace_bytes, num_splits, d_err, stream,
                     num_seqs > 0 ? k_new : nullptr, num_seqs > 0 ? v_new : nullptr,
                     host_context_lens);
}

// ---------------------------------------------------------------- shared prefix
namespace {

// The cascade's second stream and its fork and join events, per device,
// created on first use, for calls captured into a CUDA graph (a device whose
// creation failed runs the three launches on the caller's stream).
// g_fork_mu serialises the fork sequence.
struct Fork {
  cudaStream_t s2 = nullptr;
  cudaEvent_t forked = nullptr, joined = nullptr;
  bool failed = false;
};
std::mutex g_fork_mu;
Fork g_fork[64];

Fork *fork_for_device() {
  const int dev = current_device();
  if (dev < 0 || dev >= 64) return nullptr;
  Fork &f = g_fork[dev];
  if (f.s2 == nullptr && !f.failed) {
    if (cudaStreamCreateWithFlags(&f.s2, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&f.forked, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&f.joined, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      f.s2 = nullptr;
      f.failed = true;
    }
  }
  return f.s2 != nullptr ? &f : nullptr;
}

struct PrefixPlan {
  int n_psplits, tiles_per_split;  // prefix kernel
  int S, chunk;                    // suffix decode
  size_t o_pre, lse_pre, o_part, lse, total;  // offsets / size after the counter region
};

bool plan_prefix(const pa_kv_pool_t *pool, int B, int Hq, int max_pages, int prefix_len,
                 int num_splits, PrefixPlan *pl) {
  const int P = pool->page_size;
  const int G = Hq / pool->num_kv_heads;
  const int lpb = prefix_len / P;
  const int sfx_pages = max_pages - lpb;
  if (sfx_pages < 1) return false;
  // prefix: splits of whole 64-token tiles, as many as pa_prefix_plan_splits
  // finds best for a pass that runs beside the suffix decode; the suffix
  // bytes are estimated from the table width (half of it attended on average)
  const int tiles = (prefix_len + prefix_tile_tokens() - 1) / prefix_tile_tokens();
  const int mtiles = (B * G + prefix_rows_per_cta() - 1) / prefix_rows_per_cta();
  const long long units = (long long)mtiles * pool->num_kv_heads;
  const int hd = pool->head_dim;
  const int row = pool->dtype == PA_KV_BF16 ? 2 * hd
                  : pool->dtype == PA_KV_U4_PER_TOKEN ? hd / 2 + 8 : hd + 8;
  const double sfx_bytes =
      (double)B * pool->num_kv_heads * 2.0 * row * ((double)sfx_pages * P) / 2.0;
  int tp = tiles > 0 ? pa_prefix_plan_splits(units, tiles, device_sm_count(),
                                             cached_ctas_per_sm(hd, P, pool->dtype), sfx_bytes)
                     : 1;
  if (tp < 1) tp = tiles > 0 ? tiles : 1;
  if (tiles > 0 && (tiles + tp - 1) / tp > kMaxSplits) tp = (tiles + kMaxSplits - 1) / kMaxSplits;
  pl->tiles_per_split = tp;
  pl->n_psplits = tiles > 0 ? (tiles + tp - 1) / tp : 0;
  // suffix: the plain decode's split planning over the suffix pages
  pl->S = pa_decode_num_splits(pool, B, sfx_pages, num_splits);
  if (pl->S <= 0) return false;
  pl->chunk = (sfx_pages + pl->S - 1) / pl->S;
  const size_t R = (size_t)B * Hq, D = pool->head_dim;
  size_t off = 0;
  pl->o_pre = off;    off += align256(pl->n_psplits * R * D * sizeof(float));
  pl->lse_pre = off;  off += align256(pl->n_psplits * R * sizeof(float));
  pl->o_part = off;   off += align256(R * pl->S * D * sizeof(float));
  pl->lse = off;      off += align256(R * pl->S * sizeof(float));
  pl->total = off;
  return true;
}

}  // namespace

size_t pa_decode_shared_prefix_workspace_bytes(const pa_kv_pool_t *pool, int32_t num_seqs,
                                               int32_t num_q_heads, int32_t max_pages,
                                               int32_t prefix_len, int32_t num_splits) {
  if (pool == nullptr || num_seqs <= 0 || num_q_heads <= 0 || pool->num_kv_heads <= 0 ||
      pool->page_size <= 0 || prefix_len < 0 || prefix_len % pool->page_size != 0 ||
      num_q_heads % pool->num_kv_heads != 0)
    return 0;
  PrefixPlan pl;
  if (!plan_prefix(pool, num_seqs, num_q_heads, max_pages, prefix_len, num_splits, &pl)) return 0;
  return workspace_for(pl.total, (size_t)num_seqs * num_q_heads * sizeof(int32_t));
}

pa_status_t pa_decode_shared_prefix(const pa_kv_pool_t *pool, const void *q, int32_t num_seqs,
                                    int32_t num_q_heads, const int32_t *prefix_pages,
                                    int32_t prefix_len, const int32_t *block_tables,
                                    int32_t max_pages, const int32_t *context_lens, float scale,
                                    float *out, void *workspace, size_t workspace_bytes,
                                    int32_t num_splits, int32_t *d_err, void *stream) {
  g_last_error.clear();
  pa_status_t st = check_pool(pool);
  if (st != PA_OK) return st;
  if (pool->dtype != PA_KV_BF16)
    return fail(PA_ERR_UNSUPPORTED, "shared-prefix decode supports bf16 pools only");
  if (prefix_len < 0 || prefix_len % pool->page_size != 0)
    return fail(PA_ERR_INVALID_ARG, "prefix_len=%d must be a non-negative multiple of %d",
                prefix_len, pool->page_size);
  if (prefix_len == 0)
    return pa_decode(pool, q, num_seqs, num_q_heads, block_tables, max_pages, context_lens, scale,
                     out, workspace, workspace_bytes, num_splits, d_err, stream);
  if (num_seqs < 0 || num_q_heads <= 0 || max_pages <= 0 || num_splits < 0)
    return fail(PA_ERR_INVALID_ARG, "num_seqs=%d num_q_heads=%d max_pages=%d num_splits=%d",
                num_seqs, num_q_heads, max_pages, num_splits);
  if (num_q_heads % pool->num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads=%d is not a multiple of num_kv_heads=%d",
                num_q_heads, pool->num_kv_heads);
  const int G = num_q_heads / pool->num_kv_heads;
  if (G > kMaxGroup)
    return fail(PA_ERR_UNSUPPORTED, "GQA group %d > %d query heads per KV head", G, kMaxGroup);
  if (prefix_len / pool->page_size >= max_pages)
    return fail(PA_ERR_INVALID_ARG, "prefix of %d pages leaves no room in tables of %d pages",
                prefix_len / pool->page_size, max_pages);
  if (num_seqs > 65535 || (long long)max_pages * pool->page_size > (1LL << 30))
    return fail(PA_ERR_UNSUPPORTED, "too many sequences or pages");
  if (!(scale == scale)) return fail(PA_ERR_INVALID_ARG, "scale is NaN");
  if (num_seqs == 0) return PA_OK;
  if (!q || !prefix_pages || !block_tables || !context_lens || !out)
    return fail(PA_ERR_INVALID_ARG,
                "q, prefix_pages, block_tables, context_lens and out are required");
  if (!aligned(q, 16) || !aligned(out, 16))
    return fail(PA_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  PrefixPlan pl;
  if (!plan_prefix(pool, num_seqs, num_q_heads, max_pages, prefix_len, num_splits, &pl))
    return fail(PA_ERR_INVALID_ARG, "could not plan the shared-prefix decode");
  const size_t counter_bytes = (size_t)num_seqs * num_q_heads * sizeof(int32_t);
  if (workspace == nullptr || workspace_bytes < workspace_for(pl.total, counter_bytes) ||
      !workspace_fits(workspace_bytes, pl.total, counter_bytes))
    return fail(PA_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu",
                workspace_for(pl.total, counter_bytes),
                workspace == nullptr ? (size_t)0 : workspace_bytes);
  if (!aligned(workspace, 256)) return fail(PA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  // partials after the workspace's counter region (which this path leaves alone)
  char *ws = static_cast<char *>(workspace) + counter_region(workspace_bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  PrefixArgs pa;
  pa.k_pool = pool->k_pool;
  pa.v_pool = pool->v_pool;
  pa.num_pages = pool->num_pages;
  pa.hkv = pool->num_kv_heads;
  pa.q = q;
  pa.B = num_seqs;
  pa.hq = num_q_heads;
  pa.prefix_pages = prefix_pages;
  pa.prefix_len = prefix_len;
  pa.tiles_per_split = pl.tiles_per_split;
  pa.n_psplits = pl.n_psplits;
  pa.scale_log2 = scale * 1.4426950408889634f;
  pa.o_pre = reinterpret_cast<float *>(ws + pl.o_pre);
  pa.lse_pre = reinterpret_cast<float *>(ws + pl.lse_pre);
  pa.d_err = d_err;
  DecodeArgs a;
  a.k_pool = pool->k_pool;
  a.v_pool = pool->v_pool;
  a.k_sz = pool->k_sz;
  a.v_sz = pool->v_sz;
  a.num_pages = pool->num_pages;
  a.hkv = pool->num_kv_heads;
  a.q = q;
  a.B = num_seqs;
  a.hq = num_q_heads;
  a.block_tables = block_tables;
  a.max_pages = max_pages;
  a.ctx = context_lens;
  a.scale_log2 = pa.scale_log2;
  a.out = out;
  a.o_part = reinterpret_cast<float *>(ws + pl.o_part);
  a.lse = reinterpret_cast<float *>(ws + pl.lse);
  a.counters = nullptr;  // keep_partials: the suffix CTAs merge nothing themselves
  a.S = pl.S;
  a.S_main = pl.S;
  a.pages_per_split = pl.chunk;
  a.tbl_cap = pl.chunk;
  a.window = 0;
  a.sinks = 0;
  a.tok_begin = prefix_len;
  a.d_err = d_err;
  // Three launches: the prefix pass, the suffix decode (which writes its split
  // partials, an empty split lse = -inf, instead of merging), then one merge
  // of the suffix splits and the prefix splits per row with its loads batched
  // (a decode CTA merging prefix partials in its epilogue measured slower).
  // The prefix pass and the decode run side by side, the prefix CTAs placed
  // first. Called eagerly, all three go on `stream`, each a programmatic
  // dependent of the one before: the prefix pass releases the decode as soon
  // as its own wait for the earlier work returns, and the decode's last CTA
  // waits for the prefix pass, so the merge follows both with no event
  // between streams. Captured into a CUDA graph, the decode goes on a second
  // stream forked from `stream` and joined back before the merge: there the
  // fork and join are graph edges, and the two branches start at once.
  a.prior_o = nullptr;
  a.prior_lse = nullptr;
  a.n_prior = 0;
  a.keep_partials = 1;
  a.tok_end = 0x7fffffff;
  a.range_mode = 0;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  st = cuda_status(cudaStreamIsCapturing(s, &cap), "pa_decode_shared_prefix capture query");
  if (st != PA_OK) return st;
  if (cap == cudaStreamCaptureStatusNone) {
    a.pdl_defer = 1;
    st = cuda_status(launch_prefix(pool->head_dim, pool->page_size, pa, true, s),
                     "pa_decode_shared_prefix prefix launch");
    if (st == PA_OK)
      st = cuda_status(launch_decode(pool->head_dim, pool->page_size, pool->dtype, a, s),
                       "pa_decode_shared_prefix suffix launch");
  } else {
    std::lock_guard<std::mutex> lock(g_fork_mu);
    Fork *f = fork_for_device();
    if (f != nullptr) {
      st = cuda_status(cudaEventRecord(f->forked, s), "pa_decode_shared_prefix fork");
      if (st == PA_OK)
        st = cuda_status(cudaStreamWaitEvent(f->s2, f->forked, 0), "pa_decode_shared_prefix fork");
    }
    if (st == PA_OK)
      st = cuda_status(launch_prefix(pool->head_dim, pool->page_size, pa, true, s),
                       "pa_decode_shared_prefix prefix launch");
    if (st == PA_OK)
      st = cuda_status(launch_decode(pool->head_dim, pool->page_size, pool->dtype, a,
                                     f != nullptr ? f->s2 : s),
                       "pa_decode_shared_prefix suffix launch");
    if (st == PA_OK && f != nullptr) {
      st = cuda_status(cudaEventRecord(f->joined, f->s2), "pa_decode_shared_prefix join");
      if (st == PA_OK)
        st = cuda_status(cudaStreamWaitEvent(s, f->joined, 0), "pa_decode_shared_prefix join");
    }
  }
  if (st != PA_OK) return st;
  return cuda_status(launch_splitkv_reduce(a.o_part, a.lse, num_seqs, num_q_heads, pl.S,
                                           pool->head_dim, out, true, s, pa.o_pre, pa.lse_pre,
                                           pl.n_psplits),
                     "pa_decode_shared_prefix merge launch");
}

// ---------------------------------------------------------------- token ranges
namespace {

// Splits and partial slots of pa_decode_range: the range's logical pages
// [tok_begin / P, ceil(min(tok_end, max_pages * P) / P)) split like a decode.
int range_splits(const pa_kv_pool_t *pool, int B, int max_pages, int tok_begin, int tok_end,
                 int num_splits) {
  const int P = pool->page_size;
  const long long end = std::min<long long>(tok_end, (long long)max_pages * P);
  const int pages = (int)((end + P - 1) / P) - tok_begin / P;
  return pa_decode_num_splits(pool, B, pages < 1 ? 1 : pages, num_splits);
}

}  // namespace

size_t pa_decode_range_workspace_bytes(const pa_kv_pool_t *pool, int32_t num_seqs,
                                       int32_t num_q_heads, int32_t max_pages, int32_t tok_begin,
                                       int32_t tok_end, int32_t num_splits) {
  if (pool == nullptr || num_seqs <= 0 || num_q_heads <= 0 || max_pages <= 0 || tok_begin < 0 ||
      tok_end < tok_begin || num_splits < 0 || pool->page_size <= 0)
    return 0;
  const int S = range_splits(pool, num_seqs, max_pages, tok_begin, tok_end, num_splits);
  return S > 1 ? pa_decode_workspace_bytes(num_seqs, num_q_heads, pool->head_dim, S) : 0;
}

pa_status_t pa_decode_range(const pa_kv_pool_t *pool, const void *q, int32_t num_seqs,
                            int32_t num_q_heads, const int32_t *block_tables, int32_t max_pages,
                            const int32_t *context_lens, int32_t tok_begin, int32_t tok_end,
                            float scale, float *o_out, float *lse_out, void *workspace,
                            size_t workspace_bytes, int32_t num_splits, int32_t *d_err,
                            void *stream) {
  g_last_error.clear();
  pa_status_t st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || max_pages <= 0 || num_splits < 0)
    return fail(PA_ERR_INVALID_ARG, "num_seqs=%d num_q_heads=%d max_pages=%d num_splits=%d",
                num_seqs, num_q_heads, max_pages, num_splits);
  if (tok_begin < 0 || tok_end < tok_begin || tok_begin % pool->page_size != 0)
    return fail(PA_ERR_INVALID_ARG,
                "token range [%d, %d) must start on a page boundary and not be reversed",
                tok_begin, tok_end);
  if (tok_begin >= max_pages * pool->page_size && tok_end > tok_begin)
    return fail(PA_ERR_INVALID_ARG, "tok_begin=%d is past the tables' %d pages", tok_begin,
                max_pages);
  if (num_q_heads % pool->num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads=%d is not a multiple of num_kv_heads=%d",
                num_q_heads, pool->num_kv_heads);
  const int G = num_q_heads / pool->num_kv_heads;
  if (G > kMaxGroup)
    return fail(PA_ERR_UNSUPPORTED, "GQA group %d > %d query heads per KV head", G, kMaxGroup);
  if (num_seqs > 65535 || (long long)max_pages * pool->page_size > (1LL << 30))
    return fail(PA_ERR_UNSUPPORTED, "too many sequences or pages");
  if (!(scale == scale)) return fail(PA_ERR_INVALID_ARG, "scale is NaN");
  if (num_seqs == 0) return PA_OK;
  if (!q || !block_tables || !context_lens || !o_out || !lse_out)
    return fail(PA_ERR_INVALID_ARG, "q, block_tables, context_lens, o_out and lse_out are required");
  if (!aligned(q, 16) || !aligned(o_out, 16) || !aligned(lse_out, 4))
    return fail(PA_ERR_INVALID_ARG, "q and o_out must be 16-byte aligned");
  if (tok_begin >= max_pages * pool->page_size) tok_begin = tok_end = 0;  // empty range
  const int S = range_splits(pool, num_seqs, max_pages, tok_begin, tok_end, num_splits);
  if (S <= 0) return fail(PA_ERR_INVALID_ARG, "could not plan splits");
  const size_t rows = (size_t)num_seqs * num_q_heads;
  const size_t o_bytes = align256(rows * S * pool->head_dim * sizeof(float));
  const size_t l_bytes = align256(rows * S * sizeof(float));
  if (S > 1) {
    if (workspace == nullptr ||
        workspace_bytes < workspace_for(o_bytes + l_bytes, rows * sizeof(int32_t)) ||
        !workspace_fits(workspace_bytes, o_bytes + l_bytes, rows * sizeof(int32_t)))
      return fail(PA_ERR_WORKSPACE, "workspace: need %zu bytes for %d splits, got %zu",
                  pa_decode_workspace_bytes(num_seqs, num_q_heads, pool->head_dim, S), S,
                  workspace == nullptr ? (size_t)0 : workspace_bytes);
    if (!aligned(workspace, 256)) return fail(PA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  }
  char *part_base = S > 1 ? static_cast<char *>(workspace) + counter_region(workspace_bytes)
                          : nullptr;
  const int P = pool->page_size;
  const long long end = std::min<long long>(tok_end, (long long)max_pages * P);
  const int pages = std::max(1, (int)((end + P - 1) / P) - tok_begin / P);
  DecodeArgs a;
  a.k_pool = pool->k_pool;
  a.v_pool = pool->v_pool;
  a.k_sz = pool->k_sz;
  a.v_sz = pool->v_sz;
  a.num_pages = pool->num_pages;
  a.hkv = pool->num_kv_heads;
  a.q = q;
  a.B = num_seqs;
  a.hq = num_q_heads;
  a.block_tables = block_tables;
  a.max_pages = max_pages;
  a.ctx = context_lens;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = o_out;
  // one split writes o_out / lse_out directly ([row][1][D] is [row][D]); more
  // write partials after the workspace's counter region, which keep_partials
  // leaves alone
  a.o_part = S > 1 ? reinterpret_cast<float *>(part_base) : o_out;
  a.lse = S > 1 ? reinterpret_cast<float *>(part_base + o_bytes) : lse_out;
  a.counters = nullptr;
  a.S = S;
  a.S_main = S;
  a.pages_per_split = (pages + S - 1) / S;
  a.tbl_cap = a.pages_per_split;
  a.window = 0;
  a.sinks = 0;
  a.tok_begin = tok_begin;
  a.prior_o = nullptr;
  a.prior_lse = nullptr;
  a.n_prior = 0;
  a.keep_partials = 1;
  a.tok_end = tok_end;
  a.range_mode = 1;
  a.d_err = d_err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = cuda_status(launch_decode(pool->head_dim, P, pool->dtype, a, s), "pa_decode_range launch");
  if (st != PA_OK || S == 1) return st;
  return cuda_status(launch_splitkv_reduce(a.o_part, a.lse, num_seqs, num_q_heads, S,
                                           pool->head_dim, o_out, true, s, nullptr, nullptr, 0,
                                           lse_out),
                     "pa_decode_range merge launch");
}

// ------------------------------------------------------------ host packet step
size_t pa_step_packet_layout(const pa_kv_pool_t *pool, int32_t num_seqs, int32_t num_q_heads,
                             int32_t max_pages, int32_t num_new, size_t *offsets) {
  if (pool == nullptr || num_seqs < 0 || num_q_heads <= 0 || max_pages <= 0 ||
      (num_new < 0 && num_new != PA_STEP_NEWEST_PER_SEQ) || pool->num_kv_heads <= 0 ||
      pool->head_dim <= 0)
    return 0;
  const size_t D = (size_t)pool->head_dim;
  // one row per sequence (its newest token): no index sections
  const size_t rows = num_new == PA_STEP_NEWEST_PER_SEQ ? (size_t)num_seqs : (size_t)num_new;
  const size_t idx = num_new == PA_STEP_NEWEST_PER_SEQ ? 0 : (size_t)num_new;
  const size_t sizes[7] = {
      (size_t)num_seqs * num_q_heads * D * 2,    // q
      rows * pool->num_kv_heads * D * 2,         // k_new
      rows * pool->num_kv_heads * D * 2,         // v_new
      idx * 4,                                   // seq_idx
      idx * 4,                                   // pos
      (size_t)num_seqs * max_pages * 4,              // block_tables
      (size_t)num_seqs * 4};                         // context_lens
  size_t at = 0;
  for (int i = 0; i < 7; ++i) {
    if (offsets) offsets[i] = at;
    at = align256(at + sizes[i]);
  }
  return at;
}

pa_status_t pa_decode_step_host(const pa_kv_pool_t *pool, const void *packet_host,
                                void *packet_dev, size_t packet_bytes, int32_t num_seqs,
                                int32_t num_q_heads, int32_t max_pages, int32_t num_new,
                                float scale, float *out_dev, float *out_host, void *workspace,
                                size_t workspace_bytes, int32_t num_splits, int32_t *d_err,
                                void *stream, int32_t synchronize) {
  g_last_error.clear();
  pa_status_t st = check_pool(pool);
  if (st != PA_OK) return st;
  size_t off[7];
  const size_t need = pa_step_packet_layout(pool, num_seqs, num_q_heads, max_pages, num_new, off);
  if (need == 0)
    return fail(PA_ERR_INVALID_ARG, "num_seqs=%d num_q_heads=%d max_pages=%d num_new=%d",
                num_seqs, num_q_heads, max_pages, num_new);
  if (packet_bytes != need)
    return fail(PA_ERR_INVALID_ARG, "packet_bytes=%zu, the layout needs %zu", packet_bytes, need);
  if (!packet_host || !packet_dev || (num_seqs > 0 && (!out_dev || !out_host)))
    return fail(PA_ERR_INVALID_ARG, "packet_host, packet_dev, out_dev and out_host are required");
  if (!aligned(packet_dev, 256))
    return fail(PA_ERR_INVALID_ARG, "packet_dev must be 256-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = cuda_status(cudaMemcpyAsync(packet_dev, packet_host, packet_bytes, cudaMemcpyHostToDevice, s),
                   "pa_decode_step_host packet copy");
  if (st != PA_OK) return st;
  char *pd = static_cast<char *>(packet_dev);
  const int32_t *tables = reinterpret_cast<const int32_t *>(pd + off[5]);
  const int32_t *ctx = reinterpret_cast<const int32_t *>(pd + off[6]);
  // the packet's context lengths are on the host too: they schedule the launch
  const int32_t *host_ctx =
      reinterpret_cast<const int32_t *>(static_cast<const char *>(packet_host) + off[6]);
  if (num_new == PA_STEP_NEWEST_PER_SEQ) {  // cache write fused into the decode
    st = pa_decode_append_lens(pool, pd + off[0], pd + off[1], pd + off[2], num_seqs,
                               num_q_heads, tables, max_pages, ctx, host_ctx, scale, out_dev,
                               workspace, workspace_bytes, num_splits, d_err, stream);
  } else {
    st = pa_kv_append(pool, pd + off[1], pd + off[2],
                      reinterpret_cast<const int32_t *>(pd + off[3]),
                      reinterpret_cast<const int32_t *>(pd + off[4]), num_new, tables, num_seqs,
                      max_pages, d_err, stream);
    if (st == PA_OK)
      st = decode_impl(pool, pd + off[0], num_seqs, num_q_heads, tables, max_pages, ctx, scale,
                       out_dev, workspace, workspace_bytes, num_splits, d_err, stream, nullptr,
                       nullptr, host_ctx);
  }
  if (st != PA_OK || num_seqs == 0) return st;
  st = cuda_status(cudaMemcpyAsync(out_host, out_dev,
                                   (size_t)num_seqs * num_q_heads * pool->head_dim * sizeof(float),
                                   cudaMemcpyDeviceToHost, s),
                   "pa_decode_step_host output copy");
  if (st != PA_OK || !synchronize) return st;
  return cuda_status(cudaStreamSynchronize(s), "pa_decode_step_host synchronize");
}

// ------------------------------------------------------------ captured step
struct pa_step_graph {
  cudaGraphExec_t exec;
};

pa_status_t pa_step_graph_create(const pa_kv_pool_t *pool, const void *packet_host,
                                 void *packet_dev, size_t packet_bytes, int32_t num_seqs,
                                 int32_t num_q_heads, int32_t max_pages, int32_t num_new,
                                 float scale, float *out_dev, float *out_host, void *workspace,
                                 size_t workspace_bytes, int32_t num_splits, int32_t *d_err,
                                 pa_step_graph_t **graph) {
  g_last_error.clear();
  if (graph == nullptr) return fail(PA_ERR_INVALID_ARG, "graph is NULL");
  *graph = nullptr;
  pa_status_t st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_seqs <= 0 || num_q_heads <= 0 || max_pages <= 0)
    return fail(PA_ERR_INVALID_ARG, "num_seqs=%d num_q_heads=%d max_pages=%d", num_seqs,
                num_q_heads, max_pages);
  // plan (and set the kernels' shared-memory limits) before capturing, so
  // that capture records stream work only
  if (pa_decode_num_splits(pool, num_seqs, max_pages, num_splits) <= 0)
    return fail(PA_ERR_INVALID_ARG, "could not plan splits");
  cudaStream_t cs = nullptr;
  st = cuda_status(cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking),
                   "pa_step_graph_create stream");
  if (st != PA_OK) return st;
  st = cuda_status(cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal),
                   "pa_step_graph_create begin capture");
  if (st != PA_OK) {
    cudaStreamDestroy(cs);
    return st;
  }
  const pa_status_t step = pa_decode_step_host(pool, packet_host, packet_dev, packet_bytes,
                                               num_seqs, num_q_heads, max_pages, num_new, scale,
                                               out_dev, out_host, workspace, workspace_bytes,
                                               num_splits, d_err, cs, 0);
  const std::string step_error = g_last_error;
  cudaGraph_t g = nullptr;
  const cudaError_t end = cudaStreamEndCapture(cs, &g);
  cudaStreamDestroy(cs);
  if (step != PA_OK) {
    if (g) cudaGraphDestroy(g);
    g_last_error = step_error;
    return step;
  }
  if (end != cudaSuccess || g == nullptr) {
    if (g) cudaGraphDestroy(g);
    return cuda_status(end != cudaSuccess ? end : cudaErrorUnknown,
                       "pa_step_graph_create end capture");
  }
  cudaGraphExec_t exec = nullptr;
  const cudaError_t inst = cudaGraphInstantiate(&exec, g, 0);
  cudaGraphDestroy(g);
  if (inst != cudaSuccess) return cuda_status(inst, "pa_step_graph_create instantiate");
  pa_step_graph *h = new (std::nothrow) pa_step_graph;
  if (h == nullptr) {
    cudaGraphExecDestroy(exec);
    return fail(PA_ERR_INVALID_ARG, "out of host memory");
  }
  h->exec = exec;
  *graph = h;
  return PA_OK;
}

pa_status_t pa_step_graph_launch(pa_step_graph_t *graph, void *stream, int32_t synchronize) {
  g_last_error.clear();
  if (graph == nullptr) return fail(PA_ERR_INVALID_ARG, "graph is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  pa_status_t st = cuda_status(cudaGraphLaunch(graph->exec, s), "pa_step_graph_launch");
  if (st != PA_OK || !synchronize) return st;
  return cuda_status(cudaStreamSynchronize(s), "pa_step_graph_launch synchronize");
}

void pa_step_graph_destroy(pa_step_graph_t *graph) {
  if (graph == nullptr) return;
  cudaGraphExecDestroy(graph->exec);
  delete graph;
}

pa_status_t pa_merge_partials(const float *o_parts, const float *lse_parts, int32_t num_parts,
                              int32_t rows, int32_t head_dim, int64_t o_part_stride,
                              int64_t lse_part_stride, float *out, float *lse_out,
                              void *stream) {
  g_last_error.clear();
  if (num_parts < 1 || rows < 0 || head_dim <= 0 || head_dim % 4 != 0 || head_dim > 512)
    return fail(PA_ERR_INVALID_ARG, "num_parts=%d rows=%d head_dim=%d", num_parts, rows,
                head_dim);
  if (o_part_stride == 0) o_part_stride = (int64_t)rows * head_dim;
  if (lse_part_stride == 0) lse_part_stride = rows;
  if (num_parts > 1 && (o_part_stride < (int64_t)rows * head_dim || o_part_stride % 4 != 0 ||
                        lse_part_stride < rows))
    return fail(PA_ERR_INVALID_ARG,
                "part strides %lld / %lld: parts overlap or break 16-byte alignment",
                (long long)o_part_stride, (long long)lse_part_stride);
  if (rows == 0) return PA_OK;
  if (!o_parts || !lse_parts || !out)
    return fail(PA_ERR_INVALID_ARG, "o_parts, lse_parts and out are required");
  if (!aligned(o_parts, 16) || !aligned(out, 16))
    return fail(PA_ERR_INVALID_ARG, "o_parts and out must be 16-byte aligned");
  return cuda_status(launch_splitkv_reduce(nullptr, nullptr, rows, 1, 0, head_dim, out, true,
                                           static_cast<cudaStream_t>(stream), o_parts, lse_parts,
                                           num_parts, lse_out, (size_t)o_part_stride,
                                           (size_t)lse_part_stride),
                     "pa_merge_partials launch");
}

pa_status_t pa_splitkv_reduce(const float *o_part, const float *lse, int32_t num_seqs,
                              int32_t num_q_heads, int32_t num_splits, int32_t head_dim,
                              float *out, void *stream) {
  g_last_error.clear();
  if (num_seqs < 0 || num_q_heads <= 0 || num_splits < 1 || num_splits > kMaxSplits ||
      head_dim <= 0 || head_dim % 4 != 0 || head_dim > 512)
    return fail(PA_ERR_INVALID_ARG, "num_seqs=%d num_q_heads=%d num_splits=%d head_dim=%d",
                num_seqs, num_q_heads, num_splits, head_dim);
  if (num_seqs == 0) return PA_OK;
  if (!o_part || !lse || !out) return fail(PA_ERR_INVALID_ARG, "o_part, lse and out are required");
  if (!aligned(o_part, 16) || !aligned(out, 16))
    return fail(PA_ERR_INVALID_ARG, "o_part and out must be 16-byte aligned");
  if ((long long)num_seqs * num_q_heads > (1LL << 31) - 4)
    return fail(PA_ERR_UNSUPPORTED, "too many rows");
  return cuda_status(launch_splitkv_reduce(o_part, lse, num_seqs, num_q_heads, num_splits,
                                           head_dim, out, false,
                                           static_cast<cudaStream_t>(stream)),
                     "pa_splitkv_reduce launch");
}

pa_status_t pa_validate_tables(const int32_t *block_tables, int32_t num_seqs, int32_t max_pages,
                               const int32_t *context_lens, int32_t num_pages, int32_t page_size,
                               int32_t *d_err, void *stream) {
  g_last_error.clear();
  if (num_seqs < 0 || max_pages <= 0 || num_pages <= 0 || page_size <= 0)
    return fail(PA_ERR_INVALID_ARG, "num_seqs=%d max_pages=%d num_pages=%d page_size=%d",
                num_seqs, max_pages, num_pages, page_size);
  if (d_err == nullptr) return fail(PA_ERR_INVALID_ARG, "d_err is required");
  if (num_seqs == 0) return PA_OK;
  if (!block_tables || !context_lens)
    return fail(PA_ERR_INVALID_ARG, "block_tables and context_lens are required");
  return cuda_status(launch_validate_tables(block_tables, num_seqs, max_pages, context_lens,
                                            num_pages, page_size, d_err,
                                            static_cast<cudaStream_t>(stream)),
                     "pa_validate_tables launch");
}


// ------------------------------------------------------------ sinks + window
namespace {

struct WindowPlan {
  int S_main, S, chunk, tbl_cap;
};

bool plan_window(const pa_kv_pool_t *pool, int B, int max_pages, int sinks, int window,
                 int num_splits, WindowPlan *pl) {
  const int P = pool->page_size;
  // the main range [max(ctx - window, min(sinks, ctx)), ctx) spans at most this many pages
  long long wp = ((long long)window + P - 1) / P + 1;
  if (wp > max_pages) wp = max_pages;
  pl->S_main = pa_decode_num_splits(pool, B, (int)wp, num_splits);
  if (pl->S_main <= 0) return false;
  pl->chunk = ((int)wp + pl->S_main - 1) / pl->S_main;
  // the sinks are a second range of split 0 (no split of their own): its
  // table slice holds pages [0, ceil(min(sinks, ctx) / P)) and then a chunk
  pl->S = pl->S_main;
  const long long sink_tok = std::min<long long>(sinks, (long long)max_pages * P);
  const long long sink_pages = (sink_tok + P - 1) / P;
  pl->tbl_cap = (int)(pl->chunk + sink_pages);
  return pl->tbl_cap <= kMaxPagesPerSplit;
}

}  // namespace

size_t pa_decode_window_workspace_bytes(const pa_kv_pool_t *pool, int32_t num_seqs,
                                        int32_t num_q_heads, int32_t max_pages, int32_t sinks,
                                        int32_t window, int32_t num_splits) {
  if (pool == nullptr || num_seqs <= 0 || num_q_heads <= 0 || max_pages <= 0 || sinks < 0 ||
      window <= 0 || pool->page_size <= 0)
    return 0;
  WindowPlan pl;
  if (!plan_window(pool, num_seqs, max_pages, sinks, window, num_splits, &pl)) return 0;
  return pa_decode_workspace_bytes(num_seqs, num_q_heads, pool->head_dim, pl.S);
}

pa_status_t pa_decode_window(const pa_kv_pool_t *pool, const void *q, int32_t num_seqs,
                             int32_t num_q_heads, const int32_t *block_tables, int32_t max_pages,
                             const int32_t *context_lens, int32_t sinks, int32_t window,
                             float scale, float *out, void *workspace, size_t workspace_bytes,
                             int32_t num_splits, int32_t *d_err, void *stream) {
  g_last_error.clear();
  pa_status_t st = check_pool(pool);
  if (st != PA_OK) return st;
  if (window < 0 || sinks < 0)
    return fail(PA_ERR_INVALID_ARG, "window=%d sinks=%d must be non-negative", window, sinks);
  if (window == 0)  // no window: every token is kept
    return pa_decode(pool, q, num_seqs, num_q_heads, block_tables, max_pages, context_lens, scale,
                     out, workspace, workspace_bytes, num_splits, d_err, stream);
  if (num_seqs < 0 || num_q_heads <= 0 || max_pages <= 0 || num_splits < 0)
    return fail(PA_ERR_INVALID_ARG, "num_seqs=%d num_q_heads=%d max_pages=%d num_splits=%d",
                num_seqs, num_q_heads, max_pages, num_splits);
  if (num_q_heads % pool->num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads=%d is not a multiple of num_kv_heads=%d",
                num_q_heads, pool->num_kv_heads);
  const int G = num_q_heads / pool->num_kv_heads;
  if (G > kMaxGroup)
    return fail(PA_ERR_UNSUPPORTED, "GQA group %d > %d query heads per KV head", G, kMaxGroup);
  if (num_seqs > 65535 || (long long)max_pages * pool->page_size > (1LL << 30))
    return fail(PA_ERR_UNSUPPORTED, "too many sequences or pages");
  if (!(scale == scale)) return fail(PA_ERR_INVALID_ARG, "scale is NaN");
  if (num_seqs == 0) return PA_OK;
  if (!q || !block_tables || !context_lens || !out)
    return fail(PA_ERR_INVALID_ARG, "q, block_tables, context_lens and out are required");
  if (!aligned(q, 16) || !aligned(out, 16))
    return fail(PA_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  WindowPlan pl;
  if (!plan_window(pool, num_seqs, max_pages, sinks, window, num_splits, &pl))
    return fail(PA_ERR_UNSUPPORTED, "windowed decode: at most %d sink pages are supported",
                kMaxPagesPerSplit);
  if (pl.S + 1 > kMaxSplits + 1) return fail(PA_ERR_UNSUPPORTED, "too many splits");
  const size_t rows = (size_t)num_seqs * num_q_heads;
  const size_t o_bytes = align256(rows * pl.S * pool->head_dim * sizeof(float));
  const size_t l_bytes = align256(rows * pl.S * sizeof(float));
  if (pl.S > 1) {
    if (workspace == nullptr ||
        workspace_bytes < workspace_for(o_bytes + l_bytes, rows * sizeof(int32_t)) ||
        !workspace_fits(workspace_bytes, o_bytes + l_bytes, rows * sizeof(int32_t)))
      return fail(PA_ERR_WORKSPACE, "workspace: need %zu bytes for %d splits, got %zu",
                  pa_decode_workspace_bytes(num_seqs, num_q_heads, pool->head_dim, pl.S), pl.S,
                  workspace == nullptr ? (size_t)0 : workspace_bytes);
    if (!aligned(workspace, 256)) return fail(PA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  }
  DecodeArgs a;
  a.k_pool = pool->k_pool;
  a.v_pool = pool->v_pool;
  a.k_sz = pool->k_sz;
  a.v_sz = pool->v_sz;
  a.num_pages = pool->num_pages;
  a.hkv = pool->num_kv_heads;
  a.q = q;
  a.B = num_seqs;
  a.hq = num_q_heads;
  a.block_tables = block_tables;
  a.max_pages = max_pages;
  a.ctx = context_lens;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = out;
  char *ws = pl.S > 1 ? static_cast<char *>(workspace) + counter_region(workspace_bytes)
                      : nullptr;
  a.o_part = pl.S > 1 ? reinterpret_cast<float *>(ws) : nullptr;
  a.lse = pl.S > 1 ? reinterpret_cast<float *>(ws + o_bytes) : nullptr;
  a.counters = pl.S > 1 ? static_cast<int32_t *>(workspace) : nullptr;
  a.S = pl.S;
  a.S_main = pl.S_main;
  a.pages_per_split = pl.chunk;
  a.tbl_cap = pl.tbl_cap;
  a.window = window;
  a.sinks = sinks;
  a.tok_begin = 0;
  a.prior_o = nullptr;
  a.prior_lse = nullptr;
  a.n_prior = 0;
  a.keep_partials = 0;
  a.tok_end = 0x7fffffff;
  a.range_mode = 0;
  a.d_err = d_err;
  return cuda_status(launch_decode(pool->head_dim, pool->page_size, pool->dtype, a,
                                   static_cast<cudaStream_t>(stream)),
                     "pa_decode_window launch");
}

}  // extern "C"
