// Host-side declarations shared by the pagedattn translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pagedattn.h"

namespace pa {

// Most sequences a longest-first launch order can name (the order travels as
// a kernel parameter of one byte per sequence).
constexpr int kMaxOrdered = 256;

// Largest GQA group a decode CTA serves (query heads per KV head).
constexpr int kMaxGroup = 8;
// Page-table entries one decode CTA stages in shared memory; a split covers at
// most this many logical pages.
constexpr int kMaxPagesPerSplit = 2048;
// Upper bound on split-KV partitions.
constexpr int kMaxSplits = 256;

struct DecodeArgs {
  const void *k_pool;
  const void *v_pool;
  const float *k_sz;
  const float *v_sz;
  int32_t num_pages;
  int32_t hkv;
  const void *q;  // bf16 [B][Hq][D]
  int32_t B;
  int32_t hq;
  const int32_t *block_tables;
  int32_t max_pages;
  const int32_t *ctx;
  float scale_log2;  // scale * log2(e)
  float *out;        // final output (S == 1)
  float *o_part;     // partials (S > 1)
  float *lse;        // partial log-sum-exps (S > 1)
  int32_t *counters; // per (sequence, KV head) split-arrival counters (S > 1)
  int32_t S;                // partial slots (= grid splits)
  int32_t S_main;           // splits over the main range; S - S_main is the sink split
  int32_t pages_per_split;
  int32_t tbl_cap;          // table entries staged per CTA (>= pages any split covers)
  int32_t window;           // > 0: attend only the last `window` tokens (+ sinks)
  int32_t sinks;            // attention sinks kept with a window
  int32_t tok_begin;        // first attended token (page aligned); 0 for plain decode
  const float *prior_o;     // [n_prior][B*Hq][D] partials merged into the output
  const float *prior_lse;   // [n_prior][B*Hq]
  int32_t n_prior;
  int32_t keep_partials;    // 1: every split writes its partial (an empty one o = 0,
                            //    lse = -inf) to its slot and nothing is merged
  int32_t tok_end;          // attend tokens below min(ctx, tok_end) only
  int32_t range_mode;       // 1: a context shorter than tok_begin is an empty range,
                            //    not an error
  int32_t *d_err;
  // 1: launched as a programmatic dependent of a kernel whose output this
  // grid does not read (the cascade's prefix pass): only the grid's last CTA
  // waits for it, so the grid still ends after it
  int32_t pdl_defer = 0;
  // 1: blockIdx.z is a launch rank and order[rank] the sequence it serves
  // (longest context first); 2: the same, the units filling several waves of
  // CTAs (the launch may then pick a deeper ring); 0: blockIdx.z is the
  // sequence
  int32_t ordered = 0;
  uint8_t order[kMaxOrdered];
  // fused cache write (pa_decode_append): bf16 [B][Hkv][D] rows of each
  // sequence's newest token, stored at position ctx - 1 before it is read
  const unsigned char *k_new = nullptr;
  const unsigned char *v_new = nullptr;
};

struct PrefixArgs {
  const void *k_pool;
  const void *v_pool;
  int32_t num_pages;
  int32_t hkv;
  const void *q;  // bf16 [B][Hq][D]
  int32_t B;
  int32_t hq;
  const int32_t *prefix_pages;  // [ceil(prefix_len / P)]
  int32_t prefix_len;
  int32_t tiles_per_split;      // 64-token tiles per prefix split
  int32_t n_psplits;
  float scale_log2;
  float *o_pre;    // [n_psplits][B*Hq][D]
  float *lse_pre;  // [n_psplits][B*Hq]
  int32_t *d_err;
  // o_pre as a 5-D tensor [n_psplits][B][Hkv][G][D] fp32, written in boxes of
  // 32 elements x G heads x 128 / G sequences; tma_store = 0 (G does not
  // divide 128, or no encoder) writes it with plain stores instead. Filled in
  // by launch_prefix.
  CUtensorMap tmo;
  int32_t tma_store;
};

cudaError_t launch_prefix(int D, int P, const PrefixArgs &a, bool programmatic,
                          cudaStream_t stream);
int prefix_rows_per_cta();
int prefix_tile_tokens();

cudaError_t launch_decode(int D, int P, int kv_dtype, const DecodeArgs &a,
                          cudaStream_t stream);
// CTAs of the decode kernel for (D, P, kv_dtype) that fit on one SM.
int decode_ctas_per_sm(int D, int P, int kv_dtype);

// Merges, per (sequence, query head) row, the S partials o_part[row][S][D] /
// lse[row][S] and then n_prior more prior_o[p][row][D] / prior_lse[p][row].
cudaError_t launch_splitkv_reduce(const float *o_part, const float *lse, int B,
                                  int hq, int S, int D, float *out,
                                  bool programmatic, cudaStream_t stream,
                                  const float *prior_o = nullptr,
                                  const float *prior_lse = nullptr, int n_prior = 0,
                                  float *lse_out = nullptr, size_t prior_o_stride = 0,
                                  size_t prior_lse_stride = 0);

cudaError_t launch_kv_append(const pa_kv_pool_t &pool, const void *k_new,
                             const void *v_new, const int32_t *seq_idx,
                             const int32_t *pos, int32_t n,
                             const int32_t *block_tables, int32_t num_seqs,
                             int32_t max_pages, int32_t *d_err,
                             cudaStream_t stream);

cudaError_t launch_validate_tables(const int32_t *block_tables, int32_t B,
                                   int32_t max_pages, const int32_t *ctx,
                                   int32_t num_pages, int32_t page_size,
                                   int32_t *d_err, cudaStream_t stream);

int device_sm_count();

}  // namespace pa
