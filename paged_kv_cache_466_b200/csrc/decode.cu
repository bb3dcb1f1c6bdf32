// Paged decode attention (Eq. 1 of "KV-Cache Optimization Techniques",
// section "PagedAttention (vLLM)") for B200 / sm_100a.
//
// One CTA serves one (split, KV head, sequence): it walks that sequence's
// logical pages in [split * pages_per_split, (split + 1) * pages_per_split),
// looks each up in the request's block table, and reads every K/V row of the
// page exactly once for all G query heads that share the KV head (GQA, Eq. 7
// of the same page). The CTA's warps take 16-token blocks round robin; each
// warp keeps its own online-softmax state and the CTA merges its warps at the
// end by their running maxima.
//
// Per 16-token block a warp does, on the tensor cores (mma.sync m16n8k16):
//   S[8 heads x 16 tokens]  = Q[heads x D] . K[tokens x D]^T     (A = Q, B = K)
//   O^T[D x 8 heads]       += V^T[D x tokens] . P^T[tokens x heads]
// The score fragment S lands in exactly the register layout the second product
// needs for its B operand, so P never leaves registers. P is split into a bf16
// (or f16) high part and the residual low part and multiplied twice, which keeps
// ~16 significant bits of every softmax weight.
//
// Data movement: per warp, a ring of NSTAGE 16-token blocks in shared memory.
// The warp copies each block with 16-byte cp.async (L1 bypass, zero-fill past
// the context) such that every copy instruction moves 512 contiguous bytes of
// a page, then waits for its own copies and joins the warp (__syncwarp) before
// the lanes read the block back in mma-fragment order. No CTA barrier, mbarrier
// or spin-wait is involved: cp.async.wait_group on the thread's own copies is
// the only wait, and it always completes.
//
// Fragment order (what each lane reads back), chosen so that the registers are
// mma operands without shuffles:
//   K: lane (g = lane/4, t = lane%4) reads token g of each 8-token half-block,
//      16-byte chunks t, t+4, ... of its row. The contraction index (d) is
//      permuted identically for Q, which is loaded with the same pattern.
//   V: lane reads tokens {2t, 2t+1, 8+2t, 9+2t} (the B-fragment rows of P^T),
//      chunks {g, 8+g} (bf16) or chunk g (uint8); the output rows of O^T are
//      permuted accordingly and un-permuted when stored.
// Rows are stored with their 16-byte chunks XOR-permuted (staged_off) so that
// both read patterns are free of shared-memory bank conflicts.
//
// INT8, FP8 and INT4 caches (Eq. 3, "KV-Cache Quantization"; FP8 = E4M3
// codes with z = 0): with x = s*c + z per row,
//   q.x = s (q.c) + z sum(q)          and    sum_t p_t x_t = sum_t (p_t s_t) c_t + sum_t p_t z_t,
// so the codes go through the tensor cores as exact f16 values (INT8 codes and
// INT4 low nibbles as the subnormals c * 2^-24, INT4 high nibbles in place as
// c * 2^-20, E4M3 codes converted exactly) and the scale and zero are applied
// once per (token, head) instead of once per element.
#include <atomic>
#include <cfloat>
#include <cmath>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_quant.cuh"

// Tile configuration (warps per CTA, pipeline depth per warp, CTAs per SM the
// register allocation must allow); overridable at build time for tuning.
#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_DECODE_STAGES_BF16
#define PA_DECODE_STAGES_BF16 2
#endif
#ifndef PA_DECODE_STAGES_U8
#define PA_DECODE_STAGES_U8 4
#endif
#ifndef PA_DECODE_STAGES_BF16_LPT  // bf16 launched longest unit first (see launch_t)
#define PA_DECODE_STAGES_BF16_LPT 3
#endif
#ifndef PA_DECODE_STAGES_U8_LPT  // INT8 / FP8 launched longest unit first
#define PA_DECODE_STAGES_U8_LPT 6
#endif
#ifndef PA_DECODE_MIN_CTAS
#define PA_DECODE_MIN_CTAS 3
#endif
#ifndef PA_DECODE_MIN_CTAS_U4
#define PA_DECODE_MIN_CTAS_U4 4
#endif
#ifndef PA_DECODE_PDL
#define PA_DECODE_PDL 1
#endif

namespace pa {
namespace {

constexpr float kLn2 = 0.693147180559945309f;
// Lazy rescaling: the running max is only raised when a block's max exceeds it
// by more than this many powers of two, so weights stay <= 2^kRescaleLog2.
// Quantised pools keep the weights <= 2^3, so that the power of two that
// normalises the V weights (below) moves rarely.
template <int KVT>
constexpr float kRescaleLog2 = KVT == PA_KV_BF16 ? 8.0f : 3.0f;

// FP8 pools (E4M3 codes, z = 0) share the INT8 layout.
template <int KVT>
constexpr bool kIsFp8 = KVT == PA_KV_FP8_PER_TOKEN;
// Codes reach the MMA scaled by an exact power of two: an INT8 byte, or an
// INT4 low nibble, under zero high bits is the f16 subnormal c * 2^-24; an
// INT4 high nibble left in place is c * 2^-20; FP8 codes go as they are. The
// K scale and O after the loop take the powers of two back.
template <int KVT>
constexpr float kCodeScale = kIsFp8<KVT> ? 1.f : 16777216.f;

template <int D, int KVT>
struct Tile {
  static_assert(D == 64 || D == 128, "head_dim");
  // INT8 and FP8 pools share the layout: 1-byte codes + (scale, zero) per row
  static constexpr bool kU8 = KVT != PA_KV_BF16;
  static constexpr bool kU4 = KVT == PA_KV_U4_PER_TOKEN;  // two codes per byte
  static constexpr int kElem = kU8 ? 1 : 2;
  static constexpr int kRowBytes = kU4 ? D / 2 : D * kElem;
  // one 16-token block of K (or V) is 16 contiguous rows of the page
  static constexpr int kBlockBytes = 16 * kRowBytes;
  static constexpr int kCopies = kBlockBytes / 512;  // 16-byte copies per lane per tensor
  static constexpr int kSzBytes = kU8 ? 16 * 8 : 0;  // (scale, zero) of 16 rows
  static constexpr int kVOff = kBlockBytes;
  static constexpr int kKSzOff = 2 * kBlockBytes;
  static constexpr int kVSzOff = 2 * kBlockBytes + kSzBytes;
  static constexpr int kStageBytes = 2 * kBlockBytes + 2 * kSzBytes;
  // 16-byte K chunks a lane reads per 8-token half-block (fragment layout)
  static constexpr int kKChunks = kU4 ? 1 : (kU8 ? D / 64 : D / 32);
  // 16-byte V chunks a lane reads per token
  static constexpr int kVChunks = kU8 ? 1 : D / 64;
  static constexpr int kMTiles = D / 16;  // m16 tiles of O^T
  // rows of at least 128 bytes are stored with their 16-byte chunks permuted
  // (chunk ^ swz(row)), which makes both fragment read patterns conflict free
  static constexpr bool kSwizzle = kRowBytes >= 128;
  // INT4 rows (32 or 64 bytes) are permuted instead: rows 2t (and 2t + 1),
  // t = 0..3, which the V fragment reads together, land in distinct bank
  // quarters (D = 64) or halves (D = 128) of a 128-byte line.
  static __device__ __forceinline__ int staged_row(int row) {
    if constexpr (!kU4) return row;
    else if constexpr (D == 128) return row ^ ((row >> 1) & 1);
    else return row ^ ((row >> 2) & 1);
  }
};

// Shared-memory byte offset of 16-byte chunk `chunk` of row `row` in a staged
// block. swz(row) = 2*((row >> 1) & 3) ^ 4*(row & 1) keeps the chunk inside its
// 128-byte group; lanes reading (row g, chunk 4i+t) for K and (row 2t+e, chunk
// g) for V then touch 8 distinct bank groups per quarter warp.
template <class T>
__device__ __forceinline__ int staged_off(int row, int chunk) {
  const int swz = T::kSwizzle ? ((2 * ((row >> 1) & 3)) ^ (4 * (row & 1))) : 0;
  return T::staged_row(row) * T::kRowBytes + ((chunk ^ swz) << 4);
}

template <int D, int KVT, int W, int NSTAGE>
struct Smem {
  using T = Tile<D, KVT>;
  static constexpr int kRingBytesPerWarp = NSTAGE * T::kStageBytes;
  static constexpr int kRingBytes = W * kRingBytesPerWarp;
  // per-warp merge record: m[8], l[8], O[8][D]
  static constexpr int kMergeBytes = (16 + kMaxGroup * D) * 4;
  static_assert(kMergeBytes <= kRingBytesPerWarp, "merge record must fit the ring");
  static constexpr size_t bytes(int pages_per_split) {
    return (size_t)kRingBytes + (size_t)pages_per_split * 4;
  }
};

// Row of O^T held in accumulator c0/c1 (row g) of m-tile j; c2/c3 hold d + 1.
template <int D, int KVT>
__device__ __forceinline__ int out_col(int j, int g) {
  if constexpr (KVT != PA_KV_BF16) {
    return (D == 128 ? 16 * g : 8 * g) + 2 * j;
  } else {
    return 8 * (8 * (j / 4) + g) + 2 * (j % 4);
  }
}

// Final log-sum-exp merge for the G query heads of one (sequence, KV head):
// nl partials of this call's splits (workspace slots 0..nl-1) plus the
// caller's prior partials (e.g. a shared prefix), in that fixed order. Every
// thread of the CTA must call it; `wts` is shared scratch of
// G * (nl + n_prior) floats. Writes out[b][h*G + hd][:].
template <int D>
__device__ void merge_rows(const DecodeArgs &a, int b, int h, int G, int nl, float *wts) {
  const int nw = nl + a.n_prior;
  const size_t R = (size_t)a.B * a.hq;
  for (int i = threadIdx.x; i < G * nw; i += blockDim.x) {
    const int hd = i / nw;
    const int sp = i - hd * nw;
    const size_t row = (size_t)b * a.hq + (size_t)h * G + hd;
    wts[i] = sp < nl ? __ldcg(a.lse + row * a.S + sp)
                     : __ldcg(a.prior_lse + (size_t)(sp - nl) * R + row);
  }
  __syncthreads();
  if ((int)threadIdx.x < G) {
    float *wh = wts + threadIdx.x * nw;
    float M = -INFINITY;
    for (int sp = 0; sp < nw; ++sp) M = fmaxf(M, wh[sp]);
    float den = 0.f;
    for (int sp = 0; sp < nw; ++sp) {
      const float wv = M == -INFINITY ? 0.f : expf(wh[sp] - M);
      wh[sp] = wv;
      den += wv;
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    for (int sp = 0; sp < nw; ++sp) wh[sp] *= inv;
  }
  __syncthreads();
  constexpr int D4 = D / 4;
  for (int i = threadIdx.x; i < G * D4; i += blockDim.x) {
    const int hd = i / D4;
    const int d4 = i - hd * D4;
    const size_t row = (size_t)b * a.hq + (size_t)h * G + hd;
    const float *wh = wts + hd * nw;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 *op = reinterpret_cast<const float4 *>(a.o_part + row * a.S * D) + d4;
#pragma unroll 4
    for (int sp = 0; sp < nl; ++sp) {  // every live split wrote a finite partial
      const float wv = wh[sp];
      const float4 v = __ldcg(op + (size_t)sp * D4);
      acc.x = fmaf(wv, v.x, acc.x);
      acc.y = fmaf(wv, v.y, acc.y);
      acc.z = fmaf(wv, v.z, acc.z);
      acc.w = fmaf(wv, v.w, acc.w);
    }
    for (int sp = 0; sp < a.n_prior; ++sp) {
      const float wv = wh[nl + sp];
      if (wv == 0.f) continue;
      const float4 v = __ldcg(reinterpret_cast<const float4 *>(
                                  a.prior_o + ((size_t)sp * R + row) * D) + d4);
      acc.x = fmaf(wv, v.x, acc.x);
      acc.y = fmaf(wv, v.y, acc.y);
      acc.z = fmaf(wv, v.z, acc.z);
      acc.w = fmaf(wv, v.w, acc.w);
    }
    reinterpret_cast<float4 *>(a.out + row * D)[d4] = acc;
  }
}

// ---- per-block building blocks ---------------------------------------------------

// Query fragments of the head of lane group g (A operand, rows = heads; rows
// 8..15 stay zero). Returns the sum of q as the MMA sees it (quantised pools).
template <int D, int KVT>
__device__ __forceinline__ float load_q(const __nv_bfloat16 *qp, bool head_ok, int t,
                                        uint32_t (&qa)[D / 16][2]) {
  using T = Tile<D, KVT>;
  float qsum = 0.f;        // sum of this head's q (as the MMA sees it), INT8 only
  if constexpr (!T::kU8) {
#pragma unroll
    for (int i = 0; i < T::kKChunks; ++i) {
      uint4 v = head_ok ? ldg_nc128(qp + (4 * i + t) * 8) : make_uint4(0, 0, 0, 0);
      qa[2 * i][0] = v.x;
      qa[2 * i][1] = v.y;
      qa[2 * i + 1][0] = v.z;
      qa[2 * i + 1][1] = v.w;
    }
  } else if constexpr (T::kU4) {
    // lane t contracts d in [t*D/4, (t+1)*D/4); per group of 8 elements the
    // k-steps take (e0,e4 | e2,e6) (low nibbles) and (e1,e5 | e3,e7) (high
    // nibbles), as the 4-bit unpack does
#pragma unroll
    for (int w = 0; w < D / 32; ++w) {
      const uint4 v = head_ok ? ldg_nc128(qp + t * (D / 4) + 8 * w) : make_uint4(0, 0, 0, 0);
      const uint32_t f04 = pack_f16(bf16_lo(v.x), bf16_lo(v.z));
      const uint32_t f26 = pack_f16(bf16_lo(v.y), bf16_lo(v.w));
      const uint32_t f15 = pack_f16(bf16_hi(v.x), bf16_hi(v.z));
      const uint32_t f37 = pack_f16(bf16_hi(v.y), bf16_hi(v.w));
      qsum += (f16_lo(f04) + f16_hi(f04)) + (f16_lo(f26) + f16_hi(f26)) +
              (f16_lo(f15) + f16_hi(f15)) + (f16_lo(f37) + f16_hi(f37));
      qa[2 * w][0] = f04;
      qa[2 * w][1] = f26;
      qa[2 * w + 1][0] = f15;
      qa[2 * w + 1][1] = f37;
    }
    qsum += __shfl_xor_sync(0xffffffffu, qsum, 1);
    qsum += __shfl_xor_sync(0xffffffffu, qsum, 2);
  } else {
#pragma unroll
    for (int i = 0; i < T::kKChunks; ++i) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint4 v = head_ok ? ldg_nc128(qp + (4 * i + t) * 16 + hf * 8) : make_uint4(0, 0, 0, 0);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t f = pack_f16(bf16_lo(w4[k]), bf16_hi(w4[k]));
          qsum += f16_lo(f) + f16_hi(f);
          // words of this 16-d chunk: k-step 4i + (2hf + k/2), half k%2
          qa[4 * i + 2 * hf + k / 2][k % 2] = f;
        }
      }
    }
    qsum += __shfl_xor_sync(0xffffffffu, qsum, 1);
    qsum += __shfl_xor_sync(0xffffffffu, qsum, 2);
  }
  return qsum;
}

// Lane-constant offsets: where each 16-byte copy of a block lands in the stage
// (row and swizzled place), and where the lane reads its K and V fragments.
template <int D, int KVT>
struct LaneMap {
  using T = Tile<D, KVT>;
  int cp_row[T::kCopies], cp_soff[T::kCopies];
  int sz_dst;
  int koff[2][T::kKChunks];
  int voff[4][T::kVChunks];
  __device__ __forceinline__ explicit LaneMap(int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int j = 0; j < T::kCopies; ++j) {
      const int o = j * 512 + lane * 16;
      cp_row[j] = o / T::kRowBytes;
      cp_soff[j] = staged_off<T>(cp_row[j], (o % T::kRowBytes) >> 4);
    }
    sz_dst = (lane < 8 ? T::kKSzOff : T::kVSzOff) + (lane & 7) * 16;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < T::kKChunks; ++i)
        koff[nt][i] = T::kU4 ? T::staged_row(nt * 8 + g) * T::kRowBytes + t * (D / 8)
                             : staged_off<T>(nt * 8 + g, 4 * i + t);
#pragma unroll
    for (int tau = 0; tau < 4; ++tau)
#pragma unroll
      for (int c = 0; c < T::kVChunks; ++c) {
        const int row = (tau & 1) + 2 * t + (tau >> 1) * 8;
        if constexpr (T::kU4) {
          voff[tau][c] = T::kVOff + T::staged_row(row) * T::kRowBytes + g * (D / 16);
        } else {
          const int chunk = T::kU8 ? (D == 128 ? g : (g >> 1)) : 8 * c + g;
          voff[tau][c] = T::kVOff + staged_off<T>(row, chunk);
        }
      }
  }
};

// Issue the copies of one 16-token block: pool rows row0 .. row0 + 15 of K and
// V (and their scale/zero) into the stage at `dst`; rows outside [rlo, rhi)
// are zero-filled instead of read. sz_base is k_sz for lanes 0..7, else v_sz.
template <int D, int KVT>
__device__ __forceinline__ void issue_block(const LaneMap<D, KVT> &lm, uint32_t dst,
                                            const unsigned char *kbase,
                                            const unsigned char *vbase, const float *sz_base,
                                            size_t row0, int rlo, int rhi, int lane) {
  using T = Tile<D, KVT>;
  const unsigned char *ksrc = kbase + row0 * T::kRowBytes + lane * 16;
  const unsigned char *vsrc = vbase + row0 * T::kRowBytes + lane * 16;
  if (rlo == 0 && rhi == 16) {  // warp-uniform: the whole block is read
#pragma unroll
    for (int j = 0; j < T::kCopies; ++j) {
      cp_async16(dst + lm.cp_soff[j], ksrc + j * 512, 16u);
      cp_async16(dst + T::kVOff + lm.cp_soff[j], vsrc + j * 512, 16u);
    }
    if constexpr (T::kU8) {
      // lanes 0..7: K (scale, zero) of rows 2l, 2l+1; lanes 8..15: V
      if (lane < 16) cp_async16(dst + lm.sz_dst, sz_base + (row0 + 2 * (lane & 7)) * 2, 16u);
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < T::kCopies; ++j) {
    const uint32_t n = (lm.cp_row[j] >= rlo && lm.cp_row[j] < rhi) ? 16u : 0u;
    cp_async16(dst + lm.cp_soff[j], ksrc + j * 512, n);
    cp_async16(dst + T::kVOff + lm.cp_soff[j], vsrc + j * 512, n);
  }
  if constexpr (T::kU8) {
    if (lane < 16) {
      // (a row outside [rlo, rhi) may come along with its neighbour; the
      // consumer zeroes scale and zero of every masked token)
      const int l = lane & 7;
      const bool any = 2 * l + 1 >= rlo && 2 * l < rhi;
      cp_async16(dst + lm.sz_dst, sz_base + (row0 + 2 * l) * 2, any ? 16u : 0u);
    }
  }
}

// ---- bf16 pools ---------------------------------------------------------------
//
// One warp's online-softmax state for the G heads of a (sequence, KV head).
template <int D>
struct WarpAcc {
  float o[D / 16][4];
  float m_run;  // running max of this head's scores (log2 units)
  float l_run;  // this lane's share of the softmax denominator
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int j = 0; j < D / 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    m_run = -INFINITY;
    l_run = 0.f;
  }
};

// Scores, online softmax and O^T update for the 16-token bf16 block staged at
// `src`, whose first token is btok; tokens outside [tok_lo, tok1) and all
// tokens of an invalid page (pvalid false) are masked.
template <int D>
__device__ __forceinline__ void block_step(const LaneMap<D, PA_KV_BF16> &lm, uint32_t src,
                                           int btok, int tok_lo, int tok1, bool pvalid,
                                           float scale_log2, const uint32_t (&qa)[D / 16][2],
                                           int t, WarpAcc<D> &acc) {
  using T = Tile<D, PA_KV_BF16>;
  float(&o)[T::kMTiles][4] = acc.o;
  float &m_run = acc.m_run;
  float &l_run = acc.l_run;
  const auto &koff = lm.koff;
  const auto &voff = lm.voff;
  // ---- S = Q K^T -------------------------------------------------------------
  float s[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int i = 0; i < T::kKChunks; ++i) {
      const uint4 kv = lds128(src + koff[nt][i]);
      mma_bf16_16816(s[nt], qa[2 * i][0], 0u, qa[2 * i][1], 0u, kv.x, kv.y);
      mma_bf16_16816(s[nt], qa[2 * i + 1][0], 0u, qa[2 * i + 1][1], 0u, kv.z, kv.w);
    }
  }

  // ---- online softmax (log2 domain) ---------------------------------------
  float x[4] = {s[0][0], s[0][1], s[1][0], s[1][1]};  // tokens 2t, 2t+1, 8+2t, 9+2t
  if (pvalid && btok >= tok_lo && btok + 16 <= tok1) {  // warp-uniform: no mask needed
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] *= scale_log2;
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = btok + (e & 1) + 2 * t + (e >> 1) * 8;
      const bool ok = pvalid && tok >= tok_lo && tok < tok1;
      x[e] = ok ? x[e] * scale_log2 : -INFINITY;
    }
  }
  float mb = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
  mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
  mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
  const bool need = mb > m_run + kRescaleLog2<PA_KV_BF16> || (m_run == -INFINITY && mb > -INFINITY);
  if (__any_sync(0xffffffffu, need)) {
    const float m_new = fmaxf(m_run, mb);
    const float alpha = m_new == -INFINITY ? 1.f : fast_exp2(m_run - m_new);
    m_run = m_new;
    l_run *= alpha;
    const float al0 = __shfl_sync(0xffffffffu, alpha, 8 * t);      // head 2t
    const float al1 = __shfl_sync(0xffffffffu, alpha, 8 * t + 4);  // head 2t+1
#pragma unroll
    for (int j = 0; j < T::kMTiles; ++j) {
      o[j][0] *= al0;
      o[j][1] *= al1;
      o[j][2] *= al0;
      o[j][3] *= al1;
    }
  }
  const float mref = m_run == -INFINITY ? 0.f : m_run;
  float p[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) p[e] = fast_exp2(x[e] - mref);
  l_run += (p[0] + p[1]) + (p[2] + p[3]);

  // ---- O^T += V^T P^T -------------------------------------------------------
  uint32_t bh0, bl0, bh1, bl1;
  split_bf16(p[0], p[1], bh0, bl0);
  split_bf16(p[2], p[3], bh1, bl1);
#pragma unroll
  for (int c = 0; c < T::kVChunks; ++c) {
    const uint4 v0 = lds128(src + voff[0][c]);
    const uint4 v1 = lds128(src + voff[1][c]);
    const uint4 v2 = lds128(src + voff[2][c]);
    const uint4 v3 = lds128(src + voff[3][c]);
    const uint32_t x0[4] = {v0.x, v0.y, v0.z, v0.w};
    const uint32_t x1[4] = {v1.x, v1.y, v1.z, v1.w};
    const uint32_t x2[4] = {v2.x, v2.y, v2.z, v2.w};
    const uint32_t x3[4] = {v3.x, v3.y, v3.z, v3.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t a0 = __byte_perm(x0[w], x1[w], 0x5410);
      const uint32_t a1 = __byte_perm(x0[w], x1[w], 0x7632);
      const uint32_t a2 = __byte_perm(x2[w], x3[w], 0x5410);
      const uint32_t a3 = __byte_perm(x2[w], x3[w], 0x7632);
      mma_bf16_16816(o[4 * c + w], a0, a1, a2, a3, bh0, bh1);
      mma_bf16_16816(o[4 * c + w], a0, a1, a2, a3, bl0, bl1);
    }
  }
}

// ---- quantised pools (INT8, FP8, INT4): tokens as the MMA's M dimension ---------
//
// A warp step covers two 16-token blocks (32 tokens), and per block
//   S^T[16 tokens x 8 heads]  = K[tokens x D] . Q^T[D x heads]      (A = K, B = Q)
//   O^T[D x 8 heads]         += V^T[D x tokens] . P^T[tokens x heads]
// With the tokens as M every row of the score MMA is a real token (with the
// heads as M, rows 8..15 would be zero): half the score MMAs of a head-major
// product. The lane then holds the scores of tokens g and g + 8 for heads 2t
// and 2t + 1, the same two heads whose columns of O^T it accumulates, so the
// online-softmax state of those heads lives in the lane and the rescale of O
// needs no shuffle; P^T, the B operand of the second product, is the score
// fragment transposed, which movmatrix does in registers. The K fragments
// (A operand) are the registers the head-major B operand used, so the staging,
// its swizzle and the code unpack are shared with the bf16 path.
//
// The V weights p_t * s_t (s_t the row scale of Eq. 3) enter the f16 MMA
// scaled by a power of two 2^-E kept like the running max: the softmax keeps
// every p_t <= 2^kRescaleLog2, so the largest V scale seen so far bounds every
// weight, and E is set from the first nonzero scale so that this bound sits
// at 2^12 .. 2^13, and raised whenever a larger scale arrives, O then being
// multiplied by the exact power of two. O is thus carried in units of 2^E
// (fp32) and the weights stay inside the f16 range whatever the row scales
// are: no limit on the scale from the f16 range.
constexpr float kWeightHi = 16384.f;  // largest scaled V weight fed to the MMA (2^14)
// the largest scaled V scale: weights p s with p <= 2^kRescaleLog2 stay below kWeightHi
template <int KVT>
constexpr float kScaleHi = kWeightHi / (1 << (int)kRescaleLog2<KVT>);
constexpr int kWeightTopExp = 12;     // a new E puts the largest weight at 2^12 .. 2^13
constexpr int kEMin = -120, kEMax = 120;

// 2^n as a float for -126 <= n <= 127; 0 below.
__device__ __forceinline__ float exp2i(int n) {
  return n < -126 ? 0.f : __uint_as_float(static_cast<uint32_t>(n + 127) << 23);
}
// floor(log2(x)) of a positive normal float (subnormals give -127).
__device__ __forceinline__ int ilog2f(float x) {
  return static_cast<int>((__float_as_uint(x) >> 23) & 0xffu) - 127;
}

template <int D>
struct QAcc {
  float o[D / 16][4];
  float m[2];  // running max of the scores of heads 2t, 2t + 1 (log2 units)
  float l[2];  // this lane's share of their softmax denominators
  float z[2];  // this lane's share of sum_t p_t z_t
  float f;     // 2^-E; 0 until the first nonzero V scale
  int e;       // E
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int j = 0; j < D / 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      m[h] = -INFINITY;
      l[h] = z[h] = 0.f;
    }
    f = 0.f;
    e = 0;
  }
};

// S^T of the 16-token quantised block staged at `src` (codes times the
// Tile's power of two): s[0], s[1] = token g, heads 2t, 2t + 1; s[2], s[3] =
// token g + 8.
template <int D, int KVT>
__device__ __forceinline__ void scores_t(const LaneMap<D, KVT> &lm, uint32_t src,
                                         const uint32_t (&qa)[D / 16][2], float (&s)[4]) {
  using T = Tile<D, KVT>;
  s[0] = s[1] = s[2] = s[3] = 0.f;
  if constexpr (T::kU4) {
    // rows g and g + 8; per word (e2i in the low nibble of byte i) the low
    // nibbles under zero bits are the f16 subnormals c * 2^-24 (pairs e0, e4
    // and e2, e6), the high nibbles in place c * 2^-20 (pairs e1, e5 and e3, e7)
    float sh[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t r0[D / 32], r1[D / 32];
    if constexpr (D == 128) {
      const uint4 a = lds128(src + lm.koff[0][0]);
      const uint4 b = lds128(src + lm.koff[1][0]);
      r0[0] = a.x; r0[1] = a.y; r0[2] = a.z; r0[3] = a.w;
      r1[0] = b.x; r1[1] = b.y; r1[2] = b.z; r1[3] = b.w;
    } else {
      const uint2 a = lds64(src + lm.koff[0][0]);
      const uint2 b = lds64(src + lm.koff[1][0]);
      r0[0] = a.x; r0[1] = a.y;
      r1[0] = b.x; r1[1] = b.y;
    }
#pragma unroll
    for (int w = 0; w < D / 32; ++w) {
      const uint32_t u0 = r0[w] >> 8, u1 = r1[w] >> 8;
      mma_f16_16816(s, r0[w] & 0x000F000Fu, r1[w] & 0x000F000Fu, u0 & 0x000F000Fu,
                    u1 & 0x000F000Fu, qa[2 * w][0], qa[2 * w][1]);
      mma_f16_16816(sh, r0[w] & 0x00F000F0u, r1[w] & 0x00F000F0u, u0 & 0x00F000F0u,
                    u1 & 0x00F000F0u, qa[2 * w + 1][0], qa[2 * w + 1][1]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) s[e] = fmaf(sh[e], 0.0625f, s[e]);  // high nibbles: 16x
  } else {
    // two accumulators halve the dependent MMA chain
    float s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < T::kKChunks; ++i) {
      const uint4 k0 = lds128(src + lm.koff[0][i]);  // token g
      const uint4 k1 = lds128(src + lm.koff[1][i]);  // token g + 8
      const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w};
      const uint32_t w1[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t a0 = kIsFp8<KVT> ? e4m3x2_to_f16x2(w0[w]) : u8x2_to_f16x2(w0[w], 0x4140);
        const uint32_t a1 = kIsFp8<KVT> ? e4m3x2_to_f16x2(w1[w]) : u8x2_to_f16x2(w1[w], 0x4140);
        const uint32_t a2 =
            kIsFp8<KVT> ? e4m3x2_hi_to_f16x2(w0[w]) : u8x2_to_f16x2(w0[w], 0x4342);
        const uint32_t a3 =
            kIsFp8<KVT> ? e4m3x2_hi_to_f16x2(w1[w]) : u8x2_to_f16x2(w1[w], 0x4342);
        mma_f16_16816((w & 1) ? s2 : s, a0, a1, a2, a3, qa[4 * i + w][0], qa[4 * i + w][1]);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) s[e] += s2[e];
  }
}

// O^T += V^T W^T for the quantised block staged at `src`, with the weights'
// B fragments (hi and lo halves, tokens 0..7 in b?0 and 8..15 in b?1).
template <int D, int KVT, bool kTwo = true>
__device__ __forceinline__ void pv_quant(const LaneMap<D, KVT> &lm, uint32_t src, int g,
                                         uint32_t bh0, uint32_t bh1, uint32_t bl0,
                                         uint32_t bl1, float (&o)[D / 16][4]) {
  using T = Tile<D, KVT>;
  const auto &voff = lm.voff;
  if constexpr (T::kU4) {
    // byte j of this lane's slice holds d = base + 2j (low nibble) and + 1
    uint32_t xv[4][D / 64];
#pragma unroll
    for (int tau = 0; tau < 4; ++tau) {
      if constexpr (D == 128) {
        const uint2 v = lds64(src + voff[tau][0]);
        xv[tau][0] = v.x;
        xv[tau][1] = v.y;
      } else {
        xv[tau][0] = lds32(src + voff[tau][0]);
      }
    }
    // m-tiles j, j+1 use bytes j & 3, (j & 3) + 1 of word j / 4: gather them
    // per token pair as (token 2t: byte b, b + 1 | token 2t + 1: byte b,
    // b + 1), so that each 16-bit half holds one token's bytes; low nibbles
    // under zero bits (c * 2^-24) give rows d (a0, a2), high nibbles in
    // place (c * 2^-20) rows d + 1 (a1, a3)
#pragma unroll
    for (int j = 0; j < T::kMTiles; j += 2) {
      const uint32_t sel = (j & 2) ? 0x7632 : 0x5410;
      const uint32_t ya = __byte_perm(xv[0][j / 4], xv[1][j / 4], sel);
      const uint32_t yb = __byte_perm(xv[2][j / 4], xv[3][j / 4], sel);
      const uint32_t ya8 = ya >> 8, yb8 = yb >> 8;
      const uint32_t a0[2] = {ya & 0x000F000Fu, ya8 & 0x000F000Fu};
      const uint32_t a1[2] = {ya & 0x00F000F0u, ya8 & 0x00F000F0u};
      const uint32_t a2[2] = {yb & 0x000F000Fu, yb8 & 0x000F000Fu};
      const uint32_t a3[2] = {yb & 0x00F000F0u, yb8 & 0x00F000F0u};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        mma_f16_16816(o[j + u], a0[u], a1[u], a2[u], a3[u], bh0, bh1);
        if constexpr (kTwo) mma_f16_16816(o[j + u], a0[u], a1[u], a2[u], a3[u], bl0, bl1);
      }
    }
  } else {
    const uint4 v0 = lds128(src + voff[0][0]);
    const uint4 v1 = lds128(src + voff[1][0]);
    const uint4 v2 = lds128(src + voff[2][0]);
    const uint4 v3 = lds128(src + voff[3][0]);
    const uint32_t x0[4] = {v0.x, v0.y, v0.z, v0.w};
    const uint32_t x1[4] = {v1.x, v1.y, v1.z, v1.w};
    const uint32_t x2[4] = {v2.x, v2.y, v2.z, v2.w};
    const uint32_t x3[4] = {v3.x, v3.y, v3.z, v3.w};
#pragma unroll
    for (int j = 0; j < T::kMTiles; ++j) {
      const uint32_t sel = (j & 1) ? 0x7362 : 0x5140;
      // select with a runtime word offset only for D == 64
      const uint32_t w0 = D == 128 ? x0[j / 2] : ((g & 1) ? x0[2 + j / 2] : x0[j / 2]);
      const uint32_t w1 = D == 128 ? x1[j / 2] : ((g & 1) ? x1[2 + j / 2] : x1[j / 2]);
      const uint32_t w2 = D == 128 ? x2[j / 2] : ((g & 1) ? x2[2 + j / 2] : x2[j / 2]);
      const uint32_t w3 = D == 128 ? x3[j / 2] : ((g & 1) ? x3[2 + j / 2] : x3[j / 2]);
      const uint32_t xa = __byte_perm(w0, w1, sel);
      const uint32_t xb = __byte_perm(w2, w3, sel);
      const uint32_t a0 = kIsFp8<KVT> ? e4m3x2_to_f16x2(xa) : u8x2_to_f16x2(xa, 0x4140);
      const uint32_t a1 = kIsFp8<KVT> ? e4m3x2_hi_to_f16x2(xa) : u8x2_to_f16x2(xa, 0x4342);
      const uint32_t a2 = kIsFp8<KVT> ? e4m3x2_to_f16x2(xb) : u8x2_to_f16x2(xb, 0x4140);
      const uint32_t a3 = kIsFp8<KVT> ? e4m3x2_hi_to_f16x2(xb) : u8x2_to_f16x2(xb, 0x4342);
      mma_f16_16816(o[j], a0, a1, a2, a3, bh0, bh1);
      if constexpr (kTwo) mma_f16_16816(o[j], a0, a1, a2, a3, bl0, bl1);
    }
  }
}

// One warp step over two quantised 16-token blocks staged at src and src +
// one block (first tokens btok[0], btok[1]; pvalid false = invalid page or no
// block). kscale = the Tile's code scale times scale * log2(e); qz = the sums
// of q of heads 2t, 2t + 1 times scale * log2(e).
template <int D, int KVT, bool kPack>
__device__ __forceinline__ void pair_step(const LaneMap<D, KVT> &lm, uint32_t src,
                                          const int (&btok)[2], const bool (&pvalid)[2],
                                          int tok_lo, int tok1, float kscale,
                                          const float (&qz)[2],
                                          const uint32_t (&qa)[D / 16][2], int g, int t,
                                          QAcc<D> &acc) {
  using T = Tile<D, KVT>;
  float x[2][4];           // [block][token g: heads 2t, 2t+1 | token g + 8: same]
  float vs[2][2], vz[2][2];  // [block][token g | g + 8]
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const uint32_t sb = src + u * T::kStageBytes;
    float s[4];
    scores_t<D, KVT>(lm, sb, qa, s);
    const uint2 k0 = lds64(sb + T::kKSzOff + 8 * g);
    const uint2 k1 = lds64(sb + T::kKSzOff + 8 * (g + 8));
    const uint2 v0 = lds64(sb + T::kVSzOff + 8 * g);
    const uint2 v1 = lds64(sb + T::kVSzOff + 8 * (g + 8));
    // q.x = s (q.c) + z sum(q), per token
    const float ka = __uint_as_float(k0.x) * kscale, kb = __uint_as_float(k1.x) * kscale;
    const float za = __uint_as_float(k0.y), zb = __uint_as_float(k1.y);
    x[u][0] = fmaf(ka, s[0], za * qz[0]);
    x[u][1] = fmaf(ka, s[1], za * qz[1]);
    x[u][2] = fmaf(kb, s[2], zb * qz[0]);
    x[u][3] = fmaf(kb, s[3], zb * qz[1]);
    vs[u][0] = __uint_as_float(v0.x);
    vz[u][0] = __uint_as_float(v0.y);
    vs[u][1] = __uint_as_float(v1.x);
    vz[u][1] = __uint_as_float(v1.y);
    if (!(pvalid[u] && btok[u] >= tok_lo && btok[u] + 16 <= tok1)) {  // warp-uniform
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int tok = btok[u] + g + 8 * r;
        if (!(pvalid[u] && tok >= tok_lo && tok < tok1)) {
          x[u][2 * r] = x[u][2 * r + 1] = -INFINITY;
          vs[u][r] = vz[u][r] = 0.f;
        }
      }
    }
  }

  // ---- online softmax of heads 2t, 2t + 1 over the 32 tokens ----------------
  float mb[2] = {fmaxf(fmaxf(x[0][0], x[0][2]), fmaxf(x[1][0], x[1][2])),
                 fmaxf(fmaxf(x[0][1], x[0][3]), fmaxf(x[1][1], x[1][3]))};
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mb[0] = fmaxf(mb[0], __shfl_xor_sync(0xffffffffu, mb[0], off));
    mb[1] = fmaxf(mb[1], __shfl_xor_sync(0xffffffffu, mb[1], off));
  }
  bool need = false;
#pragma unroll
  for (int h = 0; h < 2; ++h)
    need |= mb[h] > acc.m[h] + kRescaleLog2<KVT> || (acc.m[h] == -INFINITY && mb[h] > -INFINITY);
  if (__any_sync(0xffffffffu, need)) {
    float al[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float m_new = fmaxf(acc.m[h], mb[h]);
      al[h] = m_new == -INFINITY ? 1.f : fast_exp2(acc.m[h] - m_new);
      acc.m[h] = m_new;
      acc.l[h] *= al[h];
      acc.z[h] *= al[h];
    }
    if constexpr (kPack) {
      // O^T columns 2t, 2t + 1 of lanes t >= 2 hold the low halves of heads
      // 2t - 4, 2t - 3, whose factors lanes t - 2 hold
      const float x0 = __shfl_xor_sync(0xffffffffu, al[0], 2);
      const float x1 = __shfl_xor_sync(0xffffffffu, al[1], 2);
      if (t >= 2) {
        al[0] = x0;
        al[1] = x1;
      }
    }
#pragma unroll
    for (int j = 0; j < T::kMTiles; ++j) {
      acc.o[j][0] *= al[0];
      acc.o[j][1] *= al[1];
      acc.o[j][2] *= al[0];
      acc.o[j][3] *= al[1];
    }
  }
  const float mr[2] = {acc.m[0] == -INFINITY ? 0.f : acc.m[0],
                       acc.m[1] == -INFINITY ? 0.f : acc.m[1]};
  float p[2][4];  // softmax weights
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int e = 0; e < 4; ++e) p[u][e] = fast_exp2(x[u][e] - mr[e & 1]);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    acc.l[h] += (p[0][h] + p[0][2 + h]) + (p[1][h] + p[1][2 + h]);
    acc.z[h] += fmaf(p[0][h], vz[0][0], p[0][2 + h] * vz[0][1]) +
                fmaf(p[1][h], vz[1][0], p[1][2 + h] * vz[1][1]);
  }

  // ---- the weights' power of two -------------------------------------------
  // A weight is p s with p <= 2^kRescaleLog2, so the largest V scale seen so
  // far bounds every weight: E keeps that scale times 2^kRescaleLog2 at
  // 2^12 .. 2^13 (one E for the warp; it only moves when a larger scale comes)
  float vm = fmaxf(fmaxf(vs[0][0], vs[0][1]), fmaxf(vs[1][0], vs[1][1]));
  const bool big = vm * acc.f > kScaleHi<KVT> || (acc.f == 0.f && vm > 0.f);
  if (__any_sync(0xffffffffu, big)) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, off));
    if (vm > 0.f) {
      const int en = min(max(ilog2f(vm) + (int)kRescaleLog2<KVT> - kWeightTopExp, kEMin), kEMax);
      if (acc.f == 0.f || en > acc.e) {
        // with no weight so far O = 0: nothing to rescale
        const float sc = acc.f == 0.f ? 1.f : exp2i(acc.e - en);
        acc.e = en;
        acc.f = exp2i(-en);
#pragma unroll
        for (int j = 0; j < T::kMTiles; ++j) {
          acc.o[j][0] *= sc;
          acc.o[j][1] *= sc;
          acc.o[j][2] *= sc;
          acc.o[j][3] *= sc;
        }
      }
    }
  }
  float vf[2][2];  // V scales times 2^-E
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    vf[u][0] = vs[u][0] * acc.f;
    vf[u][1] = vs[u][1] * acc.f;
  }

  // ---- O^T += V^T W^T, W^T = the scaled weights transposed -------------------
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    uint32_t h0, l0, h1, l1;
    split_f16(p[u][0] * vf[u][0], p[u][1] * vf[u][0], h0, l0);  // token g
    split_f16(p[u][2] * vf[u][1], p[u][3] * vf[u][1], h1, l1);  // token g + 8
    if constexpr (kPack) {
      // at most four live heads: columns 0..3 of W^T take the high halves of
      // heads 0..3, columns 4..7 their low halves (lanes t >= 2 take them from
      // lanes t - 2), and one MMA per m-tile does both
      const uint32_t x0 = __shfl_xor_sync(0xffffffffu, l0, 2);
      const uint32_t x1 = __shfl_xor_sync(0xffffffffu, l1, 2);
      pv_quant<D, KVT, false>(lm, src + u * T::kStageBytes, g,
                              movmatrix_trans(t < 2 ? h0 : x0),
                              movmatrix_trans(t < 2 ? h1 : x1), 0u, 0u, acc.o);
    } else {
      pv_quant<D, KVT>(lm, src + u * T::kStageBytes, g, movmatrix_trans(h0),
                       movmatrix_trans(h1), movmatrix_trans(l0), movmatrix_trans(l1), acc.o);
    }
  }
}

// Fused cache write: store the K/V row of KV head h of sequence b's newest
// token (bf16 k_new / v_new [B][Hkv][D]) into pool row `row`, as pa_kv_append
// does (quantised pools through the same per-row quantisers, so the stored
// bits are identical). Called by every thread of the CTA.
template <int D, int KVT>
__device__ __forceinline__ void append_new_row(const DecodeArgs &a, int b, int h, size_t row) {
  const size_t src = ((size_t)b * a.hkv + h) * D * 2;  // bytes
  unsigned char *kp = static_cast<unsigned char *>(const_cast<void *>(a.k_pool));
  unsigned char *vp = static_cast<unsigned char *>(const_cast<void *>(a.v_pool));
  if constexpr (KVT == PA_KV_BF16) {
    for (int c = threadIdx.x; c < D / 8; c += blockDim.x) {
      *reinterpret_cast<uint4 *>(kp + row * D * 2 + c * 16) = ldg_nc128(a.k_new + src + c * 16);
      *reinterpret_cast<uint4 *>(vp + row * D * 2 + c * 16) = ldg_nc128(a.v_new + src + c * 16);
    }
  } else {
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      float *ksz = const_cast<float *>(a.k_sz) + row * 2;
      float *vsz = const_cast<float *>(a.v_sz) + row * 2;
      if constexpr (KVT == PA_KV_U4_PER_TOKEN) {
        quantise_row_u4<D>(a.k_new + src, kp + row * (D / 2), ksz, lane);
        quantise_row_u4<D>(a.v_new + src, vp + row * (D / 2), vsz, lane);
      } else if constexpr (KVT == PA_KV_FP8_PER_TOKEN) {
        quantise_row_fp8<D>(a.k_new + src, kp + row * D, ksz, lane);
        quantise_row_fp8<D>(a.v_new + src, vp + row * D, vsz, lane);
      } else {
        quantise_row<D>(a.k_new + src, kp + row * D, ksz, lane);
        quantise_row<D>(a.v_new + src, vp + row * D, vsz, lane);
      }
    }
  }
}

// CTAs per SM the register allocation must allow. An INT4 CTA's ring (two
// pair stages of 2.3 KB blocks per warp, 37 KB) leaves room for a fourth CTA,
// which 128 registers allow (12 bytes of spill); measured on the ragged
// Llama-3-8B-shaped INT4 step: 63.8 -> 60.6 us at S = 4.
template <int KVT>
constexpr int kMinCtas = KVT == PA_KV_U4_PER_TOKEN ? PA_DECODE_MIN_CTAS_U4 : PA_DECODE_MIN_CTAS;

template <int D, int P, int KVT, int W, int NSTAGE>
__global__ void __launch_bounds__(W * 32, kMinCtas<KVT>) decode_kernel(const DecodeArgs a) {
  using T = Tile<D, KVT>;
  using SM = Smem<D, KVT, W, NSTAGE>;
  static_assert(P % 16 == 0, "a 16-token block must not straddle pages");
  extern __shared__ __align__(128) unsigned char smem[];

  // Launched as a programmatic dependent: wait until the previous kernel on
  // the stream (e.g. the cache write) has finished and its writes are visible.
  // Behind the cascade's prefix pass, which releases its dependents only after
  // its own wait for the work before it, nothing this grid reads is still
  // being written: one CTA (the last launched) waits, so that a kernel after
  // this grid also finds the prefix pass finished.
  if (!a.pdl_defer || (blockIdx.x == gridDim.x - 1 && blockIdx.y == gridDim.y - 1 &&
                       blockIdx.z == gridDim.z - 1))
    pdl_wait_primary();

  const int split = blockIdx.x;
  const int h = blockIdx.y;
  const int b = a.ordered ? (int)a.order[blockIdx.z] : (int)blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int G = a.hq / a.hkv;

  int *tbl = reinterpret_cast<int *>(smem + SM::kRingBytes);

  // ---- this split's token range --------------------------------------------
  // Token ranges. The main range [mlo, ctx) is split over the first S_main
  // splits: mlo = tok_begin (page aligned; > 0 when the caller supplies the
  // shared-prefix part as prior partials) or, with a window, the start of the
  // last `window` tokens. With attention sinks, split 0 also covers
  // [0, min(sinks, ctx)) ("Token Eviction Strategies", Eq. 5) as a second
  // range processed before its main one; the two ranges are disjoint and
  // together hold exactly the kept tokens.
  // Loads that do not depend on the context length go out with it: the
  // query fragments and, where the split's page range does not depend on the
  // context (no window, a main split), that range's table entries.
  int ctx = a.ctx[b];
  constexpr int kPre = 2;  // table entries prefetched per thread
  int pre[kPre];
  const bool nominal = a.window == 0 && split < a.S_main;
  {
    const int lp0n = a.tok_begin / P + split * a.pages_per_split;
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
      const int i = threadIdx.x + k * W * 32;
      pre[k] = (nominal && i < a.pages_per_split && lp0n + i < a.max_pages)
                   ? __ldg(a.block_tables + (size_t)b * a.max_pages + lp0n + i)
                   : -1;
    }
  }
  const bool head_ok = g < G;
  const size_t q_row = ((size_t)b * a.hq + (size_t)h * G + (head_ok ? g : 0)) * D;
  const __nv_bfloat16 *qp = reinterpret_cast<const __nv_bfloat16 *>(a.q) + q_row;
  uint32_t qa[D / 16][2];  // per k-step: a0 (k 2t..2t+1), a2 (k 2t+8..2t+9)
  const float qsum = load_q<D, KVT>(qp, head_ok, t, qa);

  if (ctx < 0 || ctx > a.max_pages * P) {
    if (threadIdx.x == 0) flag_error(a.d_err, PA_DERR_BAD_CTX);
    ctx = a.tok_begin;
  } else if (ctx < a.tok_begin) {
    if (threadIdx.x == 0 && !a.range_mode) flag_error(a.d_err, PA_DERR_BAD_CTX);
    ctx = a.tok_begin;
  }
  ctx = min(ctx, max(a.tok_end, a.tok_begin));
  int mlo = a.tok_begin;
  int sink_hi = 0;
  if (a.window > 0) {
    sink_hi = min(a.sinks, ctx);
    mlo = max(max(ctx - a.window, 0), sink_hi);
  }
  const int n_pages = (ctx + P - 1) / P;
  const int lpb = mlo / P;
  const int n_main_live = ctx > mlo ? (n_pages - lpb + a.pages_per_split - 1) / a.pages_per_split : 0;
  // splits holding tokens (split 0 holds the sinks even when the main range is empty)
  const int n_live = n_main_live > 0 ? n_main_live : (sink_hi > 0 ? 1 : 0);
  const int slot = split;
  // split 0's sink range: pages [0, nsp) staged first, blocks [0, nsb) of it
  const int nsp = split == 0 ? (sink_hi + P - 1) / P : 0;
  const int nsb = split == 0 ? (sink_hi + 15) / 16 : 0;
  int lp0 = lpb + split * a.pages_per_split;
  int lp1 = max(min(lp0 + a.pages_per_split, n_pages), lp0);
  int tok_lo = max(lp0 * P, mlo);
  int tok_hi = min(lp1 * P, ctx);
  if (nsp + (lp1 - lp0) > a.tbl_cap) {
    // Cannot happen with the host's plan (the table slot holds tbl_cap pages);
    // kept so that no table read or write can leave the staged slot.
    if (threadIdx.x == 0) flag_error(a.d_err, PA_DERR_BAD_CTX);
    lp1 = lp0 + max(a.tbl_cap - nsp, 0);
    tok_hi = min(tok_hi, lp1 * P);
  }
  const int blk0 = tok_lo & ~15;  // blocks stay 16-aligned inside their page
  const int nblk = tok_hi > tok_lo ? (tok_hi - blk0 + 15) / 16 : 0;
  const int tok0 = blk0;
  const int tok1 = tok_hi;

  if (nblk == 0 && nsb == 0) {
    if (a.keep_partials) {  // an empty partial: o = 0, lse = -inf (weight 0)
      for (int e = threadIdx.x; e < G * D; e += W * 32) {
        const size_t row = (size_t)b * a.hq + (size_t)h * G + e / D;
        a.o_part[(row * a.S + slot) * D + e % D] = 0.f;
        if (e % D == 0) a.lse[row * a.S + slot] = -INFINITY;
      }
      return;
    }
    if (split == 0 && n_live == 0) {
      if (a.n_prior > 0) {  // nothing of our own: the output is the priors' merge
        merge_rows<D>(a, b, h, G, 0, reinterpret_cast<float *>(smem));
      } else {  // empty context: the output is 0
        for (int e = threadIdx.x; e < G * D; e += W * 32)
          a.out[((size_t)b * a.hq + (size_t)h * G) * D + e] = 0.f;
      }
    }
    return;
  }

  // ---- stage this split's block-table entries (bounds-checked) --------------
  if (nominal && lp1 - lp0 <= kPre * W * 32) {  // CTA-uniform: the prefetch covers them
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
      const int i = threadIdx.x + k * W * 32;
      if (i < lp1 - lp0) {
        int pg = pre[k];
        if (pg < 0 || pg >= a.num_pages) {
          flag_error(a.d_err, PA_DERR_BAD_PAGE);
          pg = -1;
        }
        tbl[i] = pg;
      }
    }
  } else {
    // entries [0, nsp): the sink pages; then the main range's pages
    for (int i = threadIdx.x; i < nsp + lp1 - lp0; i += W * 32) {
      const int lp = i < nsp ? i : lp0 + i - nsp;
      int pg = __ldg(a.block_tables + (size_t)b * a.max_pages + lp);
      if (pg < 0 || pg >= a.num_pages) {
        flag_error(a.d_err, PA_DERR_BAD_PAGE);
        pg = -1;
      }
      tbl[i] = pg;
    }
  }
  __syncthreads();  // tbl visible

  // ---- fused cache write: the split whose pages hold the newest token
  // (position ctx - 1) stores its row before any of the page is read
  if (a.k_new != nullptr && ctx > 0 && split < a.S_main) {
    const int lp_new = (ctx - 1) / P;
    if (lp_new >= lp0 && lp_new < lp1) {  // CTA-uniform
      const int page = tbl[nsp + lp_new - lp0];
      if (page >= 0)
        append_new_row<D, KVT>(a, b, h, ((size_t)page * a.hkv + h) * P + (ctx - 1) % P);
      __syncthreads();  // the row is stored before the page is copied in
    }
  }

  // ---- per-warp pipeline ---------------------------------------------------------
  // Each lane copies 16-byte pieces of a block so that every copy instruction
  // of the warp moves 512 contiguous bytes; after the wait, lanes read the
  // pieces in mma-fragment order (cross-lane, hence the __syncwarp).
  const uint32_t ring = smem_u32(smem) + warp * SM::kRingBytesPerWarp;
  const unsigned char *kbase = static_cast<const unsigned char *>(a.k_pool);
  const unsigned char *vbase = static_cast<const unsigned char *>(a.v_pool);
  const LaneMap<D, KVT> lm(lane);
  const float *sz_base = lane < 8 ? a.k_sz : a.v_sz;
  // A token range of this CTA: blocks [0, nblk) starting at token tok0, tokens
  // [lo, hi) attended, table entry tb + token / P. Warp w takes blocks (pairs)
  // w, w + W, ... of each range.
  struct Range {
    int tok0, nblk, lo, hi, tb;
  };
  const Range sinks_r = {0, nsb, 0, sink_hi, 0};
  auto issue = [&](const Range &r, int kb, int st) {
    const int btok = r.tok0 + kb * 16;
    const int lp = btok / P;
    const int page = tbl[r.tb + lp];
    const int in_page = btok - lp * P;
    // rows [rlo, rhi) of the block hold tokens of this range
    const int rlo = page >= 0 ? max(0, r.lo - btok) : 16;
    const int rhi = page >= 0 ? min(16, r.hi - btok) : 0;
    // rows of an invalid page are zero-filled; the address stays inside page 0
    const size_t row0 = ((size_t)(page >= 0 ? page : 0) * a.hkv + h) * P + in_page;
    issue_block<D, KVT>(lm, ring + st * T::kStageBytes, kbase, vbase, sz_base, row0, rlo, rhi,
                        lane);
  };

  // Each warp leaves a record in its ring: the running max m and denominator
  // l of every head, and O already divided by l; the CTA merges the records.
  float *rec = reinterpret_cast<float *>(smem + warp * SM::kRingBytesPerWarp);
  float *rec_o = rec + 16;

  if constexpr (KVT == PA_KV_BF16) {
    WarpAcc<D> acc;
    acc.reset();
    // one range through the warp's ring; the online softmax state carries over
    auto pass = [&](const Range &r) {
      const int wr = warp;
      const int nmine = r.nblk > wr ? (r.nblk - wr + W - 1) / W : 0;
#pragma unroll
      for (int st = 0; st < NSTAGE - 1; ++st) {
        if (st < nmine) issue(r, wr + st * W, st);
        cp_async_commit();
      }
      for (int k = 0; k < nmine; ++k) {
        __syncwarp();
        {
          const int kn = k + NSTAGE - 1;
          if (kn < nmine) issue(r, wr + kn * W, kn % NSTAGE);
          cp_async_commit();
        }
        cp_async_wait<NSTAGE - 1>();
        __syncwarp();  // every lane's pieces of this block are now visible to the warp

        const int kb = wr + k * W;
        const int btok = r.tok0 + kb * 16;
        const bool pvalid = tbl[r.tb + btok / P] >= 0;
        const uint32_t src = ring + (k % NSTAGE) * T::kStageBytes;
        block_step<D>(lm, src, btok, r.lo, r.hi, pvalid, a.scale_log2, qa, t, acc);
      }
      cp_async_wait<0>();
      __syncwarp();
    };
    if (nsb > 0) pass(sinks_r);  // CTA-uniform: split 0's sinks first
    pass(Range{tok0, nblk, tok_lo, tok1, nsp - lp0});
    // lane (g, t) ends with head g's max and its share of head g's
    // denominator, and O^T columns of heads 2t, 2t + 1
    float l_run = acc.l_run;
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    const float inv0 = __shfl_sync(0xffffffffu, inv, 8 * t);      // head 2t
    const float inv1 = __shfl_sync(0xffffffffu, inv, 8 * t + 4);  // head 2t + 1
    if (t == 0) {
      rec[g] = acc.m_run;
      rec[8 + g] = l_run;
    }
#pragma unroll
    for (int j = 0; j < T::kMTiles; ++j) {
      const int d0 = out_col<D, KVT>(j, g);
      *reinterpret_cast<float2 *>(rec_o + (2 * t) * D + d0) =
          make_float2(acc.o[j][0] * inv0, acc.o[j][2] * inv0);
      *reinterpret_cast<float2 *>(rec_o + (2 * t + 1) * D + d0) =
          make_float2(acc.o[j][1] * inv1, acc.o[j][3] * inv1);
    }
  } else {
    // two 16-token blocks per step: pair k of this warp is blocks 2 kp and
    // 2 kp + 1, kp = warp + k W; a ring stage holds one pair
    constexpr int NPS = NSTAGE / 2;
    static_assert(NSTAGE % 2 == 0 && NPS >= 2, "quantised pools stage pairs of blocks");
    auto issue_pair = [&](const Range &r, int kp, int st) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int kb = 2 * kp + u;
        if (kb < r.nblk) {
          issue(r, kb, 2 * st + u);
        } else {  // no such block: zero-fill the stage (codes and scales 0)
          issue_block<D, KVT>(lm, ring + (2 * st + u) * T::kStageBytes, kbase, vbase, sz_base,
                              (size_t)h * P, 16, 0, lane);
        }
      }
    };
    QAcc<D> acc;
    acc.reset();
    // sums of q of heads 2t, 2t + 1 (held by lanes 8t and 8t + 4)
    const float qz[2] = {__shfl_sync(0xffffffffu, qsum, 8 * t) * a.scale_log2,
                         __shfl_sync(0xffffffffu, qsum, 8 * t + 4) * a.scale_log2};
    const float kscale = kCodeScale<KVT> * a.scale_log2;
    // one range through the warp's ring; the online softmax state carries over
    auto pass = [&](auto pack_c, const Range &r) {
      constexpr bool kPack = decltype(pack_c)::value;
      const int wr = warp;
      const int npair = (r.nblk + 1) / 2;
      const int npmine = npair > wr ? (npair - wr + W - 1) / W : 0;
#pragma unroll
      for (int st = 0; st < NPS - 1; ++st) {
        if (st < npmine) issue_pair(r, wr + st * W, st);
        cp_async_commit();
      }
      for (int k = 0; k < npmine; ++k) {
        __syncwarp();
        {
          const int kn = k + NPS - 1;
          if (kn < npmine) issue_pair(r, wr + kn * W, kn % NPS);
          cp_async_commit();
        }
        cp_async_wait<NPS - 1>();
        __syncwarp();

        const int kb = 2 * (wr + k * W);
        const int btok[2] = {r.tok0 + kb * 16, r.tok0 + kb * 16 + 16};
        const bool pvalid[2] = {tbl[r.tb + btok[0] / P] >= 0,
                                kb + 1 < r.nblk && tbl[r.tb + btok[1] / P] >= 0};
        const uint32_t src = ring + (k % NPS) * 2 * T::kStageBytes;
        pair_step<D, KVT, kPack>(lm, src, btok, pvalid, r.lo, r.hi, kscale, qz, qa, g, t, acc);
      }
      cp_async_wait<0>();
      __syncwarp();
    };
    auto loop = [&](auto pack_c) {
      constexpr bool kPack = decltype(pack_c)::value;
      if (nsb > 0) pass(pack_c, sinks_r);  // CTA-uniform: split 0's sinks first
      pass(pack_c, Range{tok0, nblk, tok_lo, tok1, nsp - lp0});
      if constexpr (kPack) {
        // high + low halves: lanes t < 2 end with the full O^T of heads 2t, 2t + 1
#pragma unroll
        for (int j = 0; j < T::kMTiles; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc.o[j][e] += __shfl_xor_sync(0xffffffffu, acc.o[j][e], 2);
      }
    };
    if (G <= 4) {  // CTA-uniform
      loop(std::true_type{});
    } else {
      loop(std::false_type{});
    }
    cp_async_wait<0>();
    __syncwarp();
    // reduce the two heads' denominators and zero-point sums over the lanes
    // holding their tokens, then O = (code scale * 2^E * O + sum p z) / l
    // (the code scale is applied to O first: code scale x 2^E alone may pass
    // the fp32 range when E is large)
    constexpr float kRowHiScale = T::kU4 ? kCodeScale<KVT> / 16.f : kCodeScale<KVT>;
    float pe[2], zl[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        acc.l[hh] += __shfl_xor_sync(0xffffffffu, acc.l[hh], off);
        acc.z[hh] += __shfl_xor_sync(0xffffffffu, acc.z[hh], off);
      }
      const float inv = acc.l[hh] > 0.f ? 1.f / acc.l[hh] : 0.f;
      pe[hh] = acc.f == 0.f ? 0.f : exp2i(acc.e) * inv;
      zl[hh] = acc.z[hh] * inv;
    }
    if (g == 0) {
      rec[2 * t] = acc.m[0];
      rec[2 * t + 1] = acc.m[1];
      rec[8 + 2 * t] = acc.l[0];
      rec[8 + 2 * t + 1] = acc.l[1];
    }
#pragma unroll
    for (int j = 0; j < T::kMTiles; ++j) {
      const int d0 = out_col<D, KVT>(j, g);
      // rows d + 1 of INT4 tiles hold the high nibbles (16x the code scale)
      *reinterpret_cast<float2 *>(rec_o + (2 * t) * D + d0) =
          make_float2(fmaf(acc.o[j][0] * kCodeScale<KVT>, pe[0], zl[0]),
                      fmaf(acc.o[j][2] * kRowHiScale, pe[0], zl[0]));
      *reinterpret_cast<float2 *>(rec_o + (2 * t + 1) * D + d0) =
          make_float2(fmaf(acc.o[j][1] * kCodeScale<KVT>, pe[1], zl[1]),
                      fmaf(acc.o[j][3] * kRowHiScale, pe[1], zl[1]));
    }
  }
  __syncthreads();

  // ---- merge the CTA's warps (fixed order: deterministic); a thread takes
  // four consecutive elements of one head
  constexpr int D4 = D / 4;
  for (int e = threadIdx.x; e < G * D4; e += W * 32) {
    const int hd = e / D4;
    const int d4 = e - hd * D4;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w)
      M = fmaxf(M, reinterpret_cast<const float *>(smem + w * SM::kRingBytesPerWarp)[hd]);
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const float *r = reinterpret_cast<const float *>(smem + w * SM::kRingBytesPerWarp);
        const float fl = fast_exp2(r[hd] - M) * r[8 + hd];  // 0 for empty warps
        const float4 v = reinterpret_cast<const float4 *>(r + 16 + hd * D)[d4];
        num.x = fmaf(fl, v.x, num.x);
        num.y = fmaf(fl, v.y, num.y);
        num.z = fmaf(fl, v.z, num.z);
        num.w = fmaf(fl, v.w, num.w);
        L += fl;
      }
    }
    const size_t row = (size_t)b * a.hq + (size_t)h * G + hd;
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const float4 val = make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
    if (n_live == 1 && a.n_prior == 0 && !a.keep_partials) {
      reinterpret_cast<float4 *>(a.out + row * D)[d4] = val;
    } else {
      reinterpret_cast<float4 *>(a.o_part + (row * a.S + slot) * D)[d4] = val;
      if (d4 == 0) a.lse[row * a.S + slot] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
  }
  if (a.keep_partials) return;  // the caller merges
  if (n_live == 1) {
    if (a.n_prior == 0) return;
    __syncthreads();  // our own partial is visible to the whole CTA
    merge_rows<D>(a, b, h, G, 1, reinterpret_cast<float *>(smem));
    return;
  }

  // ---- split-KV merge, done by whichever CTA of this (sequence, KV head)
  // finishes last. Partials are made visible device-wide before the ticket is
  // taken; the merge visits splits in index order, so the result does not
  // depend on which CTA merges. The last CTA also re-arms the counter.
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int ticket = atomicAdd(a.counters + (size_t)b * a.hkv + h, 1);
    s_last = ticket == n_live - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  merge_rows<D>(a, b, h, G, n_live, reinterpret_cast<float *>(smem));
  if (threadIdx.x == 0) a.counters[(size_t)b * a.hkv + h] = 0;
}

template <int D, int P, int KVT,
          int NS = KVT != PA_KV_BF16 ? PA_DECODE_STAGES_U8 : PA_DECODE_STAGES_BF16>
struct Config {
  static constexpr int W = PA_DECODE_WARPS;
  static constexpr int NSTAGE = NS;
  using SM = Smem<D, KVT, W, NSTAGE>;
  static auto kernel() { return &decode_kernel<D, P, KVT, W, NSTAGE>; }
  static void *fn() { return reinterpret_cast<void *>(kernel()); }
};

// Largest dynamic shared memory a decode CTA may request (ring + table slice).
template <class C>
constexpr int max_smem() {
  return (int)C::SM::bytes(kMaxPagesPerSplit);
}

// Opt each kernel instance in to its dynamic shared memory once per device.
template <class C>
cudaError_t ensure_smem_attr() {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(C::fn(), cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem<C>());
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <class C>
cudaError_t launch_cfg(const DecodeArgs &a, cudaStream_t stream) {
  cudaError_t e = ensure_smem_attr<C>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.S, a.hkv, a.B);
  cfg.blockDim = dim3(C::W * 32);
  cfg.dynamicSmemBytes = C::SM::bytes(a.tbl_cap);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = PA_DECODE_PDL ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, C::kernel(), a);
}

template <int D, int P, int KVT>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t stream) {
  // A ragged batch launched longest unit first over several waves of CTAs
  // (ordered == 2) runs one CTA per (sequence, KV head), each streaming its
  // whole unit: there deeper rings (two CTAs per SM instead of three) pay.
  // Measured on the Llama-3-8B-shaped step: bf16 with three blocks per warp
  // instead of two 2-6 % faster (and 5 % slower on one wave of equal units,
  // the Llama-3-70B step, which keeps two); INT8 and FP8 with three pairs
  // instead of two 0.7-2.7 % faster on two B200s, 0.5 % slower on a third.
  // INT4 keeps its ring (four CTAs per SM fit only with it).
  if constexpr (KVT == PA_KV_BF16)
    if (a.ordered == 2) return launch_cfg<Config<D, P, KVT, PA_DECODE_STAGES_BF16_LPT>>(a, stream);
  if constexpr (KVT == PA_KV_U8_PER_TOKEN || KVT == PA_KV_FP8_PER_TOKEN)
    if (a.ordered == 2) return launch_cfg<Config<D, P, KVT, PA_DECODE_STAGES_U8_LPT>>(a, stream);
  return launch_cfg<Config<D, P, KVT>>(a, stream);
}

template <int D, int P, int KVT>
int ctas_per_sm_t() {
  using C = Config<D, P, KVT>;
  const size_t smem = C::SM::bytes(256);
  if (ensure_smem_attr<C>() != cudaSuccess) return 1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, C::fn(), C::W * 32, smem) != cudaSuccess)
    return 1;
  return n > 0 ? n : 1;
}

}  // namespace

#define PA_DISPATCH(D_, P_, K_, CALL)                                  \
  if (D == D_ && P == P_ && kv_dtype == K_) return CALL<D_, P_, K_>

cudaError_t launch_decode(int D, int P, int kv_dtype, const DecodeArgs &a, cudaStream_t stream) {
#define PA_L(D_, P_, K_) PA_DISPATCH(D_, P_, K_, launch_t)(a, stream)
  PA_L(128, 16, 0); PA_L(128, 32, 0); PA_L(64, 16, 0); PA_L(64, 32, 0);
  PA_L(128, 16, 1); PA_L(128, 32, 1); PA_L(64, 16, 1); PA_L(64, 32, 1);
  PA_L(128, 16, 2); PA_L(128, 32, 2); PA_L(64, 16, 2); PA_L(64, 32, 2);
  PA_L(128, 16, 3); PA_L(128, 32, 3); PA_L(64, 16, 3); PA_L(64, 32, 3);
#undef PA_L
  return cudaErrorInvalidValue;
}

int decode_ctas_per_sm(int D, int P, int kv_dtype) {
#define PA_O(D_, P_, K_) PA_DISPATCH(D_, P_, K_, ctas_per_sm_t)()
  PA_O(128, 16, 0); PA_O(128, 32, 0); PA_O(64, 16, 0); PA_O(64, 32, 0);
  PA_O(128, 16, 1); PA_O(128, 32, 1); PA_O(64, 16, 1); PA_O(64, 32, 1);
  PA_O(128, 16, 2); PA_O(128, 32, 2); PA_O(64, 16, 2); PA_O(64, 32, 2);
  PA_O(128, 16, 3); PA_O(128, 32, 3); PA_O(64, 16, 3); PA_O(64, 32, 3);
#undef PA_O
  return 1;
}

}  // namespace pa
