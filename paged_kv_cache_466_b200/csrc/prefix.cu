// Shared-prefix attention: the prefix half of a cascade decode, on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// "KV-Cache Optimization Techniques", section "Prefix Caching" (Eq. 2): when
// many requests share a prompt prefix, its KV pages are stored once and every
// request's page table points at them. Eq. 1 over [prefix; own tokens] splits
// exactly into attention over the prefix and attention over the request's own
// tokens, merged by log-sum-exp. This kernel does the prefix part for all
// requests at once: per KV head, the B*G query rows that read that head form
// an [rows x D] x [D x prefix] contraction, so each prefix K/V row is read once
// per 128-row tile instead of once per request, and the products run as dense
// tensor-core tiles with a FlashAttention-style online softmax.
//
// CTA (4 warps, 128 threads) = 128 query rows of one KV head (row r of the
// head is sequence r / G, query head h * G + r % G) over one prefix split of
// 64-token tiles. Per tile:
//   S[128 x 64]  = Q K^T  : tcgen05.mma kind::f16, A = Q and B = K tile, both
//                           K-major 128-byte-swizzled in shared memory, S in
//                           tensor memory (64 fp32 columns)
//   softmax                : thread r owns row r (TMEM lane r): tcgen05.ld of
//                           its 64 scores, online max / sum in fp32, P split
//                           into bf16 hi + lo and stored back to tensor memory
//                           (tcgen05.st, two bf16 per column)
//   O[128 x D]  += P V     : A = P from tensor memory, B = V tile (MN-major in
//                           shared memory, the page rows as they are), O in
//                           tensor memory
// Thread 0 issues the MMAs and commits them to an mbarrier; every wait on it
// is bounded. K/V tiles are staged by all threads with 16-byte cp.async into
// a 2-stage ring, the copy of tile k + 1 overlapping the softmax of tile k,
// and PV(k) and S(k + 1) go to the tensor core back to back behind one CTA
// barrier per tile; 96 KB of shared memory and 256 TMEM columns let two CTAs share an
// SM, so one CTA's softmax overlaps the other's MMAs. The output per row is
// the normalised partial and its natural-log log-sum-exp, merged with the
// suffix by the decode kernel.
#include <atomic>
#include <cmath>
#include <cstring>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr float kLn2 = 0.693147180559945309f;
constexpr int kRowsPerCta = 128;  // the MMA's M
constexpr int kTileTok = 64;      // N of S, K of PV
constexpr int kThreads = 128;
constexpr int kTmemCols = 256;    // S [0, 64), P hi [64, 96), P lo [96, 128), O [128, 128 + D)
constexpr float kRescaleLog2 = 8.0f;

// Byte offset of 16-byte chunk `chunk` of row r in a K-major,
// 128-byte-swizzled tile of `rows` rows: 64-element K atoms of rows * 128
// bytes, 8-row groups of 1024 bytes, chunks XOR-permuted by row % 8 (the
// layout the tensor core's SWIZZLE_128B descriptor reads). The MN-major V
// tile uses the same formula with (row, chunk) = (token, d / 8).
__device__ __forceinline__ uint32_t sw128(int r, int chunk, int rows) {
  return (chunk >> 3) * rows * 128 + (r >> 3) * 1024 + (r & 7) * 128 +
         (((chunk & 7) ^ (r & 7)) << 4);
}

// Shared-memory matrix descriptor: start address, leading / stride byte
// offsets, version 1, SWIZZLE_128B.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  const uint32_t lo = ((addr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
  const uint32_t hi = ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
  return ((uint64_t)hi << 32) | lo;
}

// Instruction descriptor: bf16 x bf16 -> fp32, M = 128, N = n, A K-major,
// B K-major or MN-major.
__host__ __device__ constexpr uint32_t instr_desc(int n, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kRowsPerCta >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          int accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// The same with A read from tensor memory (lane = row, two bf16 per column).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                             uint32_t idesc, int accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
      bar));
}

// A commit that has not arrived after this long will not arrive: the kernel
// stops waiting, reports PA_DERR_TIMEOUT and still releases its tensor memory.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s (a tile takes microseconds)

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  return mbar_wait_bounded(bar, parity, kWaitLimitNs);
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 lanes x 32 bits x 32 columns from tensor memory: thread i of the warp
// gets lane (taddr lane + i), columns taddr .. taddr + 31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31]));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, float4 v) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}

// Box of the 5-D tensor map at `tmap` (a kernel parameter) whose first
// element is (x0 .. x4), from shared memory at `src`; completes as a bulk
// group of the issuing thread.
__device__ __forceinline__ void tma_store_5d(const CUtensorMap *tmap, uint32_t src, int x0, int x1,
                                             int x2, int x3, int x4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3, %4, %5}], "
      "[%6];" ::"l"(tmap),
      "r"(x0), "r"(x1), "r"(x2), "r"(x3), "r"(x4), "r"(src)
      : "memory");
}

template <int D>
struct PLayout {
  static constexpr int kChunks = D / 8;                       // 16-byte chunks per row
  static constexpr int kQBytes = kRowsPerCta * D * 2;         // Q tile
  static constexpr int kKVBytes = kTileTok * D * 2;           // one K or V tile
  static constexpr int kQOff = 0;
  static constexpr int kStageOff = kQBytes;                   // 2 stages of K, V
  static constexpr int kBarOff = kStageOff + 4 * kKVBytes;    // 2 mbarriers + TMEM address
  static constexpr int kPagesOff = kBarOff + 64;
  static constexpr int kKSteps = D / 16;                      // MMAs per S
};

template <int D, int P>
__global__ void __launch_bounds__(kThreads, 2)
    prefix_kernel(const __grid_constant__ PrefixArgs a) {
  using L = PLayout<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the swizzled tiles need 1024-byte aligned atoms
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  pdl_wait_primary();
  // the work before this pass is finished and visible: the suffix decode,
  // which does not read this pass's output, may start beside it now
  pdl_launch_dependents();

  const int mt = blockIdx.x;
  const int h = blockIdx.y;
  const int ps = blockIdx.z;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int G = a.hq / a.hkv;
  const int rows = a.B * G;

  const int n_tiles = (a.prefix_len + kTileTok - 1) / kTileTok;
  const int tile0 = ps * a.tiles_per_split;
  const int tile1 = min(tile0 + a.tiles_per_split, n_tiles);
  const int tok_lo = tile0 * kTileTok;
  const int tok_hi = min(tile1 * kTileTok, a.prefix_len);
  const int ntl = tile1 - tile0;

  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_s = sbase + L::kBarOff;       // S of tile k done (and PV of k - 1)
  const uint32_t bar_pv = sbase + L::kBarOff + 8;  // the last tile's PV done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kBarOff + 16);
  int *pages = reinterpret_cast<int *>(smem + L::kPagesOff);

  // prefix page ids of this split, bounds-checked
  const int pg0 = tok_lo / P;
  const int npg = tok_hi > tok_lo ? (tok_hi - 1) / P - pg0 + 1 : 0;
  for (int i = tid; i < npg; i += kThreads) {
    int pg = __ldg(a.prefix_pages + pg0 + i);
    if (pg < 0 || pg >= a.num_pages) {
      flag_error(a.d_err, PA_DERR_BAD_PAGE);
      pg = -1;
    }
    pages[i] = pg;
  }

  // this thread's query row (TMEM lane tid)
  const int r = mt * kRowsPerCta + tid;
  const bool row_ok = r < rows;
  const size_t qrow = (size_t)(row_ok ? r / G : 0) * a.hq + (size_t)h * G + (row_ok ? r % G : 0);

  // Q tile: row tid, D / 8 chunks of 16 bytes, zero rows past the batch
  {
    const unsigned char *qsrc = static_cast<const unsigned char *>(a.q) + qrow * D * 2;
#pragma unroll
    for (int c = 0; c < L::kChunks; ++c)
      cp_async16(sbase + L::kQOff + sw128(tid, c, kRowsPerCta), qsrc + c * 16, row_ok ? 16u : 0u);
    cp_async_commit();
  }

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar_s), "r"(1));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar_pv), "r"(1));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();  // page ids, barriers and the TMEM address are visible
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem;                              // S columns
  const uint32_t t_ph = tmem + kTileTok;                  // P hi: 2 bf16 per column
  const uint32_t t_pl = t_ph + kTileTok / 2;              // P lo
  const uint32_t t_o = tmem + 2 * kTileTok;               // O columns
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lanes

  const unsigned char *kbase = static_cast<const unsigned char *>(a.k_pool);
  const unsigned char *vbase = static_cast<const unsigned char *>(a.v_pool);
  // K and V tile k into stage st: 64 token rows x D / 8 chunks each; rows of
  // tokens past the split or of invalid pages are zero-filled
  auto load_tile = [&](int k, int st) {
    const int ttok = tok_lo + k * kTileTok;
    const uint32_t ks = sbase + L::kStageOff + st * 2 * L::kKVBytes;
    constexpr int kPer = kTileTok * L::kChunks / kThreads;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int c = tid + i * kThreads;
      const int row = c / L::kChunks;
      const int chunk = c % L::kChunks;
      const int tok = ttok + row;
      int page = -1;
      if (tok < tok_hi) page = pages[tok / P - pg0];
      const bool ok = page >= 0;
      const size_t grow = ((size_t)(ok ? page : 0) * a.hkv + h) * P + (ok ? tok % P : 0);
      const uint32_t so = sw128(row, chunk, kTileTok);
      cp_async16(ks + so, kbase + grow * D * 2 + chunk * 16, ok ? 16u : 0u);
      cp_async16(ks + L::kKVBytes + so, vbase + grow * D * 2 + chunk * 16, ok ? 16u : 0u);
    }
  };

  float m_run = -INFINITY;  // this row's running max (log2 units)
  float l_run = 0.f;        // this row's softmax denominator
  bool ok_waits = true;

  // S = Q K^T of the tile staged in stage st, into the S columns
  auto issue_s = [&](int st) {
    const uint32_t q0 = sbase + L::kQOff;
    const uint32_t k0 = sbase + L::kStageOff + st * 2 * L::kKVBytes;
#pragma unroll
    for (int kk = 0; kk < L::kKSteps; ++kk) {
      const uint32_t off = (kk & 3) * 32;  // 16 elements along K inside a 128-byte atom
      umma_bf16(t_s, smem_desc(q0 + (kk >> 2) * (kRowsPerCta * 128) + off, 16, 1024),
                smem_desc(k0 + (kk >> 2) * (kTileTok * 128) + off, 16, 1024),
                instr_desc(kTileTok, false), kk > 0);
    }
  };
  // O += P V for the tile in stage st (hi and lo halves of P, A from tensor
  // memory: 8 columns per 16 tokens)
  auto issue_pv = [&](int st, bool first) {
    const uint32_t v0 = sbase + L::kStageOff + st * 2 * L::kKVBytes + L::kKVBytes;
#pragma unroll
    for (int kk = 0; kk < kTileTok / 16; ++kk) {
      const uint64_t dv = smem_desc(v0 + kk * 2048, kTileTok * 128, 1024);
      umma_bf16_ts(t_o, t_ph + kk * 8, dv, instr_desc(D, true), !first || kk > 0);
      umma_bf16_ts(t_o, t_pl + kk * 8, dv, instr_desc(D, true), 1);
    }
  };

  // Pipeline: one barrier per tile. After the softmax of tile k (and the
  // arrival of tile k + 1's copies), thread 0 issues PV(k) and S(k + 1) back
  // to back and commits them together; the wait on that commit at the top of
  // the next iteration covers both, which frees stage k's V, the P columns
  // and O for the next softmax.
  if (ntl > 0) load_tile(0, 0);
  cp_async_commit();
  cp_async_wait<0>();                                           // Q and tile 0
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0 && ntl > 0) {
    issue_s(0);
    umma_commit(bar_s);
  }
  for (int k = 0; k < ntl; ++k) {
    const int st = k & 1;
    // S(k) is complete, and with it PV(k - 1): stage st ^ 1, the P columns
    // and O are free
    ok_waits &= mbar_wait(bar_s, k & 1);
    tc_fence_after();
    if (k + 1 < ntl) load_tile(k + 1, st ^ 1);
    cp_async_commit();

    // ---- online softmax of row tid (log2 units)
    const int ttok = tok_lo + k * kTileTok;
    float s[kTileTok];
    {
      uint32_t u[32];
      tmem_ld32(t_s + lane_off, u);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) s[j] = __uint_as_float(u[j]);
      tmem_ld32(t_s + lane_off + 32, u);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) s[32 + j] = __uint_as_float(u[j]);
    }
    // a whole tile of valid pages needs no mask (uniform over the CTA)
    bool full = ttok + kTileTok <= tok_hi;
#pragma unroll
    for (int i = 0; i < kTileTok / P; ++i) full = full && pages[ttok / P + i - pg0] >= 0;
    float mx = -INFINITY;
    if (full) {
#pragma unroll
      for (int j = 0; j < kTileTok; ++j) {
        s[j] *= a.scale_log2;
        mx = fmaxf(mx, s[j]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < kTileTok; ++j) {
        const int tok = ttok + j;
        const bool live = tok < tok_hi && pages[tok / P - pg0] >= 0;
        s[j] = live ? s[j] * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[j]);
      }
    }
    const bool need = mx > m_run + kRescaleLog2 || (m_run == -INFINITY && mx > -INFINITY);
    if (__any_sync(0xffffffffu, need)) {  // warp-uniform: tcgen05.ld/st are warp-wide
      const float m_new = need ? fmaxf(m_run, mx) : m_run;
      const float alpha = need && m_run != -INFINITY ? fast_exp2(m_run - m_new) : 1.f;
      if (need) {
        m_run = m_new;
        l_run *= alpha;
      }
      if (k > 0) {  // O holds earlier tiles: scale it
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t u[32];
          tmem_ld32(t_o + lane_off + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(__uint_as_float(u[j]) * alpha);
          tmem_st32(t_o + lane_off + c0, u);
        }
        tmem_wait_st();
      }
    }
    const float mref = m_run == -INFINITY ? 0.f : m_run;
    // P = exp2(s - m), split into bf16 hi + lo; column j of each half holds
    // tokens 2j (low 16 bits) and 2j + 1 of row tid
    {
      uint32_t wh[kTileTok / 2], wl[kTileTok / 2];
#pragma unroll
      for (int j = 0; j < kTileTok / 2; ++j) {
        const float p0 = fast_exp2(s[2 * j] - mref);
        const float p1 = fast_exp2(s[2 * j + 1] - mref);
        l_run += p0 + p1;
        split_bf16(p0, p1, wh[j], wl[j]);
      }
      tmem_st32(t_ph + lane_off, wh);
      tmem_st32(t_pl + lane_off, wl);
      tmem_wait_st();
    }
    cp_async_wait<0>();                                           // tile k + 1
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
    tc_fence_before();
    __syncthreads();  // P stored, O scaled, S(k) read by all, tile k + 1 staged
    tc_fence_after();
    if (tid == 0) {
      issue_pv(st, k == 0);
      if (k + 1 < ntl) {
        issue_s(st ^ 1);
        umma_commit(bar_s);
      } else {
        umma_commit(bar_pv);
      }
    }
  }
  cp_async_wait<0>();

  // ---- normalise and write this split's partial for row tid
  if (ntl > 0) ok_waits &= mbar_wait(bar_pv, 0);  // the one commit of the last PV
  tc_fence_after();
  const size_t R = (size_t)a.B * a.hq;
  const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
  if (a.tma_store) {
    // Every MMA and copy has completed, so the Q tile and the K/V stages are
    // free: O / l goes there as 32-column boxes of 128 rows (128-byte rows,
    // 16-byte pieces swizzled by row, conflict-free), and one thread writes
    // them with the tensor memory accelerator in whole lines. (Plain stores
    // put 16-byte pieces of 32 rows in every warp instruction.)
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t u[32];
      if (ntl > 0) {
        tmem_ld32(t_o + lane_off + c0, u);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) u[j] = 0u;
      }
      const uint32_t rowb = sbase + (c0 / 32) * (kRowsPerCta * 128) + tid * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        sts128(rowb + ((j ^ (tid & 7)) << 4),
               make_float4(__uint_as_float(u[4 * j]) * inv, __uint_as_float(u[4 * j + 1]) * inv,
                           __uint_as_float(u[4 * j + 2]) * inv,
                           __uint_as_float(u[4 * j + 3]) * inv));
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the copy engine
    __syncthreads();
    const int seq0 = mt * kRowsPerCta / G;
    if (tid == 0 && seq0 < a.B) {
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32)
        tma_store_5d(&a.tmo, sbase + (c0 / 32) * (kRowsPerCta * 128), c0, 0, h, seq0, ps);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // before the CTA exits
    }
  } else {
    float *orow = a.o_pre + ((size_t)ps * R + qrow) * D;
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t u[32];
      if (ntl > 0) {
        tmem_ld32(t_o + lane_off + c0, u);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) u[j] = 0u;
      }
      if (row_ok) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4 *>(orow + c0 + j) =
              make_float4(__uint_as_float(u[j]) * inv, __uint_as_float(u[j + 1]) * inv,
                          __uint_as_float(u[j + 2]) * inv, __uint_as_float(u[j + 3]) * inv);
      }
    }
  }
  if (row_ok)
    a.lse_pre[(size_t)ps * R + qrow] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
  if (!ok_waits) flag_error(a.d_err, PA_DERR_TIMEOUT);

  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
}

// cuTensorMapEncodeTiled, looked up through the runtime (the library does not
// link the driver library); null if the driver lacks it.
using TmapEncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

TmapEncodeFn tmap_encoder() {
  static const TmapEncodeFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<TmapEncodeFn>(p);
  }();
  return fn;
}

// The prefix partials o_pre [n_psplits][B][Hq][D] as the 5-D tensor
// [n_psplits][B][Hkv][G][D], written in boxes of 32 elements x G heads x
// 128 / G sequences (one 128-row tile of a KV head, 32 columns) with the
// 128-byte swizzle. False where G does not divide 128 or the driver cannot
// encode it: the kernel then uses plain stores.
// The last map this thread encoded and what it was encoded for: a cascade
// called step after step with the same workspace and shapes reuses it.
struct PartialsMapCache {
  const void *o_pre = nullptr;
  int D = 0, B = 0, hq = 0, hkv = 0, n = 0;
  bool ok = false;
  CUtensorMap map;
};

bool encode_partials(PrefixArgs *a, int D) {
  const int G = a->hq / a->hkv;
  if (kRowsPerCta % G != 0) return false;
  thread_local PartialsMapCache c;
  if (c.o_pre == a->o_pre && c.D == D && c.B == a->B && c.hq == a->hq && c.hkv == a->hkv &&
      c.n == a->n_psplits) {
    if (c.ok) std::memcpy(&a->tmo, &c.map, sizeof(CUtensorMap));
    return c.ok;
  }
  const TmapEncodeFn f = tmap_encoder();
  if (f == nullptr) return false;
  const cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)G, (cuuint64_t)a->hkv, (cuuint64_t)a->B,
                              (cuuint64_t)a->n_psplits};
  const cuuint64_t strides[4] = {(cuuint64_t)D * 4, (cuuint64_t)G * D * 4,
                                 (cuuint64_t)a->hq * D * 4, (cuuint64_t)a->B * a->hq * D * 4};
  const cuuint32_t box[5] = {32, (cuuint32_t)G, 1, (cuuint32_t)(kRowsPerCta / G), 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const bool ok =
      f(&a->tmo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, a->o_pre, dims, strides, box, estr,
        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  c.o_pre = a->o_pre;
  c.D = D;
  c.B = a->B;
  c.hq = a->hq;
  c.hkv = a->hkv;
  c.n = a->n_psplits;
  c.ok = ok;
  if (ok) std::memcpy(&c.map, &a->tmo, sizeof(CUtensorMap));
  return ok;
}

// Opt the kernel instance in to its shared memory once per device.
template <int D, int P>
cudaError_t ensure_prefix_smem(int max_smem) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(prefix_kernel<D, P>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           max_smem);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int D, int P>
cudaError_t launch_prefix_t(const PrefixArgs &a_in, bool programmatic, cudaStream_t stream) {
  using L = PLayout<D>;
  PrefixArgs a = a_in;
  a.tma_store = encode_partials(&a, D) ? 1 : 0;
  const int max_pages_per_split = a.tiles_per_split * kTileTok / P + 2;
  if (max_pages_per_split > 4096) return cudaErrorInvalidValue;
  constexpr int kMaxSmem = L::kPagesOff + 4 * 4096 + 1024;  // + alignment slack
  static_assert(kMaxSmem <= 227 * 1024, "shared memory");
  const size_t smem = L::kPagesOff + (size_t)max_pages_per_split * 4 + 1024;
  const cudaError_t e = ensure_prefix_smem<D, P>(kMaxSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.B * (a.hq / a.hkv) + kRowsPerCta - 1) / kRowsPerCta, a.hkv, a.n_psplits);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = programmatic ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, prefix_kernel<D, P>, a);
}

}  // namespace

int prefix_rows_per_cta() { return kRowsPerCta; }
int prefix_tile_tokens() { return kTileTok; }

cudaError_t launch_prefix(int D, int P, const PrefixArgs &a, bool programmatic,
                          cudaStream_t stream) {
  if (D == 128 && P == 16) return launch_prefix_t<128, 16>(a, programmatic, stream);
  if (D == 128 && P == 32) return launch_prefix_t<128, 32>(a, programmatic, stream);
  if (D == 64 && P == 16) return launch_prefix_t<64, 16>(a, programmatic, stream);
  if (D == 64 && P == 32) return launch_prefix_t<64, 32>(a, programmatic, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa
