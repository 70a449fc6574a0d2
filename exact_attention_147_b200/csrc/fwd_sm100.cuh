// Forward pass of exact attention on sm_100a tensor cores (tcgen05 + TMEM).
//
// Work split (FlashAttention-2 abstract, arXiv 2307.08691: parallelise over
// thread blocks even within one head; FlashAttention-2 wiki article
// "Technical architecture", improvement 2): the unit of work is a PAIR of
// 128-row query tiles of one (batch, head); the units (query pairs x heads x
// batch) are ordered longest-first when masks make them uneven, and a
// persistent grid of one CTA per SM walks them with a fixed stride, so a
// single long head already fills the GPU and one unit's loads and first
// products overlap the previous unit's epilogue.
//
// Inside a CTA (16 warps, four warpgroups):
//   warps 0-3   softmax for query tile 0 (thread = one query row)
//   warps 4-7   softmax for query tile 1
//   warps 8-11  epilogue: O_t / l out of TMEM, bf16 rows and LSE to HBM;
//               with dropout they also draw each block's mask (keep bits)
//               into a shared-memory ring a block ahead of the softmax
//   warp  12    TMA producer: Q once per unit, then K_j, V_j into a ring of slots
//   warp  13    MMA issuer: S_t = Q_t K_j^T and O_t += P_t V_j (tcgen05)
//   warps 14-15 idle (they complete the fourth warpgroup for setmaxnreg)
// The Q tiles stay resident in shared memory and K/V tiles stream through a
// multi-slot TMA + mbarrier ring ("FlashAttention v2" article, §3.1-§3.2:
// Q kept on chip, K/V prefetched while the current block is computed).
//
// The Q buffers are double-buffered across units (single-buffered with
// dropout, whose mask ring takes that space); O leaves through registers
// (normalised, cast to bf16 and stored by the row's own thread), so shared
// memory holds only Q, the K/V ring and, with dropout, the mask ring.
//
// Tensor memory (512 columns x 128 lanes of fp32):
//   [0,128)    S_0 (P_0 as bf16 pairs in its first 64 columns)
//   [128,256)  S_1 (P_1 likewise)
//   [256,256+d)      O_0 accumulator
//   [256+d,256+2d)   O_1 accumulator
// P is written back over S and fed to the PV product straight from TMEM.
// The tensor-core pipe runs its instructions in issue order, so S_t of the
// next block may be issued right after the PV product that still reads P_t.
// At d = 64 the O tiles leave 128 columns free and P_t gets its own 64
// ([384 + 64t, 448 + 64t)): S_t of the next block is then issued as soon as
// the softmax has read S_t into registers, and runs while the softmax is
// still working on the current block, so a softmax warpgroup never waits for
// the tensor cores between blocks.
//
// Online softmax (explainer "AI基础 | Flash Attention", "Online softmax"):
// each thread keeps its row's running max m and running sum l in registers
// and works in base 2 with the scale folded in (s * scale * log2 e).  FA2's
// first change (fewer non-matmul operations, abstract and wiki article) is
// taken twice over: O is divided by l once, at the end; and the running
// output is rescaled only when the max grows by more than TAU = 8 (a factor
// 256).  Keeping a stale max is exact -- every term of O and l carries the
// same factor 2^-m, which the final division removes -- and bounds each
// probability by 2^8, far inside fp32 and bf16 range.
//
// Masking: the KV loop covers only blocks that intersect some row's visible
// range (fully hidden blocks are never loaded); inside a block, a row that is
// not entirely visible masks element-wise.  The tail beyond N is zero-filled
// by TMA and masked the same way.
//
// Packed (variable-length) batches: a unit addresses its sequence's rows
// through the tensor-row offset of that sequence.  Tiles that run past the
// end of the sequence read the next sequence's rows; those keys are masked
// like any invisible key and those query rows are never stored, so the
// result is the one each sequence would get alone.
#pragma once

#include <math_constants.h>

#include "attn_common.cuh"
#include "philox.cuh"
#include "sm100_ptx.cuh"

namespace fa2 {

struct FwdParams {
  CUtensorMap tm_q, tm_k, tm_v;        // [B,N,H,d] bf16, box {64,1,128,1}, 128B swizzle
                                       // (packed: [1,total,H,d])
  __nv_bfloat16* o;                    // [B,N,H,d] / [total,H,d] output
  long long so_b, so_n, so_h;          // its element strides
  float* lse;                          // [B,H,N] / [H,total]
  const float* alibi;                  // [H] or null
  const int* cu_seqlens;               // [B+1] sequence offsets (packed) or null (padded)
  int total;                           // packed: tensor rows
  int stat_rows;                       // rows per (batch, head) of lse: N or total
  int N, H, B;                         // N: the (longest) sequence length
  int wl, wr;                          // inclusive window, negative = unbounded
  int npairs;                          // ceil(N / 256)
  int num_units;                       // npairs * H * B
  int heavy_first;                     // order units longest-first (masks)
  float scale_log2;                    // softmax_scale * log2(e)
  unsigned long long wait_ns;          // bounded-wait limit
  DropoutParams drop;                  // used by the DROPOUT instantiations
  float o_scale;                       // e4m3 inputs: V's dequantisation factor (else 1)
  unsigned int* sched;                 // packed / block-sparse: {next unit, finished CTAs}, 0 between calls
  const uint8_t* bmask;                // block-sparse: [B, H, nb, nb] 128 x 128 block mask
  long long bm_sb, bm_sh;              // its batch and head strides (elements)
  int nb;                              // ceil(N / 128): blocks per row and column of the mask
  int test_skip;                       // test switch, 0 in normal use: see the softmax's p_ready arrive
};

template <int HD, bool FP8 = false, bool MASK_EPI = false>
struct FwdCfg {
  static constexpr int BM = 128;        // query rows per tile
  static constexpr int BN = 128;        // keys per KV block
  static constexpr int NQT = 2;         // query tiles per unit
  // MASK_EPI (the dropout kernels): the epilogue warps draw each block's
  // dropout mask into shared memory ahead of the softmax, in a ring of
  // MASK_RING blocks of keep bytes; Q is single-buffered to make room.
  static constexpr int QBUFS = MASK_EPI ? 1 : 2;  // Q buffers (across units)
  static constexpr int ESZ = FP8 ? 1 : 2;                    // bytes per element
  static constexpr int KSTEP = FP8 ? 32 : 16;                // K of one MMA
  static constexpr int SLOTS = FP8 ? 6 : (HD == 128 ? 3 : 8);
  static constexpr int QT_BYTES = BM * HD * ESZ;
  static constexpr int KV_BYTES = BN * HD * ESZ;
  static constexpr int OFF_KV = QBUFS * NQT * QT_BYTES;
  static constexpr int MASK_RING = 2;
  static constexpr int MASK_BYTES = NQT * BM * BN;  // one block's keep bytes, both tiles
  static constexpr int OFF_MASK = OFF_KV + SLOTS * KV_BYTES;
  static constexpr int OFF_BARS = OFF_MASK + (MASK_EPI ? MASK_RING * MASK_BYTES : 0);
  static constexpr int RING = 4;        // unit-index ring of the packed scheduler
  // d = 64 leaves 128 TMEM columns free: P gets its own 64 columns per tile,
  // so the next S product need not wait for the PV product that reads P.
  static constexpr bool PSEP = HD == 64 && !FP8;
  // q_full[2], q_empty[2], slot full/empty, s_full[2], p_ready[2], o_full[2],
  // o_empty[2], drain, ring full[4], ring empty[4], stats_full[2], stats_free[2],
  // s_read[2], p_free[2], mask_full[MASK_RING], mask_empty[MASK_RING]
  static constexpr int NBARS = 4 + 2 * SLOTS + 4 * NQT + 1 + 2 * RING + 4 * NQT + (MASK_EPI ? 2 * MASK_RING : 0);
  // barriers, then the TMEM address, the abort flag, 2 spare words, the ring
  // and the per-row results (1 / l, LSE) the softmax hands to the epilogue
  static constexpr int OFF_STATS = OFF_BARS + NBARS * 8 + 16 + 4 * RING;
  static constexpr int SMEM_BYTES = OFF_STATS + NQT * BM * 8;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static constexpr int THREADS = 512;
  // registers per thread after re-balancing (launch: 128 x 512 = 65536):
  // softmax warpgroups 184, epilogue warpgroup 80, loader / MMA warpgroup 64
  // (d = 64: 200 / 48 / 64 -- none of the roles spills, and the MMA issuer,
  // whose latency from a finished P to the next S product the softmax
  // waits on, measured about 1% faster with 64 than with 56)
  // (d = 64 with the mask ring: 192 / 64 / 64, the epilogue runs the generator)
  static constexpr int REGS_SOFT = HD == 128 ? 184 : (MASK_EPI ? 192 : 200),
                       REGS_EPI = HD == 128 ? 80 : (MASK_EPI ? 64 : 48),
                       REGS_MISC = 64;
  static constexpr int REGS_AT_LAUNCH = (2 * 128 * REGS_SOFT + 128 * REGS_EPI + 128 * REGS_MISC) / 512;
  static_assert(REGS_AT_LAUNCH == 128, "register split must use exactly the launch budget");
};

// The configuration of fa2_fwd_sm100_kernel<HD, ALIBI, DROPOUT, MODE, FP8>:
// the host sizes the launch (shared memory, registers) from the same type.
template <int HD, bool DROPOUT, bool FP8>
using FwdKernelCfg = FwdCfg<HD, FP8, DROPOUT>;

namespace fwd_detail {
constexpr float TAU = 8.0f;
constexpr float LN2 = 0.69314718055994530942f;
constexpr float LOG2E = 1.44269504088896340736f;
// wait-site codes reported through the device status word
constexpr int SITE_PROD = 0x100, SITE_MMA = 0x200, SITE_SOFT = 0x300, SITE_DRAIN = 0x400;
constexpr int SITE_SMEM_ALIGN_F = 0xF01;

// Padded calls: the k-th unit of CTA c in a persistent grid of G CTAs.
// Round k covers units [kG, kG + G) of the longest-first order, walked
// forwards in even rounds and backwards in odd rounds, so each CTA's heavy
// and light units pair up when the work per unit varies (causal and
// sliding-window masks).  With equal sequence lengths this static schedule
// is within a few percent of the best one.
__device__ __forceinline__ int unit_index(int k) {
  const int G = int(gridDim.x), c = int(blockIdx.x);
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}

// Block-mask row of query block qb of head (b, h), or null past the last
// query block.
__device__ __forceinline__ const uint8_t* bm_row(const FwdParams& p, int b, int h, int qb) {
  return qb < p.nb ? p.bmask + b * p.bm_sb + h * p.bm_sh + (long long)qb * p.nb : nullptr;
}
// Does either query tile of a unit (mask rows r0, r1) need key block kb?
__device__ __forceinline__ bool pair_needs(const uint8_t* r0, const uint8_t* r1, int kb) {
  return r0[kb] != 0 || (r1 != nullptr && r1[kb] != 0);
}

// Unit index -> (head, sequence, its rows, first local query row, first and
// last KV block, KV block count).  A unit whose query pair lies past the end
// of its sequence (packed calls: shorter sequences) has nblk = 0.  With a
// block mask, the unit visits only the KV blocks either of its query tiles
// needs (at least one: a unit whose rows see nothing still writes O = 0 and
// LSE = -inf from one fully hidden block).
struct Unit {
  int h, b, bt, base, len, row0, first, last, nblk;
};
template <int MODE>
__device__ __forceinline__ Unit unit_of(const FwdParams& p, int L) {
  constexpr bool PACKED = MODE == kLayoutPacked;
  Unit u;
  const int nhb = p.H * p.B;
  int pair, hb;
  if (p.heavy_first) {
    pair = p.npairs - 1 - L / nhb;
    hb = L % nhb;
  } else {
    pair = L % p.npairs;
    hb = L / p.npairs;
  }
  u.h = hb % p.H;
  u.b = hb / p.H;
  if (PACKED) {
    const SeqView sv = seq_view(p.cu_seqlens, u.b, p.N, p.total);
    u.bt = sv.bt;
    u.base = sv.row0;
    u.len = sv.len;
  } else {
    u.bt = u.b;
    u.base = 0;
    u.len = p.N;
  }
  u.row0 = pair * 256;
  u.first = 0;
  u.last = -1;
  u.nblk = 0;
  if (u.row0 < u.len) {
    const int row_end = min(u.len, u.row0 + 256);
    const int kv_lo = p.wl >= 0 ? max(0, u.row0 - p.wl) : 0;
    const int kv_hi = p.wr >= 0 ? min(u.len - 1, row_end - 1 + p.wr) : u.len - 1;
    u.first = kv_lo / 128;
    u.last = kv_hi / 128;
    u.nblk = u.last - u.first + 1;
    if (MODE == kLayoutSparse) {
      const uint8_t* r0 = bm_row(p, u.b, u.h, 2 * pair);
      const uint8_t* r1 = bm_row(p, u.b, u.h, 2 * pair + 1);
      int cnt = 0, first = -1;
      for (int kb = u.first; kb <= u.last; ++kb)
        if (pair_needs(r0, r1, kb)) {
          if (first < 0) first = kb;
          ++cnt;
        }
      if (cnt > 0) {
        u.first = first;
        u.nblk = cnt;
      } else {
        u.nblk = 1;
      }
    }
  }
  return u;
}

// The KV block a unit visits after block kb.
template <int MODE>
__device__ __forceinline__ int next_block(const FwdParams& p, const Unit& u, int kb) {
  if (MODE != kLayoutSparse) return kb + 1;
  const int pair = u.row0 / 256;
  const uint8_t* r0 = bm_row(p, u.b, u.h, 2 * pair);
  const uint8_t* r1 = bm_row(p, u.b, u.h, 2 * pair + 1);
  for (++kb; kb < u.last; ++kb)
    if (pair_needs(r0, r1, kb)) break;
  return kb;
}

// Packed and block-sparse calls: units differ in cost with the sequence
// lengths or the block mask, which a static schedule cannot see, so the CTAs
// take units from a shared counter, each as it becomes free.  Returns the
// next non-empty unit, or -1 when none is left.  Only the producer thread
// calls this.
template <int MODE>
__device__ __forceinline__ int fetch_unit(const FwdParams& p) {
  for (;;) {
    const int L = int(atomicAdd(p.sched, 1u));
    if (L >= p.num_units) return -1;
    if (unit_of<MODE>(p, L).nblk > 0) return L;
  }
}
}  // namespace fwd_detail

// Bounded wait that ignores the CTA abort flag (used to drain in-flight
// asynchronous work before shared/tensor memory is released).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!bar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) {
      atomicCAS(&g_fa2_device_status, 0, fwd_detail::SITE_DRAIN);
      return;
    }
  }
}

template <int HD, bool ALIBI, bool DROPOUT, int MODE, bool FP8 = false>
__global__ void __launch_bounds__(512, 1) fa2_fwd_sm100_kernel(const __grid_constant__ FwdParams p) {
  // with dropout the epilogue warps draw the mask (see FwdCfg)
  constexpr bool MASK_EPI = DROPOUT;
  using C = FwdKernelCfg<HD, DROPOUT, FP8>;
  static_assert(!FP8 || (HD == 128 && !DROPOUT && MODE == kLayoutPadded),
                "e4m3 inputs: d = 128, padded layout, no dropout");
  constexpr int QBUFS = C::QBUFS;
  constexpr bool PACKED = MODE == kLayoutPacked;
  constexpr bool SPARSE = MODE == kLayoutSparse;
  constexpr bool DYN = PACKED || SPARSE;  // units taken from the shared counter
  constexpr int BM = C::BM, BN = C::BN, NQT = C::NQT, SLOTS = C::SLOTS;
  constexpr int NCH = HD * C::ESZ / 128;  // 128-byte boxes per tile row
  constexpr int KSTEP = C::KSTEP;
  // TMEM column of P_t: over S_t, or (separate-P layout) after the O tiles
  constexpr int P_COL = C::PSEP ? 256 + NQT * HD : 0, P_STRIDE = C::PSEP ? BN / 2 : 128;
  static_assert(!C::PSEP || P_COL + NQT * P_STRIDE <= 512, "tensor memory budget");
  using namespace fwd_detail;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // 128-byte-swizzled tiles need 1 KB alignment
    if (threadIdx.x == 0) {
      atomicCAS(&g_fa2_device_status, 0, SITE_SMEM_ALIGN_F);
      if (DYN) sched_cta_done(p.sched);  // takes no unit, but must still count as finished
    }
    return;
  }
  uint8_t* sQ = smem_raw;                   // [QBUFS][NQT] tiles
  uint8_t* sKV = smem_raw + C::OFF_KV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + C::OFF_BARS);
  const uint32_t bar0 = smem_u32(bars);
  auto q_full = [&](int qb) { return bar0 + 8u * qb; };
  auto q_empty = [&](int qb) { return bar0 + 8u * (2 + qb); };
  auto slot_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto slot_empty = [&](int s) { return bar0 + 8u * (4 + SLOTS + s); };
  auto s_full = [&](int t) { return bar0 + 8u * (4 + 2 * SLOTS + t); };
  auto p_ready = [&](int t) { return bar0 + 8u * (6 + 2 * SLOTS + t); };
  auto o_full = [&](int t) { return bar0 + 8u * (8 + 2 * SLOTS + t); };
  auto o_empty = [&](int t) { return bar0 + 8u * (10 + 2 * SLOTS + t); };
  const uint32_t drain_bar = bar0 + 8u * (12 + 2 * SLOTS);
  auto ring_full = [&](int r) { return bar0 + 8u * (13 + 2 * SLOTS + r); };
  auto ring_empty = [&](int r) { return bar0 + 8u * (13 + 2 * SLOTS + C::RING + r); };
  auto stats_full = [&](int t) { return bar0 + 8u * (13 + 2 * SLOTS + 2 * C::RING + t); };
  auto stats_free = [&](int t) { return bar0 + 8u * (15 + 2 * SLOTS + 2 * C::RING + t); };
  // separate-P layout only: S_t has been read into registers / P_t has been read by its PV product
  auto s_read = [&](int t) { return bar0 + 8u * (17 + 2 * SLOTS + 2 * C::RING + t); };
  auto p_free = [&](int t) { return bar0 + 8u * (19 + 2 * SLOTS + 2 * C::RING + t); };
  // MASK_EPI: a block's keep bytes written by the epilogue / read by both softmax warpgroups
  auto mask_full = [&](int m) { return bar0 + 8u * (21 + 2 * SLOTS + 2 * C::RING + m); };
  auto mask_empty = [&](int m) { return bar0 + 8u * (21 + 2 * SLOTS + 2 * C::RING + C::MASK_RING + m); };
  // [MASK_RING][NQT][BN / 16][BM] x 16 keep bytes (keys 16 c .. 16 c + 15 of
  // one row).  Within each 32 rows, row 4 m + w sits in slot 8 w + m, so that
  // the writers (a quad of lanes holds rows 4 m .. 4 m + 3) store to 32
  // different banks and every reader still takes one whole slot.
  uint4* sMask = reinterpret_cast<uint4*>(smem_raw + C::OFF_MASK);
  auto mask_slot = [](int row) { return (row & ~31) | ((row & 3) << 3) | ((row >> 2) & 7); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* ring = abort_flag + 3;  // packed: unit indices handed from the producer to the other roles
  float2* stats = reinterpret_cast<float2*>(smem_raw + C::OFF_STATS);  // [NQT][BM] (1 / l, LSE)
  AbortFlag ab{abort_flag};

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < C::NBARS; ++i) {
      const uint32_t bar = bar0 + 8u * i;
      uint32_t cnt = 1;
      if (bar == p_ready(0) || bar == p_ready(1) || bar == o_empty(0) || bar == o_empty(1)) cnt = 128;
      if (bar == stats_full(0) || bar == stats_full(1) || bar == stats_free(0) || bar == stats_free(1))
        cnt = 128;
      if (bar == s_read(0) || bar == s_read(1)) cnt = 128;
      if (MASK_EPI) {
        for (int m = 0; m < C::MASK_RING; ++m) {
          if (bar == mask_full(m)) cnt = 128;   // the epilogue threads
          if (bar == mask_empty(m)) cnt = 256;  // the softmax threads of both tiles
        }
      }
      // MMA + 8 softmax warps + 4 epilogue warps
      if (bar >= ring_empty(0) && bar <= ring_empty(C::RING - 1)) cnt = 13;
      bar_init(bar, cnt);
    }
    fence_barrier_init();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 12) {
    regs_dec<C::REGS_MISC>();
  if (warp == 12) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int n = 0, k = 0, q_issued = 0;
      bool ok = true;
      int L = DYN ? fetch_unit<MODE>(p) : unit_index(0);
      for (;; ++k) {
        if (DYN) {  // hand the unit index (or the end mark -1) to the other roles
          const int r = k % C::RING;
          if (!wait_bar(ring_empty(r), ((k / C::RING) & 1) ^ 1, ab, p.wait_ns, SITE_PROD + 3)) break;
          ring[r] = L;
          bar_arrive(ring_full(r));
          if (L < 0) break;
        } else if (L >= p.num_units) {
          break;
        }
        const Unit u = unit_of<MODE>(p, L);
        const int L_next = DYN ? fetch_unit<MODE>(p) : unit_index(k + 1);
        const int qb = k % QBUFS;
        if (!wait_bar(q_empty(qb), ((k / QBUFS) & 1) ^ 1, ab, p.wait_ns, SITE_PROD + 2)) break;
        bar_arrive_expect_tx(q_full(qb), NQT * C::QT_BYTES);
        for (int t = 0; t < NQT; ++t)
          for (int c = 0; c < NCH; ++c)
            tma_load_4d(smem_u32(sQ + (qb * NQT + t) * C::QT_BYTES + c * BM * 128), &p.tm_q, q_full(qb),
                        c * (128 / C::ESZ), u.h, u.base + u.row0 + t * BM, u.bt);
        q_issued = k + 1;
        int kb = u.first;
        for (int it = 0; it < u.nblk && ok; ++it, kb = next_block<MODE>(p, u, kb)) {
          const int kv0 = u.base + (SPARSE ? kb : u.first + it) * BN;
          for (int which = 0; which < 2; ++which, ++n) {
            const int s = n % SLOTS;
            if (!wait_bar(slot_empty(s), ((n / SLOTS) & 1) ^ 1, ab, p.wait_ns, SITE_PROD + which)) {
              ok = false;
              break;
            }
            bar_arrive_expect_tx(slot_full(s), C::KV_BYTES);
            const CUtensorMap* tm = which == 0 ? &p.tm_k : &p.tm_v;
            for (int c = 0; c < NCH; ++c)
              tma_load_4d(smem_u32(sKV + s * C::KV_BYTES + c * BN * 128), tm, slot_full(s),
                          c * (128 / C::ESZ), u.h, kv0, u.bt);
          }
        }
        if (!ok) break;
        L = L_next;
      }
      // The last CTA to finish taking units returns the counters to zero.
      if (DYN) sched_cta_done(p.sched);
      // Before the CTA may exit, every copy issued must have landed.
      for (int j = max(0, q_issued - QBUFS); j < q_issued; ++j)
        drain_wait(q_full(j % QBUFS), (j / QBUFS) & 1, p.wait_ns);
      for (int j = (n > SLOTS ? n - SLOTS : 0); j < n; ++j)
        drain_wait(slot_full(j % SLOTS), (j / SLOTS) & 1, p.wait_ns);
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = FP8 ? idesc_e4m3_f32(BM, BN, 0, 0) : idesc_bf16_f32(BM, BN, 0, 0);
      const uint32_t id_pv = FP8 ? idesc_e4m3_f32(BM, HD, 0, 1) : idesc_bf16_f32(BM, HD, 0, 1);
      // One MMA covers KSTEP elements of K = 32 bytes of a 128-byte swizzled
      // row; four of them fill a row, then the next 128-byte box follows.
      auto qk = [&](int t, int qb, int s) {
        const uint32_t a0 = smem_u32(sQ + (qb * NQT + t) * C::QT_BYTES), b0 = smem_u32(sKV + s * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < HD / KSTEP; ++kk) {
          const uint32_t ao = (kk / 4) * (BM * 128) + (kk % 4) * 32;
          const uint32_t bo = (kk / 4) * (BN * 128) + (kk % 4) * 32;
          if (FP8)
            umma_ss_f8(tmem + t * 128, sdesc_sw128(a0 + ao, 16, 1024), sdesc_sw128(b0 + bo, 16, 1024),
                       id_qk, kk > 0);
          else
            umma_ss(tmem + t * 128, sdesc_sw128(a0 + ao, 16, 1024), sdesc_sw128(b0 + bo, 16, 1024),
                    id_qk, kk > 0);
        }
      };
      // P from TMEM (KSTEP keys = 8 columns per MMA), V MN-major: KSTEP key
      // rows of 128 bytes per MMA, 128-byte column chunks BN * 128 apart.
      auto pv = [&](int t, int s, bool acc) {
        const uint32_t v0 = smem_u32(sKV + s * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < BN / KSTEP; ++kk) {
          const uint64_t vd = sdesc_sw128(v0 + kk * KSTEP * 128, BN * 128, 1024);
          if (FP8)
            umma_ts_f8(tmem + 256 + t * HD, tmem + P_COL + t * P_STRIDE + kk * 8, vd, id_pv,
                       (acc || kk > 0) ? 1u : 0u);
          else
            umma_ts(tmem + 256 + t * HD, tmem + P_COL + t * P_STRIDE + kk * 8, vd, id_pv,
                    (acc || kk > 0) ? 1u : 0u);
        }
      };
      if constexpr (DYN || C::PSEP) {
        int n = 0, g = 0;  // KV slots, blocks
        bool ok = true;
        for (int k = 0; ok; ++k) {
          int L;
          if (DYN) {
            const int r = k % C::RING;
            ok = wait_bar(ring_full(r), (k / C::RING) & 1, ab, p.wait_ns, SITE_MMA + 8);
            if (!ok) break;
            L = ring[r];
            bar_arrive(ring_empty(r));
            if (L < 0) break;
          } else {
            L = unit_index(k);
            if (L >= p.num_units) break;
          }
          const Unit u = unit_of<MODE>(p, L);
          const int qb = k % QBUFS;
          ok = wait_bar(q_full(qb), (k / QBUFS) & 1, ab, p.wait_ns, SITE_MMA + 0);
          if (!ok) break;
          if constexpr (C::PSEP) {
            // Step it issues S_t of block it as soon as softmax t has read the
            // previous S_t, then PV_t of block it-1 once P_t is ready: each
            // softmax warpgroup finds its next S finished when it completes a
            // block.  K of block it sits in slot n + 2 it, V in the next one.
            for (int it = 0; it <= u.nblk && ok; ++it) {
              const int gi = g + it;
              const int nk = n + 2 * it, nv = nk - 1;
              if (it < u.nblk) {
                ok = wait_bar(slot_full(nk % SLOTS), (nk / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 1);
                if (!ok) break;
              }
              if (it > 0) {
                ok = wait_bar(slot_full(nv % SLOTS), (nv / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 2);
                if (!ok) break;
              }
              for (int t = 0; t < NQT && ok; ++t) {
                if (it < u.nblk) {
                  if (gi > 0) ok = wait_bar(s_read(t), (gi - 1) & 1, ab, p.wait_ns, SITE_MMA + 9);
                  if (!ok) break;
                  tc_fence_after();
                  qk(t, qb, nk % SLOTS);
                  umma_commit(s_full(t));
                }
                if (it > 0) {
                  ok = wait_bar(p_ready(t), (gi - 1) & 1, ab, p.wait_ns, SITE_MMA + 3);
                  // the first PV of a unit overwrites O_t: the previous unit's
                  // epilogue must have read it
                  if (ok && it == 1 && k > 0) ok = wait_bar(o_empty(t), (k - 1) & 1, ab, p.wait_ns, SITE_MMA + 7);
                  if (!ok) break;
                  tc_fence_after();
                  pv(t, nv % SLOTS, it > 1);
                  umma_commit(p_free(t));
                  if (it == u.nblk) umma_commit(o_full(t));
                }
              }
              if (!ok) break;
              if (it < u.nblk) {
                umma_commit(slot_empty(nk % SLOTS));
                if (it == u.nblk - 1) umma_commit(q_empty(qb));  // the unit's last S products
              }
              if (it > 0) umma_commit(slot_empty(nv % SLOTS));
            }
            if (!ok) break;
            n += 2 * u.nblk;
            g += u.nblk;
            continue;
          }
          {
            const int sk = n % SLOTS;
            ok = wait_bar(slot_full(sk), (n / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 1);
            if (!ok) break;
            tc_fence_after();
            for (int t = 0; t < NQT; ++t) {
              qk(t, qb, sk);
              umma_commit(s_full(t));
            }
            umma_commit(slot_empty(sk));
            if (u.nblk == 1) umma_commit(q_empty(qb));
            ++n;
          }
          for (int it = 1; it < u.nblk && ok; ++it) {
            const int sv = n % SLOTS, sk = (n + 1) % SLOTS;
            ok = wait_bar(slot_full(sv), (n / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 2);
            for (int t = 0; t < NQT && ok; ++t) {
              ok = wait_bar(p_ready(t), (g + it - 1) & 1, ab, p.wait_ns, SITE_MMA + 3);
              // the first PV of a unit overwrites O_t: the previous unit's
              // epilogue must have read it
              if (ok && it == 1 && k > 0) ok = wait_bar(o_empty(t), (k - 1) & 1, ab, p.wait_ns, SITE_MMA + 7);
              if (!ok) break;
              tc_fence_after();
              pv(t, sv, it > 1);
              if (t == 0) {
                ok = wait_bar(slot_full(sk), ((n + 1) / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 4);
                if (!ok) break;
                tc_fence_after();
              }
              qk(t, qb, sk);
              umma_commit(s_full(t));
            }
            if (!ok) break;
            if (it == u.nblk - 1) umma_commit(q_empty(qb));  // the unit's last S products
            umma_commit(slot_empty(sv));
            umma_commit(slot_empty(sk));
            n += 2;
          }
          if (!ok) break;
          {
            const int sv = n % SLOTS;
            ok = wait_bar(slot_full(sv), (n / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 5);
            for (int t = 0; t < NQT && ok; ++t) {
              ok = wait_bar(p_ready(t), (g + u.nblk - 1) & 1, ab, p.wait_ns, SITE_MMA + 6);
              if (ok && u.nblk == 1 && k > 0) ok = wait_bar(o_empty(t), (k - 1) & 1, ab, p.wait_ns, SITE_MMA + 7);
              if (!ok) break;
              tc_fence_after();
              pv(t, sv, u.nblk > 1);
              umma_commit(o_full(t));
            }
            if (ok) umma_commit(slot_empty(sv));
            ++n;
          }
          g += u.nblk;
        }
      } else {
        // Static schedule, P over S: the last block of a unit issues PV_t
        // and at once S_t of the next unit's first block (K in the slot after
        // this unit's last V), so the softmax of tile t does not wait behind
        // both tiles' last PV products at the boundary.  The loader runs a
        // whole unit ahead here; with the shared counter (short units, the
        // next unit known late) the plain order above measured faster.
        auto fetch = [&](int k) -> int {
          const int L = unit_index(k);
          return L >= p.num_units ? -1 : L;
        };
        int n = 0, g = 0;  // KV slots, blocks
        bool ok = true;
        // this unit's first S products went out with the previous unit's last
        // PV products (every unit but the first)
        bool s0_issued = false;
        int L = fetch(0);
        for (int k = 0; ok && L >= 0; ++k) {
          const Unit u = unit_of<MODE>(p, L);
          const int qb = k % QBUFS;
          if (!s0_issued) {
            ok = wait_bar(q_full(qb), (k / QBUFS) & 1, ab, p.wait_ns, SITE_MMA + 0);
            if (!ok) break;
            const int sk = n % SLOTS;
            ok = wait_bar(slot_full(sk), (n / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 1);
            if (!ok) break;
            tc_fence_after();
            for (int t = 0; t < NQT; ++t) {
              qk(t, qb, sk);
              umma_commit(s_full(t));
            }
            umma_commit(slot_empty(sk));
            if (u.nblk == 1) umma_commit(q_empty(qb));
            ++n;
          }
          for (int it = 1; it < u.nblk && ok; ++it) {
            const int sv = n % SLOTS, sk = (n + 1) % SLOTS;
            ok = wait_bar(slot_full(sv), (n / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 2);
            for (int t = 0; t < NQT && ok; ++t) {
              ok = wait_bar(p_ready(t), (g + it - 1) & 1, ab, p.wait_ns, SITE_MMA + 3);
              // the first PV of a unit overwrites O_t: the previous unit's
              // epilogue must have read it
              if (ok && it == 1 && k > 0) ok = wait_bar(o_empty(t), (k - 1) & 1, ab, p.wait_ns, SITE_MMA + 7);
              if (!ok) break;
              tc_fence_after();
              pv(t, sv, it > 1);
              if (t == 0) {
                ok = wait_bar(slot_full(sk), ((n + 1) / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 4);
                if (!ok) break;
                tc_fence_after();
              }
              qk(t, qb, sk);
              umma_commit(s_full(t));
            }
            if (!ok) break;
            if (it == u.nblk - 1) umma_commit(q_empty(qb));  // the unit's last S products
            umma_commit(slot_empty(sv));
            umma_commit(slot_empty(sk));
            n += 2;
          }
          if (!ok) break;
          {  // last block, with the next unit's first S products
            const int sv = n % SLOTS, skn = (n + 1) % SLOTS, qbn = (k + 1) % QBUFS;
            int Ln = -1;
            Unit un{};
            ok = wait_bar(slot_full(sv), (n / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 5);
            for (int t = 0; t < NQT && ok; ++t) {
              ok = wait_bar(p_ready(t), (g + u.nblk - 1) & 1, ab, p.wait_ns, SITE_MMA + 6);
              if (ok && u.nblk == 1 && k > 0) ok = wait_bar(o_empty(t), (k - 1) & 1, ab, p.wait_ns, SITE_MMA + 7);
              if (!ok) break;
              tc_fence_after();
              pv(t, sv, u.nblk > 1);
              umma_commit(o_full(t));
              if (t == 0) {
                Ln = fetch(k + 1);
                if (Ln >= 0) {
                  un = unit_of<MODE>(p, Ln);
                  ok = wait_bar(q_full(qbn), ((k + 1) / QBUFS) & 1, ab, p.wait_ns, SITE_MMA + 0);
                  if (ok) ok = wait_bar(slot_full(skn), ((n + 1) / SLOTS) & 1, ab, p.wait_ns, SITE_MMA + 1);
                  if (ok) tc_fence_after();
                }
                if (!ok) break;
              }
              if (Ln >= 0) {
                qk(t, qbn, skn);
                umma_commit(s_full(t));
              }
            }
            if (!ok) break;
            umma_commit(slot_empty(sv));
            ++n;
            if (Ln >= 0) {
              umma_commit(slot_empty(skn));
              if (un.nblk == 1) umma_commit(q_empty(qbn));
              ++n;
            }
            L = Ln;
            s0_issued = true;
          }
          g += u.nblk;
        }
      }
      // Drain: wait until every MMA issued above has completed.
      umma_commit(drain_bar);
      drain_wait(drain_bar, 0, p.wait_ns);
    }
  }
  } else if (warp >= 8) {
    regs_dec<C::REGS_EPI>();
    // ------------------------------------------------------------ epilogue
    // One thread per TMEM lane (query row) of both tiles: takes the row's
    // 1 / l and LSE from the softmax, reads O_t out of TMEM as soon as its
    // last PV product has landed, releases the TMEM columns and stores the
    // normalised row, while the softmax warps already work on the next unit.
    const int r = (warp % 4) * 32 + lane;
    const uint32_t lane_base = uint32_t((warp % 4) * 32) << 16;
    const float o_mult = DROPOUT ? p.drop.keep_scale : (FP8 ? p.o_scale : 1.f);
    bool ok = true;
    // the output rows of unit u (the k-th unit of this CTA)
    auto store_unit = [&](const Unit& u, int k) -> bool {
      const SeqView sv = PACKED ? seq_view(p.cu_seqlens, u.b, p.N, p.total) : SeqView{u.b, 0, p.N};
      for (int t = 0; t < NQT; ++t) {
        const int i = u.row0 + t * BM + r;  // local query row (>= len for padding rows)
        bool okt = wait_bar(stats_full(t), k & 1, ab, p.wait_ns, SITE_SOFT + 4);
        okt = __all_sync(0xffffffffu, okt);
        if (!okt) return false;
        const float2 st = stats[t * BM + r];  // (1 / l, LSE)
        bar_arrive(stats_free(t));
        okt = wait_bar(o_full(t), k & 1, ab, p.wait_ns, SITE_SOFT + 1);
        okt = __all_sync(0xffffffffu, okt);
        if (!okt) return false;
        tc_fence_after();
        const float inv_l = st.x * o_mult;
        const uint32_t o_addr = tmem + lane_base + 256 + t * HD;
        __nv_bfloat16* orow = p.o + sv.bt * p.so_b + (long long)(sv.row0 + i) * p.so_n + u.h * p.so_h;
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t w32[32];
          tmem_ld32(o_addr + c * 32, w32);
          tmem_ld_wait();
          if (c == HD / 32 - 1) {  // O_t has been read: the next unit may overwrite it
            tc_fence_before();
            bar_arrive(o_empty(t));
          }
          uint32_t w16[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w16[e] = pack_bf16(__uint_as_float(w32[2 * e]) * inv_l, __uint_as_float(w32[2 * e + 1]) * inv_l);
          if (i < sv.len) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              *reinterpret_cast<uint4*>(orow + c * 32 + q4 * 8) =
                  make_uint4(w16[4 * q4], w16[4 * q4 + 1], w16[4 * q4 + 2], w16[4 * q4 + 3]);
          }
        }
        if (i < sv.len) p.lse[(size_t(sv.bt) * p.H + u.h) * (PACKED ? p.stat_rows : p.N) + sv.row0 + i] = st.y;
      }
      return true;
    };
    // MASK_EPI: the keep bytes of block `kv0` (a local key index) of unit u
    // for both tiles, into the next ring entry: the same draws the softmax
    // would make itself.  Lane s of a quad computes the generator call of
    // key group 4 c + s for the quad's four rows (rows 4 (i / 4) .. + 3) and
    // stores the four rows' words itself, so no lane needs the others' words.
    int gm = 0;  // mask blocks written
    auto write_mask = [&](const Unit& u, int kv0) -> bool {
      const int m = gm % C::MASK_RING;
      bool okm = wait_bar(mask_empty(m), ((gm / C::MASK_RING) & 1) ^ 1, ab, p.wait_ns, SITE_SOFT + 7);
      okm = __all_sync(0xffffffffu, okm);
      if (!okm) return false;
      const int s4 = lane & 3;
      // word s4 of the slots of rows 4 (r / 4) + w, w = 0..3 (slot 8 w + r / 4 mod 8)
      uint32_t* dst = reinterpret_cast<uint32_t*>(sMask + m * (C::MASK_BYTES / 16)) +
                      (mask_slot(r & ~3)) * 4 + s4;
      for (int t = 0; t < NQT; ++t) {
        const uint32_t i4 = uint32_t((u.row0 + t * BM + r) >> 2);
#pragma unroll 4
        for (int c = 0; c < BN / 16; ++c) {
          const Philox4 o = philox4x32_10(uint32_t((kv0 >> 2) + 4 * c + s4), i4, uint32_t(u.h), uint32_t(u.b), p.drop);
#pragma unroll
          for (int w = 0; w < 4; ++w)
            dst[((t * (BN / 16) + c) * BM + 8 * w) * 4] = dropout_keep_msb4(o.w[w], p.drop.threshold);
        }
      }
      bar_arrive(mask_full(m));
      ++gm;
      return true;
    };
    Unit prev{};
    int kprev = -1;
    for (int k = 0; ok; ++k) {
      int L;
      if (DYN) {
        const int rr = k % C::RING;
        ok = wait_bar(ring_full(rr), (k / C::RING) & 1, ab, p.wait_ns, SITE_SOFT + 3);
        if (!__all_sync(0xffffffffu, ok)) break;
        L = ring[rr];
        __syncwarp();
        if (lane == 0) bar_arrive(ring_empty(rr));
        if (L < 0) break;
      } else {
        L = unit_index(k);
        if (L >= p.num_units) break;
      }
      const Unit u = unit_of<MODE>(p, L);
      if (MASK_EPI) {
        // The unit's first MASK_RING - 1 mask blocks go out before the
        // previous unit's rows (the softmax starts this unit while they are
        // stored), the rest after them: the previous unit's O must be read
        // out of TMEM before this unit's first PV product, which waits on
        // the softmax, which waits on these masks.
        int kb = u.first, it = 0;
        for (; ok && it < u.nblk && it < C::MASK_RING - 1; ++it, kb = next_block<MODE>(p, u, kb))
          ok = write_mask(u, (SPARSE ? kb : u.first + it) * BN);
        if (ok && kprev >= 0) ok = store_unit(prev, kprev);
        for (; ok && it < u.nblk; ++it, kb = next_block<MODE>(p, u, kb))
          ok = write_mask(u, (SPARSE ? kb : u.first + it) * BN);
        prev = u;
        kprev = k;
      } else {
        ok = store_unit(u, k);
      }
    }
    if (MASK_EPI && ok && kprev >= 0) store_unit(prev, kprev);
  } else {
    regs_inc<C::REGS_SOFT>();
    // ------------------------------------------------------------ softmax
    const int t = warp / 4;
    const int r = (warp % 4) * 32 + lane;
    const uint32_t lane_base = uint32_t((warp % 4) * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + t * 128;
    const uint32_t p_addr = tmem + lane_base + P_COL + t * P_STRIDE;
    const uint32_t o_addr = tmem + lane_base + 256 + t * HD;
    const float C2 = p.scale_log2;
    int g = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int L;
      if (DYN) {
        const int r = k % C::RING;
        ok = wait_bar(ring_full(r), (k / C::RING) & 1, ab, p.wait_ns, SITE_SOFT + 2);
        if (!__all_sync(0xffffffffu, ok)) break;
        L = ring[r];
        __syncwarp();
        if (lane == 0) bar_arrive(ring_empty(r));
        if (L < 0) break;
      } else {
        L = unit_index(k);
        if (L >= p.num_units) break;
      }
      const Unit u = unit_of<MODE>(p, L);
      const int h = u.h, b = u.b;
      // this tile's block-mask row (null: tile past the last query block)
      const uint8_t* mrow = SPARSE ? bm_row(p, b, h, u.row0 / 128 + t) : nullptr;
      const int i = u.row0 + t * BM + r;  // local query row (>= len for padding rows)
      const int lo = p.wl >= 0 ? max(0, i - p.wl) : 0;
      const int hi = p.wr >= 0 ? min(u.len - 1, i + p.wr) : u.len - 1;
      float slope2 = 0.f;
      if (ALIBI) slope2 = -p.alibi[h] * LOG2E;
      float m_run = -CUDART_INF_F, l_run = 0.f;
      int kb = u.first;
      for (int it = 0; it < u.nblk; ++it, kb = next_block<MODE>(p, u, kb)) {
        const int kv0 = (SPARSE ? kb : u.first + it) * BN;
        // block hidden from this tile by the block mask (it is visited for
        // the other tile of the pair, or to write a fully hidden unit)
        const bool hidden = SPARSE && (mrow == nullptr || mrow[kb] == 0);
        ok = wait_bar(s_full(t), (g + it) & 1, ab, p.wait_ns, SITE_SOFT + 0);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float s[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t w32[32];
          tmem_ld32(s_addr + c * 32, w32);
#pragma unroll
          for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(w32[e]);
        }
        tmem_ld_wait();
        if (C::PSEP) {  // S_t is in registers: its columns may take the next block's S
          tc_fence_before();
          bar_arrive(s_read(t));
        }
        if (ALIBI) {
          const float fi = float(i - kv0);
#pragma unroll
          for (int c = 0; c < BN; ++c) s[c] = fmaf(slope2, fabsf(fi - float(c)), s[c] * C2);
        }
        if (hidden || !(kv0 >= lo && kv0 + BN - 1 <= hi)) {
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            const int j = kv0 + c;
            if (hidden || j < lo || j > hi) s[c] = -CUDART_INF_F;
          }
        }
        // Row maximum: four independent chains of three-input maxima.
        float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[2], s[3]);
        float mx2 = fmaxf(s[4], s[5]), mx3 = fmaxf(s[6], s[7]);
#pragma unroll
        for (int c = 8; c < BN; c += 8) {
          mx0 = max3(mx0, s[c], s[c + 1]);
          mx1 = max3(mx1, s[c + 2], s[c + 3]);
          mx2 = max3(mx2, s[c + 4], s[c + 5]);
          mx3 = max3(mx3, s[c + 6], s[c + 7]);
        }
        float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        if (!ALIBI) mx *= C2;  // now in base-2 units
        const bool resc = mx > m_run + TAU;
        float alpha = 1.f;
        if (resc) {
          alpha = ex2(m_run - mx);  // 0 when m_run is -inf
          m_run = mx;
        }
        const float m_use = m_run == -CUDART_INF_F ? 0.f : m_run;
        // Exponentials, with the scale-and-shift and the row sum done on
        // pairs of scores (one paired instruction for two).
        const uint64_t c2x2 = pk2(ALIBI ? 1.f : C2, ALIBI ? 1.f : C2);
        const uint64_t negm2 = pk2(-m_use, -m_use);
        uint64_t l2x[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          float x0, x1;
          upk2(fma2(pk2(s[c], s[c + 1]), c2x2, negm2), x0, x1);
          s[c] = ex2(x0);
          s[c + 1] = ex2(x1);
          l2x[(c / 2) % 4] = add2(l2x[(c / 2) % 4], pk2(s[c], s[c + 1]));
        }
        float la, lb, lc, ld;
        upk2(add2(l2x[0], l2x[1]), la, lb);
        upk2(add2(l2x[2], l2x[3]), lc, ld);
        l_run = fmaf(l_run, alpha, (la + lb) + (lc + ld));
        if (C::PSEP && g + it > 0) {
          // P_t and O_t are free once the previous block's PV product is done
          ok = wait_bar(p_free(t), (g + it - 1) & 1, ab, p.wait_ns, SITE_SOFT + 6);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
        }
        // P (bf16 pairs) over the first BN/2 columns of S.  With dropout, l
        // keeps the un-dropped sum and dropped probabilities leave P here: the
        // epilogue warps have drawn the keep bits (bit 7 of each key's byte)
        // into shared memory, and each pair's two bits become 16-bit masks by
        // sign-replicating byte permutes.
        const uint4* mask_row = nullptr;
        if (MASK_EPI) {
          const int gb = g + it;
          ok = wait_bar(mask_full(gb % C::MASK_RING), (gb / C::MASK_RING) & 1, ab, p.wait_ns, SITE_SOFT + 8);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          mask_row = sMask + (gb % C::MASK_RING) * (C::MASK_BYTES / 16) + t * (BN / 16) * BM + mask_slot(r);
        }
        if (FP8) {
          // e4m3 P: four per column, 32 columns.  P <= 2^TAU = 256 < 448.
#pragma unroll
          for (int c = 0; c < BN / 64; ++c) {
            uint32_t w16[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              w16[e] = pack_e4m3x4(s[c * 64 + 4 * e], s[c * 64 + 4 * e + 1], s[c * 64 + 4 * e + 2],
                                   s[c * 64 + 4 * e + 3]);
            tmem_st16(p_addr + c * 16, w16);
          }
        }
#pragma unroll
        for (int c = 0; c < (FP8 ? 0 : BN / 32); ++c) {
          uint32_t w16[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) w16[e] = pack_bf16(s[c * 32 + 2 * e], s[c * 32 + 2 * e + 1]);
          if (DROPOUT) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              // keep bits of keys kv0 + 32 c + 16 half + 4 g4 .. + 3, as bit 7 of each byte
              const uint4 w = mask_row[(2 * c + half) * BM];
              const uint32_t km[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int g4 = 0; g4 < 4; ++g4) {
                w16[8 * half + 2 * g4] &= prmt(km[g4], 0u, 0x9988);
                w16[8 * half + 2 * g4 + 1] &= prmt(km[g4], 0u, 0xBBAA);
              }
            }
          }
          tmem_st16(p_addr + c * 16, w16);
        }
        if (MASK_EPI) bar_arrive(mask_empty((g + it) % C::MASK_RING));  // its keep bytes are read
        // Rescale the running output (the PV product of the previous block has
        // completed: S_t of this block was committed after it, or, with the
        // separate-P layout, p_free said so).
        if (it > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t w32[32];
            tmem_ld32(o_addr + c * 32, w32);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) w32[e] = __float_as_uint(__uint_as_float(w32[e]) * alpha);
            tmem_st32(o_addr + c * 32, w32);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        // Test switch (off in normal use): the CTA that takes unit 0 (its
        // first unit, whichever schedule) withholds tile 0's arrive on the
        // first block, so the MMA warp's bounded wait for it runs out and
        // every role of that CTA winds down through the abort path.
        if (!(p.test_skip && L == 0 && it == 0 && t == 0)) bar_arrive(p_ready(t));
      }
      if (!ok) break;
      // ------------------------------------ hand the row's results over
      // (the epilogue warps normalise and store O; this buffer is reused
      // once they have read it)
      ok = wait_bar(stats_free(t), (k & 1) ^ 1, ab, p.wait_ns, SITE_SOFT + 5);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      stats[t * BM + r] = make_float2(l_run > 0.f ? 1.f / l_run : 0.f,
                                      l_run > 0.f ? (m_run + log2f(l_run)) * LN2 : -CUDART_INF_F);
      bar_arrive(stats_full(t));
      g += u.nblk;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa2
