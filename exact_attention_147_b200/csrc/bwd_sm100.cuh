// Backward pass of exact attention on sm_100a tensor cores (tcgen05 + TMEM).
//
// The probabilities are recomputed from Q, K and the forward's per-row
// log-sum-exp instead of being stored (explainer "AI基础 | Flash Attention",
// "Backward pass": only O(N) statistics are kept and the scores are rebuilt
// on chip).  With L = sum(O o dO), D_i = sum_c dO_ic O_ic and scale c:
//     P  = exp(c S - LSE),   dV = P^T dO,   dP = dO V^T,
//     dS = P o (dP - D),     dK = c dS^T Q,  dQ = c dS K.
//
// Kernel 1, fa2_bwd_dkdv_sm100_kernel: parallel over 128-key blocks of each
// (batch, head) (FlashAttention-2 abstract: work split across thread blocks
// even within a head); a persistent grid of one CTA per SM walks these key
// blocks.  K_j and V_j stay in shared memory; the query blocks that see them
// stream through a TMA ring.  Per query block, with keys on the TMEM lanes:
//     S^T  = K Q^T          (tcgen05, SS)       -> TMEM [0,128)
//     dP^T = V dO^T         (tcgen05, SS)       -> TMEM [128,256)
//     P^T  = exp2(S^T c log2e - LSE log2e)       (compute warps, -> bf16 over S^T)
//     dV  += P^T dO         (tcgen05, A from TMEM)
//     dS^T = P^T o (dP^T - D)                    (compute warps, -> bf16 over dP^T
//                                                 and to shared memory)
//     dK  += dS^T Q         (tcgen05, A from TMEM)
//     dQ_i = dS K           (tcgen05, A = dS from shared memory, MN-major)
//                           -> TMEM [128,128+d), added into an fp32 dQ
//                              accumulator in global memory with TMA bulk
//                              reductions (order of the adds is not fixed).
// With `deterministic`, kernel 1 skips dQ and kernel 2 produces it.
//
// Kernel 2, fa2_bwd_dq_sm100_kernel: one CTA per 128-query block; it walks
// the visible key blocks in ascending order, recomputes S, P, dP, dS with
// queries on the TMEM lanes and accumulates dQ += dS K in TMEM, so every
// element of dQ is summed in the same order on every run.
//
// Warp roles (both kernels): a TMA producer warp, a single-thread MMA issuer
// warp and a compute warpgroup (one TMEM lane = one row per thread); kernel 1
// adds a warpgroup that drains dQ from TMEM into global memory.
#pragma once

#include <math_constants.h>

#include "attn_common.cuh"
#include "fwd_sm100.cuh"
#include "philox.cuh"
#include "sm100_ptx.cuh"

namespace fa2 {

struct BwdParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;   // inputs, box {64,1,128,1} (packed: [1,total,H,d])
  CUtensorMap tm_dq, tm_dk, tm_dv;       // outputs (bf16), same boxes
  CUtensorMap tm_dqacc;                  // fp32 [B*H, N, d] / [H, total, d] accumulator, box {32,32,1}
  __nv_bfloat16 *dq, *dk, *dv;           // the outputs again, for row-wise stores of
  Strides sdq, sdk, sdv;                 // tiles that end past a packed sequence
  const float* lse;                      // [B,H,N] / [H,total]
  const float* dvec;                     // same layout
  float* dq_accum;                       // fp32 accumulator (kernel 1 with dQ)
  const float* alibi;                    // [H] or null
  const int* cu_seqlens;                 // [B+1] sequence offsets (packed) or null (padded)
  int total;                             // packed: tensor rows
  int stat_rows;                         // rows per (batch, head) of lse / D: N or total
  const uint8_t* bmask;                  // block-sparse: [B, H, nb, nb] 128 x 128 block mask
  long long bm_sb, bm_sh;                // its batch and head strides (elements)
  int nb;                                // ceil(N / 128)
  int N, H, B;                           // N: the (longest) sequence length
  int wl, wr;
  int nblocks;                           // ceil(N / 128)
  float scale;                           // softmax scale c
  float scale_log2;                      // c * log2(e)
  unsigned long long wait_ns;
  DropoutParams drop;                    // used by the DROPOUT instantiations
  int num_items;                         // key blocks x heads x batch (kernel 1 work items)
  unsigned int* sched;                   // packed / block-sparse kernel 1: {next item, finished CTAs}
  uint32_t* dq_chain;                    // ordered dQ: [2, B*H, nblocks, 4] counters (zero at launch)
  int test_skip;                         // test switch, 0 in normal use: see kernel 1's ds_ready arrive
};

template <int HD>
struct BwdCfg {
  static constexpr int TILE = 128 * HD * 2;          // one 128-row bf16 tile
  static constexpr int Q_STAGES = 2;
  static constexpr int DO_STAGES = HD == 128 ? 1 : 2;
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int SIDE_BYTES = 2 * 128 * 4;     // lse2 and D of one query block
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;
  static constexpr int OFF_DO = OFF_Q + Q_STAGES * TILE;
  static constexpr int OFF_DS = OFF_DO + DO_STAGES * TILE;
  static constexpr int OFF_SIDE = OFF_DS + DS_BYTES;
  static constexpr int OFF_STG = OFF_SIDE + Q_STAGES * SIDE_BYTES;  // dQ staging ring
  static constexpr int STG_BYTES = 2 * 16384;                         // 2 x (128 rows x 32 fp32)
  // d = 64 has room for a second K, V pair: the next item's K and V load
  // while the current item runs (d = 128 fills shared memory with one pair)
  static constexpr int KV_BUFS = HD == 64 ? 2 : 1;
  static constexpr int OFF_KV2 = OFF_STG + STG_BYTES;
  static constexpr int OFF_BARS = OFF_KV2 + (KV_BUFS - 1) * 2 * TILE;
  static constexpr int RING = 4;                      // item-index ring (packed / block-sparse)
  // kv_full, Q full/empty, dO full/empty, s_full, dp_full, p_ready, ds_ready,
  // dq_full, dq_free, acc_full, drain, kv_empty, acc_empty, ring full/empty,
  // then kv_full / kv_empty of the second K, V pair
  static constexpr int NBARS = 1 + 2 * Q_STAGES + 2 * DO_STAGES + 8 + 2 + 2 * RING + 2 * (KV_BUFS - 1);
  // No alignment slack: the kernel checks that the dynamic shared memory
  // starts on a 1024-byte boundary (it does: the reserved 1 KB precedes it).
  // barriers, then the TMEM address, the abort flag, 2 spare words, the ring
  static constexpr int SMEM_BYTES = OFF_BARS + NBARS * 8 + 16 + 4 * RING;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static constexpr int THREADS = 512;
  // registers per thread after the warpgroup re-balancing (see kernel 1)
  static constexpr int REGS_COMPUTE = 136, REGS_DRAIN = 136, REGS_MISC = 104;
  static constexpr int REGS_AT_LAUNCH = (2 * 128 * REGS_COMPUTE + 128 * REGS_DRAIN + 128 * REGS_MISC) / 512;
  static_assert(REGS_AT_LAUNCH == 128, "register split must use exactly the launch budget");
};

template <int HD>
struct DqCfg {
  static constexpr int TILE = 128 * HD * 2;
  static constexpr int SLOTS = HD == 128 ? 4 : 8;    // K/V ring
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE;
  static constexpr int OFF_KV = 2 * TILE;
  static constexpr int OFF_BARS = OFF_KV + SLOTS * TILE;
  static constexpr int NBARS = 1 + 2 * SLOTS + 5;
  static constexpr int SMEM_BYTES = OFF_BARS + NBARS * 8 + 16 + 1024;
  static constexpr int THREADS = 192;
};

namespace bwd_detail {
constexpr float LOG2E = 1.44269504088896340736f;
constexpr int SITE_BPROD = 0x500, SITE_BMMA = 0x600, SITE_BCOMP = 0x700, SITE_BRED = 0x800;
constexpr int SITE_QPROD = 0x900, SITE_QMMA = 0xA00, SITE_QCOMP = 0xB00;
constexpr int SITE_SMEM_ALIGN = 0xF00;

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// Writes 16 packed bf16x2 words (32 columns starting at column `col0`) of
// row `row` into a 128-byte-swizzled tile of 128 rows x (64-column boxes).
__device__ __forceinline__ void st_sw128_row32(uint8_t* tile, int row, int col0,
                                               const uint32_t (&w)[16]) {
  const int box = col0 / 64;
  const int u0 = (col0 % 64) / 8;
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    uint8_t* dst = tile + box * (128 * 128) + row * 128 + (((u0 + q4) ^ (row & 7)) * 16);
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
  }
}

// Block-sparse iteration: the first index after x, up to `last`, whose mask
// byte m[index * stride] is set (`last` itself when none before it is).
__device__ __forceinline__ int next_kept(const uint8_t* m, long long stride, int x, int last) {
  for (++x; x < last; ++x)
    if (m[x * stride] != 0) break;
  return x;
}

// Kept blocks among [first, last] of a mask line: sets first to the first
// kept one and returns their count, or leaves first alone and returns 1 when
// none is kept (the kernel then visits one fully hidden block, which writes
// zero gradients).
__device__ __forceinline__ int count_kept(const uint8_t* m, long long stride, int& first, int last) {
  int cnt = 0, f = -1;
  for (int x = first; x <= last; ++x)
    if (m[x * stride] != 0) {
      if (f < 0) f = x;
      ++cnt;
    }
  if (cnt == 0) return 1;
  first = f;
  return cnt;
}

// One work item of kernel 1: a 128-key block of one (batch, head), and the
// query blocks it visits ([qb_first, qb_last], only the kept ones with a
// block mask; nq of them).  An item past the end of a shorter packed
// sequence is empty.
struct BItem {
  int h, b, kb, k0, len, bt, trow, qb_first, qb_last, nq;
  const uint8_t* mcol;  // block-sparse: this key block's mask column (mcol[qb * nb])
  size_t head_off;      // row statistics of local row 0
  bool empty;
};

template <int MODE, bool ORDER = false>
__device__ __forceinline__ BItem item_of(const BwdParams& p, int I) {
  BItem it;
  // Key blocks of one head together, masked or not: they share the head's
  // Q and dO in L2.  (Ordering all heads' block 0 first, the longest-first
  // order for causal masks, ran 148 heads at once and lost 20 % to L2
  // misses.)  The ordered-dQ kernel takes a head's key blocks last first
  // (see its dQ drain).
  it.kb = ORDER ? p.nblocks - 1 - I % p.nblocks : I % p.nblocks;
  const int hb = I / p.nblocks;
  it.h = hb % p.H;
  it.b = hb / p.H;
  const SeqView sv = MODE == kLayoutPacked ? seq_view(p.cu_seqlens, it.b, p.N, p.total)
                                           : SeqView{it.b, 0, p.N};
  it.len = sv.len;
  it.bt = sv.bt;
  it.trow = sv.row0;
  it.k0 = it.kb * 128;
  it.empty = it.k0 >= it.len;
  it.mcol = nullptr;
  it.qb_first = 0;
  it.qb_last = -1;
  it.nq = 0;
  it.head_off = (size_t(sv.bt) * p.H + it.h) * (MODE == kLayoutPacked ? p.stat_rows : p.N) + sv.row0;
  if (!it.empty) {
    const int k_last = min(it.len - 1, it.k0 + 127);
    const int i_lo = p.wr >= 0 ? max(0, it.k0 - p.wr) : 0;
    const int i_hi = p.wl >= 0 ? min(it.len - 1, k_last + p.wl) : it.len - 1;
    it.qb_first = i_lo / 128;
    it.qb_last = i_hi / 128;
    if (MODE == kLayoutSparse) {
      it.mcol = p.bmask + it.b * p.bm_sb + it.h * p.bm_sh + it.kb;
      it.nq = count_kept(it.mcol, p.nb, it.qb_first, it.qb_last);
    } else {
      it.nq = it.qb_last - it.qb_first + 1;
    }
  }
  return it;
}

// The query block a work item visits after block qb.
template <int MODE>
__device__ __forceinline__ int next_qblock(const BwdParams& p, const BItem& it, int qb) {
  return MODE == kLayoutSparse ? next_kept(it.mcol, p.nb, qb, it.qb_last) : qb + 1;
}

// Static schedule of kernel 1 (padded calls, except causal ones with 128 or
// more key blocks): the k-th item of CTA c in a persistent grid of G CTAs, a
// snake over the item order.
__device__ __forceinline__ int bwd_item_index(int k) {
  const int G = int(gridDim.x), c = int(blockIdx.x);
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}

// Packed and block-sparse calls, and long causal padded calls: items taken
// from a shared counter as CTAs become free (their cost follows the lengths,
// the mask or the key block's place under the causal mask).  Next non-empty
// item, or -1.  Only the producer thread calls this.
template <int MODE, bool ORDER = false>
__device__ __forceinline__ int fetch_item(const BwdParams& p) {
  for (;;) {
    const int I = int(atomicAdd(p.sched, 1u));
    if (I >= p.num_items) return -1;
    if (!item_of<MODE, ORDER>(p, I).empty) return I;
  }
}

// Writes the same 16 words straight to row `row` of a global bf16 tensor
// (columns col0 .. col0 + 31).
__device__ __forceinline__ void st_global_row32(__nv_bfloat16* base, const Strides& s, const SeqView& v,
                                                int row, int h, int col0, const uint32_t (&w)[16]) {
  __nv_bfloat16* dst = row_ptr<__nv_bfloat16>(base, s, v, row, h) + col0;
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4)
    reinterpret_cast<uint4*>(dst)[q4] = make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
}
}  // namespace bwd_detail

// ---------------------------------------------------------------------------
// Kernel 1: dK, dV (and the atomically accumulated dQ when WITH_DQ)
//
// Persistent: one CTA per SM walks work items (a 128-key block of one head),
// so barriers, TMEM and registers are set up once and one item's tail
// overlaps the next one's start: the MMA warp releases K and V as soon as
// the item's last products have read them and the loader brings the next
// item's K and V while the compute warps write dK and dV out of TMEM.
//
// 16 warps: warpgroups 0 and 1 compute (thread = key row; warpgroup w owns
// query columns [64w, 64w+64) of every S^T / dP^T tile), warpgroup 2 drains
// dQ (thread = query row), warp 12 loads, warp 13 issues the MMAs.  Register
// budget after the split: compute 136, drain 136, loader/MMA warpgroup 104
// (the loader and the MMA warp follow their own item schedule) (2*128*136 +
// 128*136 + 128*104 = 65536 = 512 threads x 128 at launch; the host checks
// the launch register count before every launch).
//
// dQ path: the drain warpgroup reads the whole dQ tile out of TMEM into
// registers, releases the TMEM columns (the next dP^T reuses them), then
// stages it 32 columns at a time through a two-slot shared-memory ring and
// adds it into the fp32 accumulator with TMA bulk reductions, which go
// through the TMA unit rather than the load/store queues.
//
// Barrier phases run on two counters kept identically by every role: jn,
// the items this CTA has processed (kv_full / kv_empty / acc_full /
// acc_empty), and g, the query blocks it has processed (the Q / dO rings
// and the per-block barriers).
// ---------------------------------------------------------------------------
// DSCHED: padded calls whose items differ in cost (a causal mask over many
// key blocks) also take their items from the shared counter.
// ORDER: deterministic dQ under a causal mask (padded layout, with DSCHED):
// the partial dQ tiles of a query block are added in a fixed order (see the
// dQ drain), so dq is bitwise repeatable without a second pass.
template <int HD, bool ALIBI, bool WITH_DQ, bool DROPOUT, int MODE, bool DSCHED = false, bool ORDER = false>
__global__ void __launch_bounds__(512, 1) fa2_bwd_dkdv_sm100_kernel(const __grid_constant__ BwdParams p) {
  static_assert(!ORDER || (WITH_DQ && DSCHED && MODE == kLayoutPadded), "ordered dQ: padded, counter-scheduled");
  using C = BwdCfg<HD>;
  constexpr bool PACKED = MODE == kLayoutPacked;
  constexpr bool SPARSE = MODE == kLayoutSparse;
  constexpr bool DYN = PACKED || SPARSE || DSCHED;  // items taken from the shared counter
  // K, V pairs in use: the counter-scheduled calls keep one, so that a CTA
  // claims its next item only once its current item's K and V are free (a
  // second pair let CTAs claim a whole item earlier, which unbalanced the
  // end of long causal calls: d = 64, N = 16384, -8%)
  constexpr int KVB = DYN ? 1 : C::KV_BUFS;
  using namespace bwd_detail;
  constexpr int QS = C::Q_STAGES, DS = C::DO_STAGES;
  // Register split.  The ordered dQ's drain holds a whole 128-column fp32
  // tile and the chain state, so (without a dropout mask in the compute
  // warps, which need their registers then) it takes 16 registers from the
  // compute warpgroups: 128 / 152 / 104, no spills.
  constexpr bool DRAIN_HEAVY = ORDER && !DROPOUT;
  constexpr int REGS_CMP = DRAIN_HEAVY ? C::REGS_COMPUTE - 8 : C::REGS_COMPUTE;
  constexpr int REGS_DRN = DRAIN_HEAVY ? C::REGS_DRAIN + 16 : C::REGS_DRAIN;
  static_assert(2 * 128 * REGS_CMP + 128 * REGS_DRN + 128 * C::REGS_MISC == 512 * C::REGS_AT_LAUNCH,
                "register split must use exactly the launch budget");
  constexpr int NCH = HD / 64;
  constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + HD;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // 128-byte-swizzled tiles need 1 KB alignment
    if (threadIdx.x == 0) {
      atomicCAS(&g_fa2_device_status, 0, SITE_SMEM_ALIGN);
      if (DYN) sched_cta_done(p.sched);  // takes no item, but must still count as finished
    }
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sDO = smem + C::OFF_DO;
  uint8_t* sDS = smem + C::OFF_DS;
  uint8_t* sStg = smem + C::OFF_STG;
  float* sSide = reinterpret_cast<float*>(smem + C::OFF_SIDE);  // [QS][2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BARS);
  const uint32_t b0 = smem_u32(bars);
  auto q_full = [&](int s) { return b0 + 8u * (1 + s); };
  auto q_empty = [&](int s) { return b0 + 8u * (1 + QS + s); };
  auto do_full = [&](int s) { return b0 + 8u * (1 + 2 * QS + s); };
  auto do_empty = [&](int s) { return b0 + 8u * (1 + 2 * QS + DS + s); };
  const uint32_t s_full = b0 + 8u * (1 + 2 * QS + 2 * DS);
  const uint32_t dp_full = s_full + 8, p_ready = s_full + 16, ds_ready = s_full + 24;
  const uint32_t dq_full = s_full + 32, dq_free = s_full + 40, acc_full = s_full + 48;
  const uint32_t drain_bar = s_full + 56;
  const uint32_t acc_empty = s_full + 72;
  // K, V buffer pair b and its barriers (pair 1 after the ring's barriers)
  auto kv_full = [&](int b) { return b == 0 ? b0 : s_full + 80 + 16u * C::RING; };
  auto kv_empty = [&](int b) { return b == 0 ? s_full + 64 : s_full + 88 + 16u * C::RING; };
  auto kv_k = [&](int b) { return b == 0 ? sK : smem + C::OFF_KV2; };
  auto kv_v = [&](int b) { return b == 0 ? sV : smem + C::OFF_KV2 + C::TILE; };
  auto ring_full = [&](int r) { return s_full + 80 + 8u * r; };
  auto ring_empty = [&](int r) { return s_full + 80 + 8u * (C::RING + r); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* ring = abort_flag + 3;  // item indices handed from the loader to the other roles
  AbortFlag ab{abort_flag};

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int wg = warp / 4;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < C::NBARS; ++i) {
      const uint32_t bar = b0 + 8u * i;
      uint32_t cnt = 1;
      if (bar == p_ready || bar == ds_ready || bar == acc_empty) cnt = 256;
      if (bar == dq_free) cnt = 128;
      // MMA thread + 8 compute warps + 4 drain warps
      if (bar >= ring_empty(0) && bar <= ring_empty(C::RING - 1)) cnt = 13;
      bar_init(bar, cnt);
    }
    fence_barrier_init();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // The next item of a consumer role (MMA, compute, drain): the ring entry
  // the loader published (DYN), or the static schedule; -1 at the end.
  // `k` counts the schedule entries this role has looked at.  Returns false
  // when a wait gave up.
  auto next_item = [&](int& k, int& I, bool warp_wide, int site) -> bool {
    for (;;) {
      if (DYN) {
        const int rr = k % C::RING;
        bool ok = wait_bar(ring_full(rr), (k / C::RING) & 1, ab, p.wait_ns, site);
        if (warp_wide) ok = __all_sync(0xffffffffu, ok);
        if (!ok) return false;
        I = ring[rr];
        if (warp_wide) __syncwarp();
        if (!warp_wide || lane == 0) bar_arrive(ring_empty(rr));
        ++k;
        return true;  // the loader publishes only non-empty items, then -1
      }
      I = bwd_item_index(k++);
      if (I >= p.num_items) {
        I = -1;
        return true;
      }
      if (!item_of<MODE, ORDER>(p, I).empty) return true;
    }
  };

  if (wg == 3) {
    regs_dec<C::REGS_MISC>();
    if (warp == 12) {
      // ---------------------------------------------------------- producer
      int issued_q = 0, issued_do = 0, issued_kv = 0, jn = 0, g = 0, k = 0;
      bool ok = true;
      int I = DYN ? (lane == 0 ? fetch_item<MODE, ORDER>(p) : 0) : -1;
      if (DYN) I = __shfl_sync(0xffffffffu, I, 0);
      for (;;) {
        if (DYN) {  // publish the item (or the end mark -1) to the other roles
          const int rr = k % C::RING;
          ok = wait_bar(ring_empty(rr), ((k / C::RING) & 1) ^ 1, ab, p.wait_ns, SITE_BPROD + 3);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          if (lane == 0) {
            ring[rr] = I;
            bar_arrive(ring_full(rr));
          }
          ++k;
          if (I < 0) break;
        } else {
          for (;;) {  // the static schedule, skipping empty items
            I = bwd_item_index(k++);
            if (I >= p.num_items || !item_of<MODE, ORDER>(p, I).empty) break;
          }
          if (I >= p.num_items) break;
        }
        const BItem itm = item_of<MODE, ORDER>(p, I);
        int I_next = 0;
        // K and V of this item once the products of the item that last used
        // this buffer pair have read them
        const int kvb = jn % KVB;
        ok = wait_bar(kv_empty(kvb), ((jn / KVB) & 1) ^ 1, ab, p.wait_ns, SITE_BPROD + 2);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (lane == 0) {
          bar_arrive_expect_tx(kv_full(kvb), 2 * C::TILE);
          for (int c = 0; c < NCH; ++c) {
            tma_load_4d(smem_u32(kv_k(kvb) + c * 16384), &p.tm_k, kv_full(kvb), c * 64, itm.h,
                        itm.trow + itm.k0, itm.bt);
            tma_load_4d(smem_u32(kv_v(kvb) + c * 16384), &p.tm_v, kv_full(kvb), c * 64, itm.h,
                        itm.trow + itm.k0, itm.bt);
          }
        }
        ++issued_kv;
        // the next item's index: the atomic is in flight while this item
        // loads.  (The ordered dQ claims its next item only once this item's
        // loads are out, about one query block before it can start: claims
        // must start in the order they were made, see the dQ drain.)
        if (DYN && !ORDER && lane == 0) I_next = fetch_item<MODE, ORDER>(p);
        int qb = itm.qb_first;
        for (int it = 0; it < itm.nq && ok; ++it, qb = next_qblock<MODE>(p, itm, qb)) {
          const int gi = g + it;
          const int i0 = (SPARSE ? qb : itm.qb_first + it) * 128;
          const int sq = gi % QS;
          // log2-scaled LSE and D of this query block, +inf / 0 past the end;
          // loaded before waiting for the slot so the latency overlaps the wait
          float l2v[4], dvv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = i0 + lane + 32 * e;
            l2v[e] = CUDART_INF_F;
            dvv[e] = 0.f;
            if (i < itm.len) {
              const float l = p.lse[itm.head_off + i];
              l2v[e] = l == -CUDART_INF_F ? CUDART_INF_F : l * LOG2E;
              dvv[e] = p.dvec[itm.head_off + i];
            }
          }
          ok = wait_bar(q_empty(sq), ((gi / QS) & 1) ^ 1, ab, p.wait_ns, SITE_BPROD + 0);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          float* side = sSide + sq * 256;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // stored negated: the compute warps add them with paired FMAs
            side[lane + 32 * e] = -l2v[e];
            side[128 + lane + 32 * e] = -dvv[e];
          }
          __threadfence_block();
          __syncwarp();
          if (lane == 0) {
            bar_arrive_expect_tx(q_full(sq), C::TILE);
            for (int c = 0; c < NCH; ++c)
              tma_load_4d(smem_u32(sQ + sq * C::TILE + c * 16384), &p.tm_q, q_full(sq), c * 64, itm.h,
                          itm.trow + i0, itm.bt);
          }
          ++issued_q;
          const int sd = gi % DS;
          ok = wait_bar(do_empty(sd), ((gi / DS) & 1) ^ 1, ab, p.wait_ns, SITE_BPROD + 1);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          if (lane == 0) {
            bar_arrive_expect_tx(do_full(sd), C::TILE);
            for (int c = 0; c < NCH; ++c)
              tma_load_4d(smem_u32(sDO + sd * C::TILE + c * 16384), &p.tm_do, do_full(sd), c * 64, itm.h,
                          itm.trow + i0, itm.bt);
          }
          ++issued_do;
        }
        if (!ok) break;
        if (ORDER && lane == 0) I_next = fetch_item<MODE, ORDER>(p);
        g += itm.nq;
        ++jn;
        if (DYN) I = __shfl_sync(0xffffffffu, I_next, 0);
      }
      // The last CTA to finish taking items returns the counters to zero.
      if (DYN && lane == 0) sched_cta_done(p.sched);
      if (lane == 0) {  // every copy issued must land before the CTA exits
        for (int j = max(0, issued_kv - KVB); j < issued_kv; ++j)
          drain_wait(kv_full(j % KVB), (j / KVB) & 1, p.wait_ns);
        for (int q = max(0, issued_q - QS); q < issued_q; ++q)
          drain_wait(q_full(q % QS), (q / QS) & 1, p.wait_ns);
        for (int q = max(0, issued_do - DS); q < issued_do; ++q)
          drain_wait(do_full(q % DS), (q / DS) & 1, p.wait_ns);
      }
    } else if (warp == 13) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t id_kq = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
      const uint32_t id_pd = idesc_bf16_f32(128, HD, 0, 1);   // dV, dK (B MN-major)
      const uint32_t id_dq = idesc_bf16_f32(128, HD, 1, 1);   // dQ (A and B MN-major)
      auto kmajor = [&](uint32_t d_tmem, const uint8_t* a, const uint8_t* bm) {
        const uint32_t a0 = smem_u32(a), bb = smem_u32(bm);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
          umma_ss(d_tmem, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(bb + off, 16, 1024), id_kq, kk > 0);
        }
      };
      // A operand from TMEM: 16 queries per MMA; queries [64w, 64w+64) were
      // packed by compute warpgroup w into columns [64w, 64w+32) of its region.
      auto from_tmem = [&](uint32_t d_tmem, uint32_t a_tmem, const uint8_t* bm, bool acc) {
        const uint32_t bb = smem_u32(bm);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          umma_ts(d_tmem, a_tmem + 64 * (kk / 4) + (kk % 4) * 8,
                  sdesc_sw128(bb + kk * 2048, 16384, 1024), id_pd, (acc || kk > 0) ? 1u : 0u);
      };
      // Issue order.  Item prologue: S_0, dP_0, dV_0, S_1.  Then for block i:
      //   dK_i, dQ_i       (need dS_i)
      //   dP_{i+1}         (needs dQ_i drained out of the shared TMEM columns;
      //                     runs while the compute warps form P_{i+1})
      //   dV_{i+1}         (needs P_{i+1})
      //   S_{i+2}          (S columns are free once dV_{i+1} has read P_{i+1})
      // The compute warps work in the order P_0, dS_0, P_1, dS_1, ...
      // Indices below are the CTA-wide query-block counter g + i.
      const uint8_t* curK = sK;  // this item's K and V
      const uint8_t* curV = sV;
      auto dp = [&](int k) {                      // dP_k^T = V dO_k^T
        const int sd = k % DS;
        if (!wait_bar(do_full(sd), (k / DS) & 1, ab, p.wait_ns, SITE_BMMA + 2)) return false;
        if (WITH_DQ && k > 0 && !wait_bar(dq_free, (k - 1) & 1, ab, p.wait_ns, SITE_BMMA + 3))
          return false;
        tc_fence_after();
        kmajor(tmem + T_DP, curV, sDO + sd * C::TILE);
        umma_commit(dp_full);
        return true;
      };
      auto dv = [&](int k, bool acc) {            // dV += P_k^T dO_k
        const int sd = k % DS;
        if (!wait_bar(p_ready, k & 1, ab, p.wait_ns, SITE_BMMA + 4)) return false;
        tc_fence_after();
        from_tmem(tmem + T_DV, tmem + T_S, sDO + sd * C::TILE, acc);
        umma_commit(do_empty(sd));
        return true;
      };
      auto s_next = [&](int k) {                  // S_k^T = K Q_k^T
        const int sn = k % QS;
        if (!wait_bar(q_full(sn), (k / QS) & 1, ab, p.wait_ns, SITE_BMMA + 5)) return false;
        tc_fence_after();
        kmajor(tmem + T_S, curK, sQ + sn * C::TILE);
        umma_commit(s_full);
        return true;
      };
      int jn = 0, g = 0, k = 0;
      bool ok = true;
      for (;;) {
        int I;
        if (lane == 0) ok = next_item(k, I, false, SITE_BMMA + 8);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        I = __shfl_sync(0xffffffffu, I, 0);
        if (!ok || I < 0) break;
        const BItem itm = item_of<MODE, ORDER>(p, I);
        const int nq = itm.nq;
        const int kvb = jn % KVB;
        curK = kv_k(kvb);
        curV = kv_v(kvb);
        if (lane == 0) {
          ok = wait_bar(kv_full(kvb), (jn / KVB) & 1, ab, p.wait_ns, SITE_BMMA + 0);
          ok = ok && s_next(g);
          ok = ok && dp(g);
          // dV_0 and dK_0 overwrite the accumulators: the compute warps must
          // have read the previous item's
          if (ok && jn > 0) ok = wait_bar(acc_empty, (jn - 1) & 1, ab, p.wait_ns, SITE_BMMA + 7);
          ok = ok && dv(g, false);
          if (ok && nq > 1) ok = s_next(g + 1);
          for (int it = 0; it < nq && ok; ++it) {
            const int gi = g + it;
            const int sq = gi % QS;
            ok = wait_bar(ds_ready, gi & 1, ab, p.wait_ns, SITE_BMMA + 6);
            if (!ok) break;
            tc_fence_after();
            from_tmem(tmem + T_DK, tmem + T_DP, sQ + sq * C::TILE, it > 0);   // dK += dS^T Q
            umma_commit(q_empty(sq));
            if (WITH_DQ) {
              // dQ_i = dS K: A = dS (queries x keys) read MN-major from the
              // dS^T tile, B = K (keys x d) MN-major.
              const uint32_t a0 = smem_u32(sDS), kb0 = smem_u32(curK);
#pragma unroll
              for (int kk = 0; kk < 128 / 16; ++kk)
                umma_ss(tmem + T_DP, sdesc_sw128(a0 + kk * 2048, 16384, 1024),
                        sdesc_sw128(kb0 + kk * 2048, 16384, 1024), id_dq, kk > 0);
              umma_commit(dq_full);
            }
            if (it + 1 < nq) ok = dp(gi + 1) && dv(gi + 1, true);
            if (ok && it + 2 < nq) ok = s_next(gi + 2);
          }
          if (ok) {
            umma_commit(kv_empty(kvb));   // every product reading K and V is issued
            umma_commit(acc_full);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        g += nq;
        ++jn;
      }
      if (lane == 0) {
        umma_commit(drain_bar);
        drain_wait(drain_bar, 0, p.wait_ns);
      }
    }
  } else if (wg < 2) {
    regs_inc<REGS_CMP>();
    // ------------------------------------------------------------ compute (key rows)
    const int r = (warp % 4) * 32 + lane;
    const int cq = 64 * wg;  // this warpgroup's query columns [cq, cq + 64)
    const uint32_t lane_base = uint32_t((warp % 4) * 32) << 16;
    const float C2 = p.scale_log2;
    int jn = 0, g = 0, k = 0;
    bool ok = true;
    for (;;) {
      int I;
      ok = next_item(k, I, true, SITE_BCOMP + 3);
      if (!ok || I < 0) break;
      const BItem itm = item_of<MODE, ORDER>(p, I);
      const int h = itm.h, b = itm.b;
      const int j = itm.k0 + r;
      int lo_q = p.wr >= 0 ? max(0, j - p.wr) : 0;
      int hi_q = p.wl >= 0 ? min(itm.len - 1, j + p.wl) : itm.len - 1;
      if (j >= itm.len) {
        lo_q = 1;
        hi_q = 0;
      }
      float slope2 = 0.f;
      if (ALIBI) slope2 = -p.alibi[h] * LOG2E;
      int qb = itm.qb_first;
      for (int it = 0; it < itm.nq; ++it, qb = next_qblock<MODE>(p, itm, qb)) {
        const int gi = g + it;
        const int i0 = (SPARSE ? qb : itm.qb_first + it) * 128 + cq;
        // a fully hidden block is visited only when the mask keeps none
        const bool hidden = SPARSE && itm.mcol[qb * p.nb] == 0;
        const float* side = sSide + (gi % QS) * 256 + cq;
        ok = wait_bar(s_full, gi & 1, ab, p.wait_ns, SITE_BCOMP + 0);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float pr[64];
        const bool full = (i0 >= lo_q) && (i0 + 63 <= hi_q);
        const float fj = float(i0 - j);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t u[32];
          tmem_ld32(tmem + lane_base + T_S + cq + h2 * 32, u);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const int c = h2 * 32 + e;
            const float4 l4 = *reinterpret_cast<const float4*>(side + c);  // -LSE log2(e)
            float x0, x1, x2, x3;
            if (ALIBI) {
              x0 = fmaf(slope2, fabsf(fj + float(c)), fmaf(__uint_as_float(u[e]), C2, l4.x));
              x1 = fmaf(slope2, fabsf(fj + float(c + 1)), fmaf(__uint_as_float(u[e + 1]), C2, l4.y));
              x2 = fmaf(slope2, fabsf(fj + float(c + 2)), fmaf(__uint_as_float(u[e + 2]), C2, l4.z));
              x3 = fmaf(slope2, fabsf(fj + float(c + 3)), fmaf(__uint_as_float(u[e + 3]), C2, l4.w));
            } else {
              const uint64_t c2x2 = pk2(C2, C2);
              upk2(fma2(pk2(__uint_as_float(u[e]), __uint_as_float(u[e + 1])), c2x2, pk2(l4.x, l4.y)), x0,
                   x1);
              upk2(fma2(pk2(__uint_as_float(u[e + 2]), __uint_as_float(u[e + 3])), c2x2, pk2(l4.z, l4.w)),
                   x2, x3);
            }
            pr[c] = ex2(x0);
            pr[c + 1] = ex2(x1);
            pr[c + 2] = ex2(x2);
            pr[c + 3] = ex2(x3);
          }
        }
        if (!full || hidden) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int i = i0 + c;
            if (hidden || i < lo_q || i > hi_q) pr[c] = 0.f;
          }
        }
        // Dropout: one generator call gives the bytes of four consecutive keys
        // (a quad of lanes: k0 is a multiple of 128) for four consecutive
        // queries; each lane computes one call in four and the quad trades.
        uint32_t keep_lo = 0xFFFFFFFFu, keep_hi = 0xFFFFFFFFu;
        if (DROPOUT) {
          keep_lo = keep_hi = 0u;
#pragma unroll
          for (int t16 = 0; t16 < 4; ++t16) {
            uint32_t z[4];
            dropout_words_col16(p.drop, b, h, j, (i0 >> 2) + 4 * t16, z);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              // bit 7 of each kept byte, the four gathered into bits 28..31
              // by one multiply (the shifted copies never overlap)
              const uint32_t m = dropout_keep_msb4(z[c4], p.drop.threshold);
              const uint32_t nib = (m * 0x00204081u) >> 28;  // bit e: query 4 c4 + e kept
              const int c = 16 * t16 + 4 * c4;
              if (c < 32) keep_lo |= nib << c;
              else keep_hi |= nib << (c - 32);
            }
          }
        }
        auto kept = [&](int c) {
          return ((c < 32 ? keep_lo >> c : keep_hi >> (c - 32)) & 1u) != 0u;
        };
        // P^T (bf16, dropped and rescaled when dropout is on) into columns
        // [cq, cq+32) of the S^T region (already read)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = c * 32 + 2 * e;
            if (DROPOUT) {
              // the pair's two keep bits become 0xFFFF over each kept bf16
              // half: ((bits 0x8001) & 0x10001) 0xFFFF maps 0,1,2,3 to
              // 0, 0xFFFF, 0xFFFF0000, 0xFFFFFFFF (a dropped half is +0)
              const uint32_t two = ((c == 0 ? keep_lo : keep_hi) >> (2 * e)) & 3u;
              w[e] = pack_bf16(pr[c0] * p.drop.keep_scale, pr[c0 + 1] * p.drop.keep_scale) &
                     (((two * 0x8001u) & 0x10001u) * 0xFFFFu);
            } else {
              w[e] = pack_bf16(pr[c0], pr[c0 + 1]);
            }
          }
          tmem_st16(tmem + lane_base + T_S + cq + c * 16, w);
        }
        tmem_st_wait();
        tc_fence_before();
        bar_arrive(p_ready);
        // dS^T = P^T o (dP^T - D), 32 columns at a time
        ok = wait_bar(dp_full, gi & 1, ab, p.wait_ns, SITE_BCOMP + 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t u[32];
          tmem_ld32(tmem + lane_base + T_DP + cq + c * 32, u);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int cc = c * 32 + 2 * e;
            const float4 d4 = *reinterpret_cast<const float4*>(side + 128 + cc);  // -D
            float g0 = __uint_as_float(u[2 * e]), g1 = __uint_as_float(u[2 * e + 1]);
            float g2 = __uint_as_float(u[2 * e + 2]), g3 = __uint_as_float(u[2 * e + 3]);
            if (DROPOUT) {  // dP = (dO V^T) o keep / (1 - p)
              g0 = kept(cc) ? g0 * p.drop.keep_scale : 0.f;
              g1 = kept(cc + 1) ? g1 * p.drop.keep_scale : 0.f;
              g2 = kept(cc + 2) ? g2 * p.drop.keep_scale : 0.f;
              g3 = kept(cc + 3) ? g3 * p.drop.keep_scale : 0.f;
            }
            float s0, s1, s2, s3;  // dS = P o (dP - D), two at a time
            upk2(mul2(pk2(pr[cc], pr[cc + 1]), add2(pk2(g0, g1), pk2(d4.x, d4.y))), s0, s1);
            upk2(mul2(pk2(pr[cc + 2], pr[cc + 3]), add2(pk2(g2, g3), pk2(d4.z, d4.w))), s2, s3);
            w[e] = pack_bf16(s0, s1);
            w[e + 1] = pack_bf16(s2, s3);
          }
          // written over columns this thread has already read
          tmem_st16(tmem + lane_base + T_DP + cq + c * 16, w);
          if (WITH_DQ) st_sw128_row32(sDS, r, cq + c * 32, w);
        }
        tmem_st_wait();
        if (WITH_DQ) fence_proxy_async_smem();
        tc_fence_before();
        // Test switch (off in normal use): in the CTA that takes item 0 (its
        // first item, whichever schedule), compute warpgroup 0 withholds its
        // arrive on the first query block, so the MMA warp's bounded wait
        // for dS runs out and every role of that CTA winds down.
        if (!(p.test_skip && I == 0 && it == 0 && wg == 0)) bar_arrive(ds_ready);
      }
      if (!ok) break;
      // -------------------------------------------------------- item epilogue
      // This warpgroup's half of the d columns of dV and dK leaves TMEM into
      // registers (then the accumulators are free for the next item) and
      // goes to global memory as 16-byte row stores; the rows of a key block
      // that runs past the end of a packed sequence are not written.
      ok = wait_bar(acc_full, jn & 1, ab, p.wait_ns, SITE_BCOMP + 2);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      constexpr int NC = HD / 64;  // 32-column chunks per warpgroup and tensor
      uint32_t wv[NC][16], wk[NC][16];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_base + T_DV + wg * (HD / 2) + c * 32, u);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) wv[c][e] = pack_bf16(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1]));
        tmem_ld32(tmem + lane_base + T_DK + wg * (HD / 2) + c * 32, u);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          wk[c][e] = pack_bf16(__uint_as_float(u[2 * e]) * p.scale, __uint_as_float(u[2 * e + 1]) * p.scale);
      }
      tc_fence_before();
      bar_arrive(acc_empty);
      const SeqView so{itm.bt, itm.trow, itm.len};
      if (j < itm.len) {
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const int col = wg * (HD / 2) + c * 32;
          st_global_row32(p.dv, p.sdv, so, j, h, col, wv[c]);
          st_global_row32(p.dk, p.sdk, so, j, h, col, wk[c]);
        }
      }
      g += itm.nq;
      ++jn;
    }
  } else {
    regs_inc<REGS_DRN>();
    if (WITH_DQ) {
      // ---------------------------------------------------------- dQ drain (query rows)
      const int q = (warp % 4) * 32 + lane;
      const uint32_t lane_base = uint32_t((warp % 4) * 32) << 16;
      const int wq = warp % 4;
      int g = 0, k = 0;
      bool ok = true;
      long long pend_box = -1;  // ordered dQ: the box whose adds are in flight
      uint32_t pend_val = 0;
      for (;;) {
        int I;
        ok = next_item(k, I, true, SITE_BRED + 1);
        if (!ok || I < 0) break;
        const BItem itm = item_of<MODE, ORDER>(p, I);
        const int bh = itm.bt * p.H + itm.h;
        int qb = itm.qb_first;
        for (int it = 0; it < itm.nq; ++it, qb = next_qblock<MODE>(p, itm, qb)) {
          const int gi = g + it;
          const int i0 = (SPARSE ? qb : itm.qb_first + it) * 128;
          ok = wait_bar(dq_full, gi & 1, ab, p.wait_ns, SITE_BRED);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          // dQ leaves TMEM 32 columns (one 128-byte swizzled box of 128 rows)
          // at a time and is added into the accumulator with one TMA bulk
          // reduction per box, staged through a two-slot ring.  The whole tile
          // is read into registers before TMEM is released, then staged as
          // the slots free up.  Each warp stages its own 32 rows (a 32 x
          // 32-column box, 4 KB) and issues the bulk reduction for them: no
          // cross-warp barrier.
          // acc: which of the ordered dQ's two accumulators (0 otherwise)
          auto stage = [&](const uint32_t (&u)[32], int chunk, int acc) {
            if (lane == 0) bulk_wait_read_1();   // this warp's previous box in the slot was read
            __syncwarp();
            uint8_t* row = sStg + (chunk & 1) * 16384 + q * 128;
#pragma unroll
            for (int e = 0; e < 8; ++e)
              *reinterpret_cast<uint4*>(row + ((e ^ (q & 7)) * 16)) =
                  make_uint4(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_reduce_add_3d(&p.tm_dqacc, smem_u32(sStg + (chunk & 1) * 16384 + wq * 4096), chunk * 32,
                                itm.trow + i0 + wq * 32, bh + acc * p.B * p.H);
              bulk_commit();
            }
          };
          constexpr int NC = HD / 32;
          uint32_t u[NC][32];
#pragma unroll
          for (int c = 0; c < NC; ++c) tmem_ld32(tmem + lane_base + T_DP + c * 32, u[c]);
          tmem_ld_wait();
          tc_fence_before();
          bar_arrive(dq_free);   // TMEM columns may now take the next dP^T
          if (ORDER) {
            // Deterministic dQ under a causal mask.  The partial sums of a
            // 32-row box go to one of two accumulators by the parity of the
            // key block, and each accumulator takes them in descending
            // key-block order: key block kb reaches query block qb after
            // qb - kb steps of its own walk, two steps after kb + 2, the one
            // before it in its chain, and the key blocks of a head are taken
            // last first, so a box only ever waits for items taken earlier
            // (no wait can close a cycle).  A counter per box and accumulator
            // holds how many sums it has received: wait for our rank, add, and
            // raise it once the adds are complete.  That is checked at the
            // next box, before its own turn is awaited: a release must never
            // wait behind a later box's turn, or the waits of one chain would
            // queue behind those of the chains further down the diagonal.
            if (lane == 0 && pend_box >= 0) {
              bulk_wait_all();  // the previous box's adds are complete
              fence_proxy_async_global();
              st_release_gpu(p.dq_chain + pend_box, pend_val);
            }
            pend_box = -1;
            const int acc = itm.kb & 1;
            const long long box =
                ((long long)(acc * p.B * p.H + bh) * p.nblocks + qb) * 4 + wq;
            const uint32_t rank = uint32_t(qb - itm.kb) >> 1;
            bool turn = true;
            if (lane == 0) {
              turn = wait_counter_eq(p.dq_chain + box, rank, ab, p.wait_ns, SITE_BRED + 3);
              if (turn) fence_proxy_async_global();
            }
            ok = __shfl_sync(0xffffffffu, turn ? 1 : 0, 0) != 0;
            if (!ok) break;
#pragma unroll
            for (int c = 0; c < NC; ++c) stage(u[c], c, acc);
            pend_box = box;
            pend_val = rank + 1u;
            continue;
          }
#pragma unroll
          for (int c = 0; c < NC; ++c) stage(u[c], c, 0);
        }
        if (!ok) break;
        g += itm.nq;
        if (ORDER && pend_box >= 0) {  // the item's last box: release it now
          if (lane == 0) {
            bulk_wait_all();
            fence_proxy_async_global();
            st_release_gpu(p.dq_chain + pend_box, pend_val);
          }
          pend_box = -1;
        }
      }
      if (lane == 0) bulk_wait_all();
    } else if (DYN) {
      // without dQ this warpgroup still takes its ring entries, so the
      // loader can reuse them
      int k = 0;
      for (;;) {
        int I;
        if (!next_item(k, I, true, SITE_BRED + 2) || I < 0) break;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Kernel 2: dQ by an ordered walk over key blocks (deterministic mode)
// ---------------------------------------------------------------------------
template <int HD, bool ALIBI, bool DROPOUT, int MODE>
__global__ void __launch_bounds__(192, 1) fa2_bwd_dq_sm100_kernel(const __grid_constant__ BwdParams p) {
  using C = DqCfg<HD>;
  constexpr bool PACKED = MODE == kLayoutPacked;
  constexpr bool SPARSE = MODE == kLayoutSparse;
  using namespace bwd_detail;
  constexpr int SLOTS = C::SLOTS;
  constexpr int NCH = HD / 64;
  constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sDO = smem + C::OFF_DO;
  uint8_t* sKV = smem + C::OFF_KV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BARS);
  const uint32_t b0 = smem_u32(bars);
  const uint32_t qd_full = b0;
  auto slot_full = [&](int s) { return b0 + 8u * (1 + s); };
  auto slot_empty = [&](int s) { return b0 + 8u * (1 + SLOTS + s); };
  const uint32_t s_full = b0 + 8u * (1 + 2 * SLOTS);
  const uint32_t dp_full = s_full + 8, ds_ready = s_full + 16, acc_full = s_full + 24;
  const uint32_t drain_bar = s_full + 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  AbortFlag ab{abort_flag};

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // the query blocks of one head are launched together (they share its K
  // and V in L2), the last one first: under a causal mask it visits the most
  // key blocks, so the grid ends on short blocks rather than long ones
  const int qb = p.nblocks - 1 - int(blockIdx.x % p.nblocks);
  const int hb = int(blockIdx.x / p.nblocks);
  const int h = hb % p.H, b = hb / p.H;
  const SeqView sv = PACKED ? seq_view(p.cu_seqlens, b, p.N, p.total) : SeqView{b, 0, p.N};
  const int len = sv.len;
  const int i0 = qb * 128;        // local query row of this block
  if (i0 >= len) return;          // past the end of a shorter packed sequence: no work
  const int i_last = min(len - 1, i0 + 127);
  const int kv_lo = p.wl >= 0 ? max(0, i0 - p.wl) : 0;
  const int kv_hi = p.wr >= 0 ? min(len - 1, i_last + p.wr) : len - 1;
  // key blocks visited: [kb_first, kb_last], only the kept ones when a block
  // mask is given (this query block's mask row)
  int kb_first = kv_lo / 128;
  const int kb_last = kv_hi / 128;
  const uint8_t* mrow = SPARSE ? p.bmask + b * p.bm_sb + h * p.bm_sh + (long long)qb * p.nb : nullptr;
  const int nk = SPARSE ? count_kept(mrow, 1, kb_first, kb_last) : kb_last - kb_first + 1;
  auto next_kb = [&](int kb) { return SPARSE ? next_kept(mrow, 1, kb, kb_last) : kb + 1; };
  const size_t head_off = (size_t(sv.bt) * p.H + h) * (PACKED ? p.stat_rows : p.N) + sv.row0;
  const int trow = sv.row0;       // tensor row of local row 0

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < C::NBARS; ++i) {
      const uint32_t bar = b0 + 8u * i;
      bar_init(bar, bar == ds_ready ? 128 : 1);
    }
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bar_arrive_expect_tx(qd_full, 2 * C::TILE);
      for (int c = 0; c < NCH; ++c) {
        tma_load_4d(smem_u32(sQ + c * 16384), &p.tm_q, qd_full, c * 64, h, trow + i0, sv.bt);
        tma_load_4d(smem_u32(sDO + c * 16384), &p.tm_do, qd_full, c * 64, h, trow + i0, sv.bt);
      }
      int n = 0;
      bool ok = true;
      int kb = kb_first;
      for (int it = 0; it < nk && ok; ++it, kb = next_kb(kb)) {
        const int kv0 = trow + (SPARSE ? kb : kb_first + it) * 128;
        for (int which = 0; which < 2; ++which, ++n) {
          const int s = n % SLOTS;
          if (!wait_bar(slot_empty(s), ((n / SLOTS) & 1) ^ 1, ab, p.wait_ns, SITE_QPROD)) {
            ok = false;
            break;
          }
          bar_arrive_expect_tx(slot_full(s), C::TILE);
          const CUtensorMap* tm = which == 0 ? &p.tm_k : &p.tm_v;
          for (int c = 0; c < NCH; ++c)
            tma_load_4d(smem_u32(sKV + s * C::TILE + c * 16384), tm, slot_full(s), c * 64, h, kv0, sv.bt);
        }
      }
      drain_wait(qd_full, 0, p.wait_ns);
      for (int k = max(0, n - SLOTS); k < n; ++k) drain_wait(slot_full(k % SLOTS), (k / SLOTS) & 1, p.wait_ns);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_dq = idesc_bf16_f32(128, HD, 0, 1);
      auto kmajor = [&](uint32_t d_tmem, const uint8_t* a, const uint8_t* bm) {
        const uint32_t a0 = smem_u32(a), bb = smem_u32(bm);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
          umma_ss(d_tmem, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(bb + off, 16, 1024), id_qk, kk > 0);
        }
      };
      bool ok = wait_bar(qd_full, 0, ab, p.wait_ns, SITE_QMMA + 0);
      int n = 0;
      for (int it = 0; it < nk && ok; ++it, n += 2) {
        const int sk = n % SLOTS, sv = (n + 1) % SLOTS;
        ok = wait_bar(slot_full(sk), (n / SLOTS) & 1, ab, p.wait_ns, SITE_QMMA + 1);
        if (!ok) break;
        tc_fence_after();
        kmajor(tmem + T_S, sQ, sKV + sk * C::TILE);     // S = Q K^T
        umma_commit(s_full);
        ok = wait_bar(slot_full(sv), ((n + 1) / SLOTS) & 1, ab, p.wait_ns, SITE_QMMA + 2);
        if (!ok) break;
        tc_fence_after();
        kmajor(tmem + T_DP, sDO, sKV + sv * C::TILE);   // dP = dO V^T
        umma_commit(dp_full);
        ok = wait_bar(ds_ready, it & 1, ab, p.wait_ns, SITE_QMMA + 3);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kb0 = smem_u32(sKV + sk * C::TILE);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)            // dQ += dS K
          umma_ts(tmem + T_DQ, tmem + T_S + kk * 8, sdesc_sw128(kb0 + kk * 2048, 16384, 1024), id_dq,
                  (it > 0 || kk > 0) ? 1u : 0u);
        umma_commit(slot_empty(sk));
        umma_commit(slot_empty(sv));
      }
      umma_commit(acc_full);
      umma_commit(drain_bar);
      drain_wait(drain_bar, 0, p.wait_ns);
    }
  } else {
    // ------------------------------------------------------------ compute (query rows)
    const int r = warp * 32 + lane;
    const int i = i0 + r;
    const int lo = p.wl >= 0 ? max(0, i - p.wl) : 0;
    const int hi = i >= len ? -1 : (p.wr >= 0 ? min(len - 1, i + p.wr) : len - 1);
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const float C2 = p.scale_log2;
    float lse2 = CUDART_INF_F, dval = 0.f, slope2 = 0.f;
    if (i < len) {
      const float l = p.lse[head_off + i];
      lse2 = l == -CUDART_INF_F ? CUDART_INF_F : l * LOG2E;
      dval = p.dvec[head_off + i];
    }
    if (ALIBI) slope2 = -p.alibi[h] * LOG2E;
    bool ok = true;
    int kb = kb_first;
    for (int it = 0; it < nk; ++it, kb = next_kb(kb)) {
      const int kv0 = (SPARSE ? kb : kb_first + it) * 128;
      // a fully hidden block is visited only when the mask keeps none
      const bool hidden = SPARSE && mrow[kb] == 0;
      ok = wait_bar(s_full, it & 1, ab, p.wait_ns, SITE_QCOMP + 0);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float pr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_base + T_S + c * 32, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) pr[c * 32 + e] = __uint_as_float(u[e]);
      }
      tmem_ld_wait();
      const float fi = float(i - kv0);
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float x = fmaf(pr[c], C2, -lse2);
        if (ALIBI) x = fmaf(slope2, fabsf(fi - float(c)), x);
        pr[c] = ex2(x);
      }
      if (hidden || !(kv0 >= lo && kv0 + 127 <= hi)) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int j = kv0 + c;
          if (hidden || j < lo || j > hi) pr[c] = 0.f;
        }
      }
      ok = wait_bar(dp_full, it & 1, ab, p.wait_ns, SITE_QCOMP + 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_base + T_DP + c * 32, u);
        // dropout bytes of keys kv0 + c*32 .. +31 for this row (one generator
        // call per quad of rows and 16 keys; i0 is a multiple of 128)
        uint32_t dw[8];
        if (DROPOUT) {
          uint32_t z[4];
          dropout_words_row16(p.drop, b, h, i, ((kv0 + c * 32) >> 2), z);
#pragma unroll
          for (int e = 0; e < 4; ++e) dw[e] = z[e];
          dropout_words_row16(p.drop, b, h, i, ((kv0 + c * 32) >> 2) + 4, z);
#pragma unroll
          for (int e = 0; e < 4; ++e) dw[4 + e] = z[e];
        }
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          // dropout bytes of keys kv0 + c*32 + 4*e4 .. +3 for this row
          uint32_t word = 0xFFFFFFFFu;
          if (DROPOUT) word = dw[e4];
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int e = 2 * e4 + e2;
            const int cc = c * 32 + 2 * e;
            float g0 = __uint_as_float(u[2 * e]), g1 = __uint_as_float(u[2 * e + 1]);
            if (DROPOUT) {
              g0 = dropout_keep(word, 2 * e2, p.drop.threshold) ? g0 * p.drop.keep_scale : 0.f;
              g1 = dropout_keep(word, 2 * e2 + 1, p.drop.threshold) ? g1 * p.drop.keep_scale : 0.f;
            }
            w[e] = pack_bf16(pr[cc] * (g0 - dval), pr[cc + 1] * (g1 - dval));
          }
        }
        tmem_st16(tmem + lane_base + T_S + c * 16, w);   // dS (bf16) over S
      }
      tmem_st_wait();
      tc_fence_before();
      bar_arrive(ds_ready);
    }
    if (ok) ok = wait_bar(acc_full, 0, ab, p.wait_ns, SITE_QCOMP + 2);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    const SeqView so = PACKED ? seq_view(p.cu_seqlens, b, p.N, p.total) : SeqView{b, 0, p.N};
    const bool tile_store = !PACKED || i0 + 128 <= so.len;
    if (ok) {
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t u[32], w[16];
        tmem_ld32(tmem + lane_base + T_DQ + c * 32, u);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16(__uint_as_float(u[2 * e]) * p.scale, __uint_as_float(u[2 * e + 1]) * p.scale);
        if (tile_store) st_sw128_row32(sQ, r, c * 32, w);   // Q tile is free once every MMA is done
        else if (i < so.len) st_global_row32(p.dq, p.sdq, so, i, h, c * 32, w);
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1, 128);
    if (ok && tile_store && r == 0) {
      for (int c = 0; c < NCH; ++c)
        tma_store_4d(&p.tm_dq, smem_u32(sQ + c * 16384), c * 64, h, so.row0 + i0, so.bt);
      bulk_commit();
      bulk_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Zero-fill of the fp32 dQ accumulator (n4 float4 elements).
__global__ void __launch_bounds__(256) zero_f32x4_kernel(float4* __restrict__ p, long long n4) {
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n4; i += (long long)gridDim.x * 256)
    p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace fa2
