// libfa2: the C ABI declared in include/fa2.h.
//
// Host side only: argument checks, TMA descriptor encoding, kernel choice and
// launch on the caller's stream.  All arithmetic of the attention path runs
// in the kernels included below.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <type_traits>
#include <utility>

#include "../../include/fa2.h"
#include "attn_common.cuh"
#include "bwd_sm100.cuh"
#include "fwd_sm100.cuh"
#include "rowwise.cuh"
#include "simt.cuh"
#include "sm100_ptx.cuh"

using namespace fa2;

namespace {

std::atomic<unsigned long long> g_wait_ns{1000ull * 1000ull * 1000ull};
std::atomic<int> g_test_skip{0};  // fa2_test_skip_arrive: 0 off, 1 forward, 2 backward
std::atomic<uint64_t> g_launches{0};

constexpr int kMaxDevices = 64;

// ----------------------------------------------------------------- checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa2_status check_shape(int B, int N, int H, int d, fa2_dtype dtype) {
  if (B < 1 || N < 1 || H < 1) return FA2_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA2_ERR_INVALID_ARG;
  if (dtype != FA2_BF16 && dtype != FA2_F32) return FA2_ERR_INVALID_ARG;
  // grid limits of the launches below
  if (B > 65535 || H > 65535) return FA2_ERR_INVALID_ARG;
  // key blocks x heads x batch (the backward's work items, walked by a
  // persistent grid with int indices) must stay well inside int
  const long long blocks = (N + 127) / 128;
  if (blocks * H * B > 0x7fff0000LL) return FA2_ERR_INVALID_ARG;
  if ((long long)B * H * N > (1LL << 40)) return FA2_ERR_INVALID_ARG;
  return FA2_OK;
}

fa2_status check_tensor(const void* p, const fa2_strides& s, fa2_dtype dtype) {
  if (p == nullptr || !aligned16(p)) return FA2_ERR_INVALID_ARG;
  const int64_t vec = dtype == FA2_BF16 ? 8 : 4;  // elements per 16 bytes
  const int64_t lim = (int64_t(1) << 40) / (dtype == FA2_BF16 ? 2 : 4);
  for (int64_t x : {s.b, s.n, s.h})
    if (x < 1 || x % vec != 0 || x >= lim) return FA2_ERR_INVALID_ARG;
  return FA2_OK;
}

fa2_status check_options(float softmax_scale, float dropout_p, const float* alibi) {
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale)) return FA2_ERR_INVALID_ARG;
  if (std::isnan(dropout_p) || dropout_p < 0.f || dropout_p >= 1.f) return FA2_ERR_INVALID_ARG;
  // the byte threshold t = round(256 p) must leave something to keep
  if (std::floor(double(dropout_p) * 256.0 + 0.5) > 255.0) return FA2_ERR_INVALID_ARG;
  if (alibi != nullptr && (reinterpret_cast<uintptr_t>(alibi) & 3u) != 0) return FA2_ERR_INVALID_ARG;
  return FA2_OK;
}

DropoutParams make_dropout(float dropout_p, unsigned long long seed) {
  DropoutParams d;
  const int t = int(std::floor(double(dropout_p) * 256.0 + 0.5));
  d.seed_lo = uint32_t(seed & 0xFFFFFFFFull);
  d.seed_hi = uint32_t(seed >> 32);
  d.threshold = uint32_t(t);
  d.keep_scale = float(256.0 / (256.0 - t));
  for (int r = 0; r < kPhiloxRounds; ++r) {  // Philox4x32's Weyl key schedule
    d.rk0[r] = d.seed_lo + uint32_t(r) * 0x9E3779B9u;
    d.rk1[r] = d.seed_hi + uint32_t(r) * 0xBB67AE85u;
  }
  return d;
}

#define FA2_TRY(expr)                 \
  do {                                \
    const fa2_status st_ = (expr);    \
    if (st_ != FA2_OK) return st_;    \
  } while (0)

// ----------------------------------------------------------------- device
// Device objects of the library that host code needs the address of: the
// work counters of the counter-scheduled calls and the scratch of
// fa2_bwd_noalloc.  In host code these names are only stand-ins for the
// device objects; their device addresses come from cudaGetSymbolAddress,
// looked up once per device, with that device current, the first time any
// entry point reaches the device, so that no later call (one made during
// stream capture, say) has to.
constexpr int kSchedSlots = 64;
static __device__ unsigned int g_fa2_sched[2 * kSchedSlots];
static __device__ __align__(256) float g_fa2_noalloc_dq[FA2_NOALLOC_MAX_DQ_FLOATS];

struct DeviceInfo {
  int sm_major = -1;
  int sm_minor = -1;
  int sm_count = 0;
  unsigned int* sched = nullptr;  // device address of g_fa2_sched
  float* noalloc_dq = nullptr;    // device address of g_fa2_noalloc_dq
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

fa2_status current_device(int* dev, DeviceInfo* info) {
  if (cudaGetDevice(dev) != cudaSuccess) return FA2_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return FA2_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[*dev];
  if (di.sm_major < 0) {
    DeviceInfo n;
    void* sched = nullptr;
    void* scratch = nullptr;
    if (cudaDeviceGetAttribute(&n.sm_major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n.sm_minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n.sm_count, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess ||
        cudaGetSymbolAddress(&sched, g_fa2_sched) != cudaSuccess || sched == nullptr ||
        cudaGetSymbolAddress(&scratch, g_fa2_noalloc_dq) != cudaSuccess || scratch == nullptr)
      return FA2_ERR_CUDA;
    n.sched = static_cast<unsigned int*>(sched);
    n.noalloc_dq = static_cast<float*>(scratch);
    di = n;
  }
  *info = di;
  return FA2_OK;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per
// device.
template <typename K>
fa2_status ensure_smem(K kernel, int bytes, int dev, std::atomic<uint64_t>& done_mask) {
  const uint64_t bit = uint64_t(1) << dev;
  if (done_mask.load() & bit) return FA2_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return FA2_ERR_CUDA;
  done_mask.fetch_or(bit);
  return FA2_OK;
}

// ----------------------------------------------------------------- TMA
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

fa2_status get_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::call_once(g_encode_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  *fn = g_encode;
  return g_encode ? FA2_OK : FA2_ERR_CUDA;
}

// 4-D map over a bf16 [B, N, H, d] tensor: dims (d, H, N, B), box
// (64, 1, rows, 1), 128-byte swizzle; rows past N read as zeros and are not
// written by stores.
fa2_status encode_bf16_4d(CUtensorMap* m, const void* ptr, const fa2_strides& s, int B, int N, int H,
                          int d, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  FA2_TRY(get_encoder(&enc));
  cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(H), cuuint64_t(N), cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(s.h) * 2, cuuint64_t(s.n) * 2, cuuint64_t(s.b) * 2};
  cuuint32_t box[4] = {64, 1, cuuint32_t(box_rows), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA2_OK : FA2_ERR_CUDA;
}

// The same map over an e4m3 [B, N, H, d] tensor (bytes): box (128, 1, 128,
// 1), one 128-byte swizzled row per tile row at d = 128.
fa2_status encode_u8_4d(CUtensorMap* m, const void* ptr, const fa2_strides& s, int B, int N, int H,
                        int d) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  FA2_TRY(get_encoder(&enc));
  cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(H), cuuint64_t(N), cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(s.h), cuuint64_t(s.n), cuuint64_t(s.b)};
  cuuint32_t box[4] = {128, 1, 128, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA2_OK : FA2_ERR_CUDA;
}

// 3-D map over the fp32 dQ accumulator [B*H, N, d] (dense): dims (d, N, B*H),
// box (32, 32, 1) -- one warp's 32 rows -- 128-byte swizzle; used for TMA
// bulk reductions.
fa2_status encode_dqacc_3d(CUtensorMap* m, void* ptr, int B, int N, int H, int d) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  FA2_TRY(get_encoder(&enc));
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(B) * cuuint64_t(H)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 4, cuuint64_t(N) * cuuint64_t(d) * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA2_OK : FA2_ERR_CUDA;
}

Strides to_s(const fa2_strides& s) { return Strides{s.b, s.n, s.h}; }

// The tensors as the TMA maps see them: B x N rows (padded) or one batch
// entry of `total` rows (packed, whose b stride is unused and is given a
// value that keeps the map well formed).
struct MapShape {
  int bt, rows;
};
MapShape map_shape(const AttnArgs& a) { return a.cu_seqlens ? MapShape{1, a.total} : MapShape{a.B, a.N}; }
fa2_strides map_strides(const AttnArgs& a, fa2_strides s) {
  if (a.cu_seqlens) s.b = s.n * int64_t(a.total > 0 ? a.total : 1);
  return s;
}
fa2_status encode_input(CUtensorMap* m, const void* ptr, const fa2_strides& s, const AttnArgs& a, int d) {
  const MapShape ms = map_shape(a);
  return encode_bf16_4d(m, ptr, map_strides(a, s), ms.bt, ms.rows, a.H, d, 128);
}

void normalise_window(int causal, int* wl, int* wr) {
  if (*wl < 0) *wl = -1;
  if (*wr < 0) *wr = -1;
  if (causal) *wr = 0;  // causal: key j <= query i, the same as a right bound of 0
  // (a right bound above 0 with causal still means j <= i)
}

float resolve_scale(float s, int d) { return s > 0.f ? s : 1.0f / std::sqrt(float(d)); }

// Call after every group of `n` kernel launches.
fa2_status launched(int n) {
  if (cudaGetLastError() != cudaSuccess) return FA2_ERR_CUDA;
  g_launches.fetch_add(uint64_t(n));
  return FA2_OK;
}

// Work counters of the counter-scheduled calls (packed, block-sparse, and
// padded backward calls with a causal mask over many key blocks): pairs
// {next item, finished CTAs} in g_fa2_sched.  Each stream that makes such
// calls owns one pair, so calls that may run at the same time (on different
// streams) never share one, and calls on one stream, which run one after the
// other, reuse it.  The pair is cleared on the call's stream right before
// each launch (the call's last CTA clears it too), which also repairs a pair
// that an aborted call left non-zero.  Up to kSchedSlots streams per device
// own a pair at a time; a further stream takes over the pair used least
// recently.  Every launch (outside stream capture) first makes its stream
// wait (cudaStreamWaitEvent) for the event recorded after the pair's last
// launch, so two calls can never overlap on a pair -- also when a stream
// handle is destroyed and reused while its last call still runs.
// During stream capture nothing is recorded: the captured call keeps the
// capturing stream's pair, and a hand-over that would need a wait is refused
// (FA2_ERR_UNSUPPORTED).
struct SchedSlots {
  cudaStream_t owner[kSchedSlots] = {};
  bool owned[kSchedSlots] = {};
  uint64_t last_use[kSchedSlots] = {};
  cudaEvent_t done[kSchedSlots] = {};  // recorded after the pair's last (uncaptured) launch
  bool done_valid[kSchedSlots] = {};
};
SchedSlots g_slots[kMaxDevices];
std::mutex g_sched_mu;
uint64_t g_sched_clock = 0;

// The counter pair of one launch.  acquire() takes the stream's pair and
// clears it on the stream; finish(), called right after the launch, records
// the pair's event.  The table stays locked in between, so the launch and
// its event are ordered with every other stream's hand-over.
class SchedLease {
 public:
  fa2_status acquire(int dev, const DeviceInfo& di, cudaStream_t st, unsigned int** out) {
    lk_ = std::unique_lock<std::mutex>(g_sched_mu);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return FA2_ERR_CUDA;
    capturing_ = cs != cudaStreamCaptureStatusNone;
    SchedSlots& t = g_slots[dev];
    int s = -1;
    for (int i = 0; i < kSchedSlots && s < 0; ++i)
      if (t.owned[i] && t.owner[i] == st) s = i;
    for (int i = 0; i < kSchedSlots && s < 0; ++i)
      if (!t.owned[i]) s = i;
    bool handover = false;
    if (s < 0) {  // every pair is owned: take over the least recently used one
      s = 0;
      for (int i = 1; i < kSchedSlots; ++i)
        if (t.last_use[i] < t.last_use[s]) s = i;
      handover = true;
    }
    // Order this launch after the pair's last one.  On the pair's own stream
    // that costs nothing on the GPU, and it keeps the pair safe when a stream
    // handle is destroyed and handed out again while its last call still runs.
    if (t.done_valid[s]) {
      if (capturing_) {
        if (handover) return FA2_ERR_UNSUPPORTED;  // a capture cannot wait on it
      } else if (cudaStreamWaitEvent(st, t.done[s], 0) != cudaSuccess) {
        return FA2_ERR_CUDA;
      }
    }
    if (!capturing_ && t.done[s] == nullptr &&
        cudaEventCreateWithFlags(&t.done[s], cudaEventDisableTiming) != cudaSuccess)
      return FA2_ERR_CUDA;
    t.owner[s] = st;
    t.owned[s] = true;
    t.last_use[s] = ++g_sched_clock;
    unsigned int* pair = di.sched + 2 * s;
    if (cudaMemsetAsync(pair, 0, 2 * sizeof(unsigned int), st) != cudaSuccess) return FA2_ERR_CUDA;
    dev_ = dev;
    slot_ = s;
    st_ = st;
    *out = pair;
    return FA2_OK;
  }
  fa2_status finish() {
    if (slot_ < 0) return FA2_OK;
    SchedSlots& t = g_slots[dev_];
    if (!capturing_) {
      if (cudaEventRecord(t.done[slot_], st_) != cudaSuccess) return FA2_ERR_CUDA;
      t.done_valid[slot_] = true;
    }
    slot_ = -1;
    lk_.unlock();
    return FA2_OK;
  }

 private:
  std::unique_lock<std::mutex> lk_;
  int dev_ = -1, slot_ = -1;
  cudaStream_t st_ = nullptr;
  bool capturing_ = false;
};

DeviceInfo device_info(int dev) {
  std::lock_guard<std::mutex> lk(g_dev_mu);
  return g_dev[dev];
}

template <int HD>
fa2_status dispatch_fwd_sm100(const AttnArgs& a, const fa2_strides& sq, const fa2_strides& sk,
                              const fa2_strides& sv, const fa2_strides& so, int dev, int sm_count,
                              int causal_order, cudaStream_t st);

template <int HD, bool ALIBI, bool DROPOUT, int MODE, bool FP8 = false>
fa2_status launch_fwd_sm100(const AttnArgs& a, const fa2_strides& sq, const fa2_strides& sk,
                            const fa2_strides& sv, const fa2_strides& so, int dev, int sm_count,
                            int causal_order, cudaStream_t st) {
  static std::atomic<uint64_t> mask{0};
  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  if (FP8) {
    FA2_TRY(encode_u8_4d(&p.tm_q, a.q, sq, a.B, a.N, a.H, HD));
    FA2_TRY(encode_u8_4d(&p.tm_k, a.k, sk, a.B, a.N, a.H, HD));
    FA2_TRY(encode_u8_4d(&p.tm_v, a.v, sv, a.B, a.N, a.H, HD));
  } else {
    FA2_TRY(encode_input(&p.tm_q, a.q, sq, a, HD));
    FA2_TRY(encode_input(&p.tm_k, a.k, sk, a, HD));
    FA2_TRY(encode_input(&p.tm_v, a.v, sv, a, HD));
  }
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.so_b = a.cu_seqlens ? 0 : so.b;
  p.so_n = so.n;
  p.so_h = so.h;
  p.lse = a.lse;
  p.alibi = a.alibi;
  p.cu_seqlens = a.cu_seqlens;
  p.total = a.total;
  p.stat_rows = map_shape(a).rows;
  p.N = a.N;
  p.H = a.H;
  p.B = a.B;
  p.wl = a.wl;
  p.wr = a.wr;
  p.npairs = (a.N + 255) / 256;
  p.num_units = p.npairs * a.H * a.B;
  p.heavy_first = causal_order;
  p.scale_log2 = a.scale * a.descale_qk * 1.4426950408889634f;
  p.o_scale = a.descale_v;
  p.wait_ns = g_wait_ns.load();
  p.drop = a.drop;
  p.bmask = a.block_mask;
  p.bm_sb = a.bm_sb;
  p.bm_sh = a.bm_sh;
  p.nb = (a.N + 127) / 128;
  p.test_skip = g_test_skip.load() == 1;
  SchedLease lease;
  if (MODE != kLayoutPadded) FA2_TRY(lease.acquire(dev, device_info(dev), st, &p.sched));
  auto kern = fa2_fwd_sm100_kernel<HD, ALIBI, DROPOUT, MODE, FP8>;
  using Cfg = FwdKernelCfg<HD, DROPOUT, FP8>;  // the kernel's own configuration
  constexpr int smem = Cfg::SMEM_BYTES;
  FA2_TRY(ensure_smem(kern, smem, dev, mask));
  // The kernel re-balances registers between its warpgroups; the shares add
  // up to 512 threads x REGS_AT_LAUNCH, so it must launch with that many per
  // thread, or a warpgroup's increase would wait forever.
  {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return FA2_ERR_CUDA;
    if (fa.numRegs < Cfg::REGS_AT_LAUNCH) return FA2_ERR_UNSUPPORTED;
  }
  // persistent grid: one CTA per SM (shared memory and TMEM allow one)
  const unsigned grid = unsigned(std::min(p.num_units, std::max(sm_count, 1)));
  kern<<<grid, Cfg::THREADS, smem, st>>>(p);
  FA2_TRY(launched(1));
  return lease.finish();
}

template <int HD, bool ALIBI, bool DROPOUT, int MODE>
fa2_status launch_bwd_sm100(const AttnArgs& a, const fa2_strides& sq, const fa2_strides& sk,
                            const fa2_strides& sv, const fa2_strides& sdo, const fa2_strides& sdq,
                            const fa2_strides& sdk, const fa2_strides& sdv, int deterministic,
                            int dev, cudaStream_t st) {
  static std::atomic<uint64_t> mask_dkdv{0}, mask_dkdv_nodq{0}, mask_dq{0};
  static std::atomic<uint64_t> mask_dkdv_dyn{0}, mask_dkdv_nodq_dyn{0}, mask_dkdv_ord{0};
  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  const MapShape ms = map_shape(a);
  FA2_TRY(encode_input(&p.tm_q, a.q, sq, a, HD));
  FA2_TRY(encode_input(&p.tm_k, a.k, sk, a, HD));
  FA2_TRY(encode_input(&p.tm_v, a.v, sv, a, HD));
  FA2_TRY(encode_input(&p.tm_do, a.dout, sdo, a, HD));
  FA2_TRY(encode_input(&p.tm_dq, a.dq, sdq, a, HD));
  FA2_TRY(encode_input(&p.tm_dk, a.dk, sdk, a, HD));
  FA2_TRY(encode_input(&p.tm_dv, a.dv, sdv, a, HD));
  // Deterministic calls under a causal mask (padded layout) add dQ in a
  // fixed order inside the dK/dV kernel; other deterministic calls run the
  // ordered second pass (kernel 2).
  constexpr bool CAN_DYN = MODE == kLayoutPadded;
  const bool ordered = CAN_DYN && deterministic && a.wr == 0;
  const bool accumulate = !deterministic || ordered;  // dQ through the fp32 accumulator
  // (the ordered dQ keeps two accumulators, stacked: [2 * B * H, N, d])
  if (accumulate)
    FA2_TRY(encode_dqacc_3d(&p.tm_dqacc, a.dq_accum, ordered ? 2 * ms.bt : ms.bt, ms.rows, a.H, HD));
  p.dq = static_cast<__nv_bfloat16*>(a.dq);
  p.dk = static_cast<__nv_bfloat16*>(a.dk);
  p.dv = static_cast<__nv_bfloat16*>(a.dv);
  p.sdq = a.sdq;
  p.sdk = a.sdk;
  p.sdv = a.sdv;
  p.lse = a.lse;
  p.dvec = a.dvec;
  p.dq_accum = a.dq_accum;
  p.alibi = a.alibi;
  p.cu_seqlens = a.cu_seqlens;
  p.total = a.total;
  p.stat_rows = ms.rows;
  p.bmask = a.block_mask;
  p.bm_sb = a.bm_sb;
  p.bm_sh = a.bm_sh;
  p.nb = (a.N + 127) / 128;
  p.N = a.N;
  p.H = a.H;
  p.B = a.B;
  p.wl = a.wl;
  p.wr = a.wr;
  p.nblocks = (a.N + 127) / 128;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.wait_ns = g_wait_ns.load();
  p.drop = a.drop;
  p.test_skip = g_test_skip.load() == 2;
  const unsigned grid = unsigned(p.nblocks) * unsigned(a.H) * unsigned(a.B);
  // kernel 1 is persistent: one CTA per SM walks the work items
  p.num_items = int(grid);
  DeviceInfo di;
  {
    int dev2;
    FA2_TRY(current_device(&dev2, &di));
  }
  const unsigned grid1 = std::min<unsigned>(grid, unsigned(std::max(di.sm_count, 1)));
  // Under a causal mask (right window 0) key block j of a head has nq - j
  // query blocks.  With many key blocks the static snake leaves some CTAs far
  // behind the rest (25 % over the mean at N = 16384, simulated), so such
  // calls take their items from the shared counter in the same head-major
  // order.  Measured (d = 128, B N = 16384): the counter wins from 128 key
  // blocks on (N = 16384: +9 %; d = 64: +5 %; window (4096, 0) at N = 32768:
  // +1 %) and loses below (N = 4096: -3 %, N = 8192: -5 %).
  // The ordered dQ needs the counter schedule (its key blocks are taken in
  // a fixed order as CTAs become free).
  const bool dyn = CAN_DYN && a.wr == 0 && (p.nblocks >= 128 || ordered);
  SchedLease lease;
  if (MODE != kLayoutPadded || dyn) FA2_TRY(lease.acquire(dev, di, st, &p.sched));
  const size_t accum_floats = size_t(ordered ? 2 : 1) * ms.bt * a.H * ms.rows * HD;
  if (ordered) p.dq_chain = reinterpret_cast<uint32_t*>(a.dq_accum + accum_floats);
  using K1 = void (*)(BwdParams);
  const K1 k1_dq = ordered ? fa2_bwd_dkdv_sm100_kernel<HD, ALIBI, true, DROPOUT, MODE, CAN_DYN, CAN_DYN>
                   : dyn   ? fa2_bwd_dkdv_sm100_kernel<HD, ALIBI, true, DROPOUT, MODE, CAN_DYN>
                           : fa2_bwd_dkdv_sm100_kernel<HD, ALIBI, true, DROPOUT, MODE>;
  const K1 k1_nodq = dyn ? fa2_bwd_dkdv_sm100_kernel<HD, ALIBI, false, DROPOUT, MODE, CAN_DYN>
                         : fa2_bwd_dkdv_sm100_kernel<HD, ALIBI, false, DROPOUT, MODE>;
  constexpr int smem1 = BwdCfg<HD>::SMEM_BYTES;
  // Kernel 1 re-balances registers between its warpgroups; the shares add up
  // to 512 threads x REGS_AT_LAUNCH, so the compiled kernel must launch with
  // at least that many registers per thread, or the increase would wait
  // forever.  Refuse to launch otherwise.
  {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, accumulate ? k1_dq : k1_nodq) != cudaSuccess) return FA2_ERR_CUDA;
    if (fa.numRegs < BwdCfg<HD>::REGS_AT_LAUNCH) return FA2_ERR_UNSUPPORTED;
  }
  if (accumulate) {
    // clear the accumulator (and the ordered dQ's counters, which follow it)
    const long long n4 = (long long)(accum_floats + (ordered ? size_t(2) * ms.bt * a.H * p.nblocks * 4 : 0)) / 4;
    const unsigned zgrid = unsigned(std::min<long long>((n4 + 255) / 256, 148 * 16));
    zero_f32x4_kernel<<<zgrid, 256, 0, st>>>(reinterpret_cast<float4*>(a.dq_accum), n4);
    FA2_TRY(launched(1));
    FA2_TRY(ensure_smem(k1_dq, smem1, dev, ordered ? mask_dkdv_ord : dyn ? mask_dkdv_dyn : mask_dkdv));
    k1_dq<<<grid1, BwdCfg<HD>::THREADS, smem1, st>>>(p);
    FA2_TRY(launched(1));
    FA2_TRY(lease.finish());
    AttnArgs c = a;  // the accumulator is [bt * H, rows, d] in both layouts
    c.B = ms.bt;
    c.N = ms.rows;
    c.cu_seqlens = nullptr;
    const long long rows = (long long)c.B * c.H * c.N;
    const long long per_block = 256 / (HD / 4);
    const unsigned cgrid = unsigned((rows + per_block - 1) / per_block);
    if (ordered) dq_convert_kernel<HD, 2><<<cgrid, 256, 0, st>>>(c);
    else dq_convert_kernel<HD><<<cgrid, 256, 0, st>>>(c);
    return launched(1);
  }
  FA2_TRY(ensure_smem(k1_nodq, smem1, dev, dyn ? mask_dkdv_nodq_dyn : mask_dkdv_nodq));
  k1_nodq<<<grid1, BwdCfg<HD>::THREADS, smem1, st>>>(p);
  FA2_TRY(launched(1));
  FA2_TRY(lease.finish());
  auto k2 = fa2_bwd_dq_sm100_kernel<HD, ALIBI, DROPOUT, MODE>;
  constexpr int smem2 = DqCfg<HD>::SMEM_BYTES;
  FA2_TRY(ensure_smem(k2, smem2, dev, mask_dq));
  k2<<<grid, DqCfg<HD>::THREADS, smem2, st>>>(p);
  return launched(1);
}

// Calls f(std::bool_constant<x>...) for the run-time flags x: picks the
// kernel instantiation that matches the call's options.
template <bool... Fixed, typename F>
fa2_status static_bools(F&& f) {
  return f(std::bool_constant<Fixed>{}...);
}
template <bool... Fixed, typename F, typename... Rest>
fa2_status static_bools(F&& f, bool first, Rest... rest) {
  return first ? static_bools<Fixed..., true>(f, rest...) : static_bools<Fixed..., false>(f, rest...);
}

template <int HD>
fa2_status dispatch_fwd_sm100(const AttnArgs& a, const fa2_strides& sq, const fa2_strides& sk,
                              const fa2_strides& sv, const fa2_strides& so, int dev, int sm_count,
                              int causal_order, cudaStream_t st) {
  return static_bools(
      [&](auto alibi, auto dropout) {
        constexpr bool A = decltype(alibi)::value, D = decltype(dropout)::value;
        if (a.cu_seqlens)
          return launch_fwd_sm100<HD, A, D, kLayoutPacked>(a, sq, sk, sv, so, dev, sm_count, causal_order, st);
        if (a.block_mask)
          return launch_fwd_sm100<HD, A, D, kLayoutSparse>(a, sq, sk, sv, so, dev, sm_count, causal_order, st);
        return launch_fwd_sm100<HD, A, D, kLayoutPadded>(a, sq, sk, sv, so, dev, sm_count, causal_order, st);
      },
      a.alibi != nullptr, a.dropout != 0);
}

template <int HD>
fa2_status dispatch_bwd_sm100(const AttnArgs& a, const fa2_strides& sq, const fa2_strides& sk,
                              const fa2_strides& sv, const fa2_strides& sdo, const fa2_strides& sdq,
                              const fa2_strides& sdk, const fa2_strides& sdv, int deterministic,
                              int dev, cudaStream_t st) {
  return static_bools(
      [&](auto alibi, auto dropout) {
        constexpr bool A = decltype(alibi)::value, D = decltype(dropout)::value;
        if (a.cu_seqlens)
          return launch_bwd_sm100<HD, A, D, kLayoutPacked>(a, sq, sk, sv, sdo, sdq, sdk, sdv,
                                                           deterministic, dev, st);
        if (a.block_mask)
          return launch_bwd_sm100<HD, A, D, kLayoutSparse>(a, sq, sk, sv, sdo, sdq, sdk, sdv,
                                                           deterministic, dev, st);
        return launch_bwd_sm100<HD, A, D, kLayoutPadded>(a, sq, sk, sv, sdo, sdq, sdk, sdv,
                                                         deterministic, dev, st);
      },
      a.alibi != nullptr, a.dropout != 0);
}

// ----------------------------------------------------------------- packed checks
fa2_status check_packed_shape(const int32_t* cu, int B, int max_seqlen, int total, int H, int d,
                              fa2_dtype dtype) {
  if (cu == nullptr || (reinterpret_cast<uintptr_t>(cu) & 3u) != 0) return FA2_ERR_INVALID_ARG;
  if (max_seqlen < 1 || total < 0) return FA2_ERR_INVALID_ARG;
  return check_shape(B, max_seqlen, H, d, dtype);
}

// A packed tensor [total, H, d]: only the row and head strides are used.
fa2_status check_packed_tensor(const void* p, fa2_strides s, fa2_dtype dtype, int total) {
  const int64_t lim = (int64_t(1) << 40) / (dtype == FA2_BF16 ? 2 : 4);
  if (s.n >= 1 && int64_t(total) * s.n >= lim) return FA2_ERR_INVALID_ARG;
  s.b = s.n;  // checked like the others, then ignored
  return check_tensor(p, s, dtype);
}

// Block mask: device bytes, batch/head strides >= 0 (0 shares one mask).
fa2_status check_block_mask(const uint8_t* m, int64_t sb, int64_t sh) {
  if (m == nullptr || sb < 0 || sh < 0) return FA2_ERR_INVALID_ARG;
  if (sb >= (int64_t(1) << 40) || sh >= (int64_t(1) << 40)) return FA2_ERR_INVALID_ARG;
  return FA2_OK;
}

fa2_status check_workspace(const void* ws, size_t bytes, size_t need) {
  if (need == 0) return FA2_OK;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || bytes < need)
    return FA2_ERR_INVALID_ARG;
  return FA2_OK;
}

// ----------------------------------------------------------------- argument blocks
void fill_common(AttnArgs* a, int B, int N, int H, int d, float softmax_scale, int causal,
                 int window_left, int window_right, const float* alibi, float dropout_p,
                 unsigned long long dropout_seed) {
  a->B = B; a->N = N; a->H = H; a->d = d;
  a->alibi = alibi;
  a->scale = resolve_scale(softmax_scale, d);
  a->wl = window_left;
  a->wr = window_right;
  normalise_window(causal, &a->wl, &a->wr);
  a->dropout = dropout_p != 0.f;
  a->drop = make_dropout(dropout_p, dropout_seed);
  a->descale_qk = 1.f;
  a->descale_v = 1.f;
}

void fill_fwd_args(AttnArgs* a, const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int N, int H, int d, const fa2_strides& sq, const fa2_strides& sk,
                   const fa2_strides& sv, const fa2_strides& so, float softmax_scale, int causal,
                   int window_left, int window_right, const float* alibi, float dropout_p,
                   unsigned long long dropout_seed) {
  std::memset(a, 0, sizeof(*a));
  a->q = q; a->k = k; a->v = v; a->o = o; a->lse = lse;
  a->sq = to_s(sq); a->sk = to_s(sk); a->sv = to_s(sv); a->so = to_s(so);
  fill_common(a, B, N, H, d, softmax_scale, causal, window_left, window_right, alibi, dropout_p,
              dropout_seed);
}

void fill_bwd_args(AttnArgs* a, const void* q, const void* k, const void* v, const void* dout,
                   const float* lse, const float* D, void* dq, void* dk, void* dv, void* workspace,
                   int B, int N, int H, int d, const fa2_strides& sq, const fa2_strides& sk,
                   const fa2_strides& sv, const fa2_strides& sdo, const fa2_strides& sdq,
                   const fa2_strides& sdk, const fa2_strides& sdv, float softmax_scale, int causal,
                   int window_left, int window_right, const float* alibi, float dropout_p,
                   unsigned long long dropout_seed) {
  std::memset(a, 0, sizeof(*a));
  a->q = q; a->k = k; a->v = v; a->dout = dout;
  a->lse = const_cast<float*>(lse); a->dvec = D;
  a->dq = dq; a->dk = dk; a->dv = dv;
  a->dq_accum = static_cast<float*>(workspace);
  a->sq = to_s(sq); a->sk = to_s(sk); a->sv = to_s(sv); a->sdo = to_s(sdo);
  a->sdq = to_s(sdq); a->sdk = to_s(sdk); a->sdv = to_s(sdv);
  fill_common(a, B, N, H, d, softmax_scale, causal, window_left, window_right, alibi, dropout_p,
              dropout_seed);
}

// ----------------------------------------------------------------- kernel choice
fa2_status run_fwd(const AttnArgs& a, fa2_dtype dtype, const fa2_strides& sq, const fa2_strides& sk,
                   const fa2_strides& sv, const fa2_strides& so, cudaStream_t st) {
  int dev;
  DeviceInfo di;
  FA2_TRY(current_device(&dev, &di));
  if (dtype == FA2_F32) {
    dim3 grid((a.N + 3) / 4, a.H, a.B);
    if (a.d == 64) simt_fwd_kernel<float, 64><<<grid, 128, 0, st>>>(a);
    else simt_fwd_kernel<float, 128><<<grid, 128, 0, st>>>(a);
    return launched(1);
  }
  if (di.sm_major != 10 || di.sm_minor != 0) return FA2_ERR_UNSUPPORTED;  // sm_100a kernels only
  // Longest-first unit order when masks make the work per unit vary;
  // otherwise the query pairs of one head run together and share its K/V
  // in L2.  (Packed calls take units dynamically in this order.)
  const int heavy_first = (a.wr >= 0 || a.wl >= 0) ? 1 : 0;
  return a.d == 128 ? dispatch_fwd_sm100<128>(a, sq, sk, sv, so, dev, di.sm_count, heavy_first, st)
                    : dispatch_fwd_sm100<64>(a, sq, sk, sv, so, dev, di.sm_count, heavy_first, st);
}

fa2_status run_bwd(const AttnArgs& a, fa2_dtype dtype, const fa2_strides& sq, const fa2_strides& sk,
                   const fa2_strides& sv, const fa2_strides& sdo, const fa2_strides& sdq,
                   const fa2_strides& sdk, const fa2_strides& sdv, int deterministic,
                   cudaStream_t st) {
  int dev;
  DeviceInfo di;
  FA2_TRY(current_device(&dev, &di));
  if (dtype == FA2_F32) {
    dim3 grid((a.N + 3) / 4, a.H, a.B);
    if (a.d == 64) {
      simt_bwd_dkdv_kernel<float, 64><<<grid, 128, 0, st>>>(a);
      simt_bwd_dq_kernel<float, 64><<<grid, 128, 0, st>>>(a);
    } else {
      simt_bwd_dkdv_kernel<float, 128><<<grid, 128, 0, st>>>(a);
      simt_bwd_dq_kernel<float, 128><<<grid, 128, 0, st>>>(a);
    }
    return launched(2);
  }
  if (di.sm_major != 10 || di.sm_minor != 0) return FA2_ERR_UNSUPPORTED;
  return a.d == 128 ? dispatch_bwd_sm100<128>(a, sq, sk, sv, sdo, sdq, sdk, sdv, deterministic, dev, st)
                    : dispatch_bwd_sm100<64>(a, sq, sk, sv, sdo, sdq, sdk, sdv, deterministic, dev, st);
}

}  // namespace

extern "C" {

const char* fa2_strerror(fa2_status s) {
  switch (s) {
    case FA2_OK: return "FA2_OK";
    case FA2_ERR_INVALID_ARG: return "FA2_ERR_INVALID_ARG: invalid pointer, shape, stride or option";
    case FA2_ERR_UNSUPPORTED: return "FA2_ERR_UNSUPPORTED: valid but not implemented";
    case FA2_ERR_CUDA: return "FA2_ERR_CUDA: a CUDA call failed";
    case FA2_ERR_DEVICE_TIMEOUT:
      return "FA2_ERR_DEVICE_TIMEOUT: a kernel gave up a bounded wait or met malformed cu_seqlens";
    case FA2_ERR_SCRATCH_LIMIT:
      return "FA2_ERR_SCRATCH_LIMIT: B*H*N*d exceeds the fixed scratch of fa2_bwd_noalloc";
  }
  return "unknown fa2_status";
}

uint64_t fa2_kernel_launches(void) { return g_launches.load(); }

fa2_status fa2_set_wait_limit_ms(int ms) {
  if (ms < 1) return FA2_ERR_INVALID_ARG;
  g_wait_ns.store((unsigned long long)ms * 1000ull * 1000ull);
  return FA2_OK;
}

fa2_status fa2_test_skip_arrive(int which) {
  if (which < 0 || which > 2) return FA2_ERR_INVALID_ARG;
  g_test_skip.store(which);
  return FA2_OK;
}

fa2_status fa2_device_status(int* code, int clear) {
  if (code == nullptr) return FA2_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return FA2_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fa2_device_status, sizeof(int)) != cudaSuccess) return FA2_ERR_CUDA;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fa2_device_status, &zero, sizeof(int)) != cudaSuccess) return FA2_ERR_CUDA;
  }
  *code = v;
  return v ? FA2_ERR_DEVICE_TIMEOUT : FA2_OK;
}

fa2_status fa2_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N,
                   int H, int d, fa2_dtype dtype, fa2_strides sq, fa2_strides sk, fa2_strides sv,
                   fa2_strides so, float softmax_scale, int causal, int window_left, int window_right,
                   const float* alibi_slopes, float dropout_p, unsigned long long dropout_seed,
                   void* stream) {
  FA2_TRY(check_shape(B, N, H, d, dtype));
  FA2_TRY(check_tensor(q, sq, dtype));
  FA2_TRY(check_tensor(k, sk, dtype));
  FA2_TRY(check_tensor(v, sv, dtype));
  FA2_TRY(check_tensor(o, so, dtype));
  if (lse == nullptr || !aligned16(lse)) return FA2_ERR_INVALID_ARG;
  if (o == q || o == k || o == v) return FA2_ERR_INVALID_ARG;
  FA2_TRY(check_options(softmax_scale, dropout_p, alibi_slopes));
  AttnArgs a;
  fill_fwd_args(&a, q, k, v, o, lse, B, N, H, d, sq, sk, sv, so, softmax_scale, causal, window_left,
                window_right, alibi_slopes, dropout_p, dropout_seed);
  return run_fwd(a, dtype, sq, sk, sv, so, static_cast<cudaStream_t>(stream));
}

fa2_status fa2_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                          const int32_t* cu_seqlens, int B, int max_seqlen, int total, int H, int d,
                          fa2_dtype dtype, fa2_strides sq, fa2_strides sk, fa2_strides sv,
                          fa2_strides so, float softmax_scale, int causal, int window_left,
                          int window_right, const float* alibi_slopes, float dropout_p,
                          unsigned long long dropout_seed, void* stream) {
  FA2_TRY(check_packed_shape(cu_seqlens, B, max_seqlen, total, H, d, dtype));
  FA2_TRY(check_options(softmax_scale, dropout_p, alibi_slopes));
  if (total == 0) return FA2_OK;  // every sequence is empty
  FA2_TRY(check_packed_tensor(q, sq, dtype, total));
  FA2_TRY(check_packed_tensor(k, sk, dtype, total));
  FA2_TRY(check_packed_tensor(v, sv, dtype, total));
  FA2_TRY(check_packed_tensor(o, so, dtype, total));
  if (lse == nullptr || !aligned16(lse)) return FA2_ERR_INVALID_ARG;
  if (o == q || o == k || o == v) return FA2_ERR_INVALID_ARG;
  AttnArgs a;
  fill_fwd_args(&a, q, k, v, o, lse, B, max_seqlen, H, d, sq, sk, sv, so, softmax_scale, causal,
                window_left, window_right, alibi_slopes, dropout_p, dropout_seed);
  a.cu_seqlens = cu_seqlens;
  a.total = total;
  return run_fwd(a, dtype, sq, sk, sv, so, static_cast<cudaStream_t>(stream));
}

fa2_status fa2_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                               int N, int H, int d, fa2_dtype dtype, fa2_strides sq, fa2_strides sk,
                               fa2_strides sv, fa2_strides so, const uint8_t* block_mask,
                               int64_t mask_stride_b, int64_t mask_stride_h, float softmax_scale,
                               int causal, int window_left, int window_right,
                               const float* alibi_slopes, float dropout_p,
                               unsigned long long dropout_seed, void* stream) {
  FA2_TRY(check_shape(B, N, H, d, dtype));
  FA2_TRY(check_tensor(q, sq, dtype));
  FA2_TRY(check_tensor(k, sk, dtype));
  FA2_TRY(check_tensor(v, sv, dtype));
  FA2_TRY(check_tensor(o, so, dtype));
  if (lse == nullptr || !aligned16(lse)) return FA2_ERR_INVALID_ARG;
  if (o == q || o == k || o == v) return FA2_ERR_INVALID_ARG;
  FA2_TRY(check_options(softmax_scale, dropout_p, alibi_slopes));
  FA2_TRY(check_block_mask(block_mask, mask_stride_b, mask_stride_h));
  AttnArgs a;
  fill_fwd_args(&a, q, k, v, o, lse, B, N, H, d, sq, sk, sv, so, softmax_scale, causal, window_left,
                window_right, alibi_slopes, dropout_p, dropout_seed);
  a.block_mask = block_mask;
  a.bm_sb = mask_stride_b;
  a.bm_sh = mask_stride_h;
  return run_fwd(a, dtype, sq, sk, sv, so, static_cast<cudaStream_t>(stream));
}

fa2_status fa2_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N,
                       int H, int d, fa2_strides sq, fa2_strides sk, fa2_strides sv, fa2_strides so,
                       float q_descale, float k_descale, float v_descale, float softmax_scale,
                       int causal, int window_left, int window_right, const float* alibi_slopes,
                       void* stream) {
  FA2_TRY(check_shape(B, N, H, d, FA2_BF16));
  // e4m3 tensors: strides in bytes must keep rows 16-byte aligned (the
  // check for a 1-byte type is the fp32 one with four times the stride)
  for (auto [ptr, s] : {std::pair<const void*, fa2_strides>{q, sq}, {k, sk}, {v, sv}}) {
    if (s.b % 16 != 0 || s.n % 16 != 0 || s.h % 16 != 0) return FA2_ERR_INVALID_ARG;
    FA2_TRY(check_tensor(ptr, s, FA2_BF16));
  }
  FA2_TRY(check_tensor(o, so, FA2_BF16));
  if (lse == nullptr || !aligned16(lse)) return FA2_ERR_INVALID_ARG;
  if (o == q || o == k || o == v) return FA2_ERR_INVALID_ARG;
  FA2_TRY(check_options(softmax_scale, 0.f, alibi_slopes));
  for (float x : {q_descale, k_descale, v_descale})
    if (!(x > 0.f) || std::isinf(x)) return FA2_ERR_INVALID_ARG;
  if (d != 128) return FA2_ERR_UNSUPPORTED;
  AttnArgs a;
  fill_fwd_args(&a, q, k, v, o, lse, B, N, H, d, sq, sk, sv, so, softmax_scale, causal, window_left,
                window_right, alibi_slopes, 0.f, 0);
  a.descale_qk = q_descale * k_descale;
  a.descale_v = v_descale;
  int dev;
  DeviceInfo di;
  FA2_TRY(current_device(&dev, &di));
  if (di.sm_major != 10 || di.sm_minor != 0) return FA2_ERR_UNSUPPORTED;
  const int heavy_first = (a.wr >= 0 || a.wl >= 0) ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return a.alibi ? launch_fwd_sm100<128, true, false, kLayoutPadded, true>(a, sq, sk, sv, so, dev,
                                                                          di.sm_count, heavy_first, st)
                 : launch_fwd_sm100<128, false, false, kLayoutPadded, true>(a, sq, sk, sv, so, dev,
                                                                           di.sm_count, heavy_first, st);
}

fa2_status fa2_bwd_preprocess(const void* o, const void* dout, float* D, int B, int N, int H, int d,
                              fa2_dtype dtype, fa2_strides so, fa2_strides sdo, void* stream) {
  FA2_TRY(check_shape(B, N, H, d, dtype));
  FA2_TRY(check_tensor(o, so, dtype));
  FA2_TRY(check_tensor(dout, sdo, dtype));
  if (D == nullptr || !aligned16(D)) return FA2_ERR_INVALID_ARG;
  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.o = const_cast<void*>(o); a.dout = dout; a.dvec = D;
  a.so = to_s(so); a.sdo = to_s(sdo);
  a.B = B; a.N = N; a.H = H; a.d = d;
  int dev;
  DeviceInfo di;
  FA2_TRY(current_device(&dev, &di));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long rows = (long long)B * H * N;
  const int lanes = dtype == FA2_BF16 ? d / 8 : d / 4;
  const long long per_block = 256 / lanes;
  const unsigned grid = unsigned((rows + per_block - 1) / per_block);
  if (dtype == FA2_BF16) {
    if (d == 64) bwd_preprocess_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(a);
    else bwd_preprocess_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(a);
  } else {
    if (d == 64) bwd_preprocess_kernel<float, 64><<<grid, 256, 0, st>>>(a);
    else bwd_preprocess_kernel<float, 128><<<grid, 256, 0, st>>>(a);
  }
  return launched(1);
}

size_t fa2_bwd_workspace_size(int B, int N, int H, int d, fa2_dtype dtype, int deterministic) {
  if (check_shape(B, N, H, d, dtype) != FA2_OK) return 0;
  if (dtype != FA2_BF16) return 0;
  // fp32 dQ accumulator [B*H, N, d]; deterministic calls keep two of them
  // and a counter per 32-row box of every query block for each,
  // [2, B*H, ceil(N/128), 4]
  size_t bytes = size_t(deterministic ? 2 : 1) * B * H * N * d * sizeof(float);
  if (deterministic) bytes += size_t(2) * B * H * ((N + 127) / 128) * 4 * sizeof(uint32_t);
  return (bytes + 255) & ~size_t(255);
}

fa2_status fa2_bwd(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                   const float* D, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, int B, int N, int H, int d, fa2_dtype dtype,
                   fa2_strides sq, fa2_strides sk, fa2_strides sv, fa2_strides sdo,
                   fa2_strides sdq, fa2_strides sdk, fa2_strides sdv, float softmax_scale,
                   int causal, int window_left, int window_right, const float* alibi_slopes,
                   float dropout_p, unsigned long long dropout_seed, int deterministic,
                   void* stream) {
  FA2_TRY(check_shape(B, N, H, d, dtype));
  for (auto [ptr, s] : {std::pair<const void*, fa2_strides>{q, sq}, {k, sk}, {v, sv}, {dout, sdo},
                        {dq, sdq}, {dk, sdk}, {dv, sdv}})
    FA2_TRY(check_tensor(ptr, s, dtype));
  if (lse == nullptr || !aligned16(lse) || D == nullptr || !aligned16(D)) return FA2_ERR_INVALID_ARG;
  FA2_TRY(check_options(softmax_scale, dropout_p, alibi_slopes));
  FA2_TRY(check_workspace(workspace, workspace_bytes,
                          fa2_bwd_workspace_size(B, N, H, d, dtype, deterministic)));
  AttnArgs a;
  fill_bwd_args(&a, q, k, v, dout, lse, D, dq, dk, dv, workspace, B, N, H, d, sq, sk, sv, sdo, sdq,
                sdk, sdv, softmax_scale, causal, window_left, window_right, alibi_slopes, dropout_p,
                dropout_seed);
  return run_bwd(a, dtype, sq, sk, sv, sdo, sdq, sdk, sdv, deterministic,
                 static_cast<cudaStream_t>(stream));
}

fa2_status fa2_bwd_varlen(const void* q, const void* k, const void* v, const void* dout,
                          const float* lse, const float* D, void* dq, void* dk, void* dv,
                          void* workspace, size_t workspace_bytes, const int32_t* cu_seqlens, int B,
                          int max_seqlen, int total, int H, int d, fa2_dtype dtype, fa2_strides sq,
                          fa2_strides sk, fa2_strides sv, fa2_strides sdo, fa2_strides sdq,
                          fa2_strides sdk, fa2_strides sdv, float softmax_scale, int causal,
                          int window_left, int window_right, const float* alibi_slopes,
                          float dropout_p, unsigned long long dropout_seed, int deterministic,
                          void* stream) {
  FA2_TRY(check_packed_shape(cu_seqlens, B, max_seqlen, total, H, d, dtype));
  FA2_TRY(check_options(softmax_scale, dropout_p, alibi_slopes));
  if (total == 0) return FA2_OK;
  for (auto [ptr, s] : {std::pair<const void*, fa2_strides>{q, sq}, {k, sk}, {v, sv}, {dout, sdo},
                        {dq, sdq}, {dk, sdk}, {dv, sdv}})
    FA2_TRY(check_packed_tensor(ptr, s, dtype, total));
  if (lse == nullptr || !aligned16(lse) || D == nullptr || !aligned16(D)) return FA2_ERR_INVALID_ARG;
  FA2_TRY(check_workspace(workspace, workspace_bytes,
                          fa2_bwd_workspace_size(1, total, H, d, dtype, deterministic)));
  AttnArgs a;
  fill_bwd_args(&a, q, k, v, dout, lse, D, dq, dk, dv, workspace, B, max_seqlen, H, d, sq, sk, sv,
                sdo, sdq, sdk, sdv, softmax_scale, causal, window_left, window_right, alibi_slopes,
                dropout_p, dropout_seed);
  a.cu_seqlens = cu_seqlens;
  a.total = total;
  return run_bwd(a, dtype, sq, sk, sv, sdo, sdq, sdk, sdv, deterministic,
                 static_cast<cudaStream_t>(stream));
}

fa2_status fa2_bwd_blocksparse(const void* q, const void* k, const void* v, const void* dout,
                               const float* lse, const float* D, void* dq, void* dk, void* dv,
                               void* workspace, size_t workspace_bytes, int B, int N, int H, int d,
                               fa2_dtype dtype, fa2_strides sq, fa2_strides sk, fa2_strides sv,
                               fa2_strides sdo, fa2_strides sdq, fa2_strides sdk, fa2_strides sdv,
                               const uint8_t* block_mask, int64_t mask_stride_b,
                               int64_t mask_stride_h, float softmax_scale, int causal,
                               int window_left, int window_right, const float* alibi_slopes,
                               float dropout_p, unsigned long long dropout_seed, int deterministic,
                               void* stream) {
  FA2_TRY(check_shape(B, N, H, d, dtype));
  for (auto [ptr, s] : {std::pair<const void*, fa2_strides>{q, sq}, {k, sk}, {v, sv}, {dout, sdo},
                        {dq, sdq}, {dk, sdk}, {dv, sdv}})
    FA2_TRY(check_tensor(ptr, s, dtype));
  if (lse == nullptr || !aligned16(lse) || D == nullptr || !aligned16(D)) return FA2_ERR_INVALID_ARG;
  FA2_TRY(check_options(softmax_scale, dropout_p, alibi_slopes));
  FA2_TRY(check_block_mask(block_mask, mask_stride_b, mask_stride_h));
  FA2_TRY(check_workspace(workspace, workspace_bytes,
                          fa2_bwd_workspace_size(B, N, H, d, dtype, deterministic)));
  AttnArgs a;
  fill_bwd_args(&a, q, k, v, dout, lse, D, dq, dk, dv, workspace, B, N, H, d, sq, sk, sv, sdo, sdq,
                sdk, sdv, softmax_scale, causal, window_left, window_right, alibi_slopes, dropout_p,
                dropout_seed);
  a.block_mask = block_mask;
  a.bm_sb = mask_stride_b;
  a.bm_sh = mask_stride_h;
  return run_bwd(a, dtype, sq, sk, sv, sdo, sdq, sdk, sdv, deterministic,
                 static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// fa2_bwd_noalloc: fa2_bwd (bf16, non-deterministic) with its fp32 dQ
// accumulator in a fixed device array (g_fa2_noalloc_dq above) instead of
// caller workspace.
// ---------------------------------------------------------------------------

fa2_status fa2_bwd_noalloc(const void* q, const void* k, const void* v, const void* dout,
                           const float* lse, const float* D, void* dq, void* dk, void* dv, int B,
                           int N, int H, int d, fa2_strides sq, fa2_strides sk, fa2_strides sv,
                           fa2_strides sdo, fa2_strides sdq, fa2_strides sdk, fa2_strides sdv,
                           float softmax_scale, int causal, int window_left, int window_right,
                           const float* alibi_slopes, float dropout_p, void* stream) {
  const fa2_dtype dtype = FA2_BF16;
  FA2_TRY(check_shape(B, N, H, d, dtype));
  FA2_TRY(check_tensor(q, sq, dtype));
  FA2_TRY(check_tensor(k, sk, dtype));
  FA2_TRY(check_tensor(v, sv, dtype));
  FA2_TRY(check_tensor(dout, sdo, dtype));
  FA2_TRY(check_tensor(dq, sdq, dtype));
  FA2_TRY(check_tensor(dk, sdk, dtype));
  FA2_TRY(check_tensor(dv, sdv, dtype));
  if (lse == nullptr || !aligned16(lse) || D == nullptr || !aligned16(D)) return FA2_ERR_INVALID_ARG;
  FA2_TRY(check_options(softmax_scale, dropout_p, alibi_slopes));
  if (dropout_p != 0.f) return FA2_ERR_UNSUPPORTED;  // this entry point has no seed argument
  if ((unsigned long long)B * H * N * d > (unsigned long long)FA2_NOALLOC_MAX_DQ_FLOATS)
    return FA2_ERR_SCRATCH_LIMIT;
  int dev;
  DeviceInfo di;
  FA2_TRY(current_device(&dev, &di));
  if (di.sm_major != 10 || di.sm_minor != 0) return FA2_ERR_UNSUPPORTED;
  float* scratch = di.noalloc_dq;  // device address of the fixed scratch array
  AttnArgs a;  // the scratch is cleared by the first kernel of the launch sequence
  fill_bwd_args(&a, q, k, v, dout, lse, D, dq, dk, dv, scratch, B, N, H, d, sq, sk, sv, sdo, sdq,
                sdk, sdv, softmax_scale, causal, window_left, window_right, alibi_slopes, 0.f, 0);
  return run_bwd(a, dtype, sq, sk, sv, sdo, sdq, sdk, sdv, 0, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
