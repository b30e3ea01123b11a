// libsambay: C ABI of the SambaY scan + Gated Memory Unit hot path on B200.
// Host side: argument validation, workspace carving, TMA descriptors and
// kernel launches.  Every step of the computation runs in the kernels of
// scan_kernels.cuh, step_kernels.cuh, tc_gemm.cuh and simt_gemm.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include <unistd.h>

#include "../../include/sambay.h"
#include "common.cuh"
#include "attn_kernels.cuh"
#include "scan_kernels.cuh"
#include "simt_gemm.cuh"
#include "ssd_kernels.cuh"
#include "step_kernels.cuh"
#include "tc_gemm.cuh"

using sambay::bf16;

namespace {

constexpr int kMaxDevices = 64;

// ------------------------------------------------------------ device facts

struct DeviceInfo {
  int checked = 0;
  int ok = 0;
  int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];

sambay_status current_device(int* dev_out, int* sms_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAMBAY_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SAMBAY_ERR_DEVICE;
  DeviceInfo& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SAMBAY_ERR_CUDA;
    d.ok = (major == 10);
    d.sms = sms;
    d.checked = 1;
  }
  if (!d.ok) return SAMBAY_ERR_DEVICE;
  *dev_out = dev;
  *sms_out = d.sms;
  return SAMBAY_OK;
}

// ------------------------------------------------------------ kernel timing
//
// While a measurement session is open on the calling thread
// (sambay_profile_begin), every kernel launch records the caller's events
// 2i and 2i+1 on its stream around the i-th launch and remembers the kernel's
// name.  Host-side bookkeeping only; closed sessions cost one branch.

struct ProfState {
  cudaEvent_t* ev = nullptr;
  int cap = 0;      // events available
  int n = 0;        // events used
  std::vector<const char*> names;
};
thread_local ProfState* g_prof = nullptr;
thread_local ProfState g_prof_storage;

struct ProfScope {
  cudaStream_t st;
  bool on;
  ProfScope(const char* name, cudaStream_t s) : st(s), on(g_prof != nullptr && g_prof->n + 2 <= g_prof->cap) {
    if (on) {
      cudaEventRecord(g_prof->ev[g_prof->n], st);
      g_prof->names.push_back(name);
    }
  }
  ~ProfScope() {
    if (on) {
      cudaEventRecord(g_prof->ev[g_prof->n + 1], st);
      g_prof->n += 2;
    }
  }
};

// ------------------------------------------------------------ validation

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t io_bytes(int io) { return io == SAMBAY_BF16 ? 2 : 4; }

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

sambay_status check_dims(const sambay_dims* d, bool need_model, bool need_scan) {
  if (!d) return SAMBAY_ERR_INVALID_ARG;
  if (d->io != SAMBAY_F32 && d->io != SAMBAY_BF16) return SAMBAY_ERR_INVALID_ARG;
  if (d->batch < 1 || d->d_inner < 1) return SAMBAY_ERR_INVALID_ARG;
  if (need_scan) {
    if (d->seqlen < 1 || d->d_state < 1 || d->d_conv < 1 || d->dt_rank < 1)
      return SAMBAY_ERR_INVALID_ARG;
    if (d->d_state != 16 || d->d_conv != 4) return SAMBAY_ERR_UNSUPPORTED;
    if (d->dt_rank % 4 != 0) return SAMBAY_ERR_UNSUPPORTED;
    if (d->dt_rank + 2 * d->d_state > 256) return SAMBAY_ERR_UNSUPPORTED;
    if (d->d_inner % 32 != 0) return SAMBAY_ERR_UNSUPPORTED;
    if (d->io == SAMBAY_BF16 && (d->d_inner % 64 != 0 || d->dt_rank % 8 != 0))
      return SAMBAY_ERR_UNSUPPORTED;
  }
  if (need_model) {
    if (d->d_model < 1) return SAMBAY_ERR_INVALID_ARG;
    if (d->io == SAMBAY_BF16 && (d->d_model % 64 != 0 || d->d_inner % 64 != 0))
      return SAMBAY_ERR_UNSUPPORTED;
    if (d->io == SAMBAY_F32 && (d->d_model % 4 != 0 || d->d_inner % 4 != 0))
      return SAMBAY_ERR_UNSUPPORTED;
  }
  return SAMBAY_OK;
}

sambay_status check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return SAMBAY_ERR_INVALID_ARG;
    if (!aligned16(p)) return SAMBAY_ERR_UNSUPPORTED;
  }
  return SAMBAY_OK;
}

sambay_status check_weights(const sambay_scan_weights* w) {
  if (!w) return SAMBAY_ERR_INVALID_ARG;
  return check_ptrs({w->conv_w, w->conv_b, w->x_proj_w, w->dt_proj_w, w->dt_bias, w->A, w->D});
}

sambay_status check_ws(const void* ws, size_t have, size_t need) {
  if (need == 0) return SAMBAY_OK;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || have < need) return SAMBAY_ERR_WORKSPACE;
  return SAMBAY_OK;
}

// ------------------------------------------------------------ workspace

// Split-K factor of the tensor-core GEMMs that reduce over a long K with few
// output tiles (x_proj, GMU decode).  A function of the sizes only, sized for
// B200's 148 SMs, so the workspace and the summation order do not depend on
// the device.
constexpr int kSplitTarget = 148;

int split_count(long long out_tiles, long long k, int max_splits) {
  const long long k_blocks = (k + sambay::tc::BK - 1) / sambay::tc::BK;
  long long s = std::max(1LL, kSplitTarget / std::max(1LL, out_tiles));
  s = std::min<long long>(s, max_splits);
  s = std::min(s, k_blocks);
  const long long per = (k_blocks + s - 1) / s;  // k-blocks per split
  return static_cast<int>((k_blocks + per - 1) / per);
}

constexpr int kXprojMaxSplits = 64;

// bf16 mode: x_proj reduces over K = 2*Di (the split uc pair)
int xproj_splits(long long rows, int d_inner) {
  return split_count((rows + sambay::tc::BM - 1) / sambay::tc::BM, 2LL * d_inner, kXprojMaxSplits);
}

// dt_rank rounded up to whole 64-wide K blocks (each half of the split delta)
int rank_pad(int R) { return (R + 63) / 64 * 64; }

// The bf16 decode step (step_kernels.cuh): the channels are cut into slices of
// `chan` (a multiple of 8, at most kMaxChan) with about one slice per SM of a
// 148-SM B200 (a function of the sizes only, so the workspace and the
// summation order do not depend on the device), and each CTA takes up to
// `group` sequences of its slice.
constexpr int kMaxDynSmemBytes = 232448;

struct StepPlan {
  bool ok = false;
  int chan = 0, nslice = 0, group = 0, Rp = 0;
  size_t smem = 0;
  bool fused = false;      // one cooperative kernel (batch <= 64 and its layout fits)
  size_t fused_smem = 0;
};

StepPlan step_plan(const sambay_dims* d) {
  StepPlan sp;
  if (d->io != SAMBAY_BF16) return sp;
  const int Di = d->d_inner;
  for (int c = 8; c <= sambay::step::kMaxChan; c += 8)
    if (Di % c == 0 && Di / c <= kSplitTarget) { sp.chan = c; break; }
  if (sp.chan == 0) return sp;                    // wider than 148 slices of 48 channels
  sp.nslice = Di / sp.chan;
  sp.Rp = (d->dt_rank + 15) / 16 * 16;
  int group = std::min(d->batch, sambay::step::kMaxGroup);
  while (group > 4 && sambay::step::ScanStepLayout(sp.chan, group, sp.Rp).bytes > kMaxDynSmemBytes) group -= 4;
  const sambay::step::ScanStepLayout ly(sp.chan, group, sp.Rp);
  if (ly.bytes > kMaxDynSmemBytes) return sp;
  sp.group = group;
  sp.smem = static_cast<size_t>(ly.bytes);
  sp.ok = true;
  if (d->batch <= sambay::step::kMaxGroup) {
    const int ldx = d->dt_rank + 2 * d->d_state;
    const sambay::step::FusedStepLayout fl(sp.chan, d->batch, sp.Rp, ldx, sp.nslice);
    if (fl.bytes <= kMaxDynSmemBytes) {
      sp.fused = true;
      sp.fused_smem = static_cast<size_t>(fl.bytes);
    }
  }
  return sp;
}

struct ScanWs {
  size_t uc, part, xdbl, delta, dt, bcp, total;
  int splits;
};

// Scratch of the bf16 decode step: conv output, x_proj partials per slice,
// the split delta, B | C, and the single-kernel form's meeting words.
struct StepWs {
  size_t uc, part, dts, bc, bar, total;
};

StepWs step_ws_layout(const sambay_dims* d, const StepPlan& sp) {
  StepWs w{};
  const size_t B = d->batch, Di = d->d_inner, ldx = d->dt_rank + 2 * d->d_state;
  size_t off = 0;
  w.uc = off;   off += round256(B * Di * 4);
  w.part = off; off += round256(static_cast<size_t>(sp.nslice) * ldx * B * 4);
  w.dts = off;  off += round256(2 * B * static_cast<size_t>(sp.Rp) * 2);
  w.bc = off;   off += round256(B * 2 * d->d_state * 4);
  w.bar = off;  off += round256(static_cast<size_t>(sambay::step::fused_bar_words(sp.nslice)) * 8);
  w.total = off;
  return w;
}

ScanWs scan_ws_layout(const sambay_dims* d, long long T, bool step = false) {
  ScanWs w{};
  if (step) {
    const StepPlan sp = step_plan(d);
    if (sp.ok) {
      w.total = step_ws_layout(d, sp).total;
      return w;
    }
  }
  const long long Di = d->d_inner, R = d->dt_rank, ldx = d->dt_rank + 2 * d->d_state;
  const bool tc = d->io == SAMBAY_BF16;
  w.splits = tc ? xproj_splits(T, d->d_inner) : 1;
  size_t off = 0;
  // uc: f32, or the bf16 split pair (hi | lo): 4 bytes per element either way
  w.uc = off;    off += round256(static_cast<size_t>(T * Di) * 4);
  w.part = off;  off += tc ? round256(static_cast<size_t>(w.splits) * T * ldx * 4) : 0;
  w.xdbl = off;  off += round256(static_cast<size_t>(T * ldx) * 4);
  w.delta = off; off += tc ? round256(static_cast<size_t>(T) * 2 * rank_pad(static_cast<int>(R)) * 2) : 0;
  w.dt = off;    off += round256(static_cast<size_t>(T * Di) * 4);
  // B | C regrouped into token pairs for the prefill scan: ceil(L / 2) pairs
  // of 64 floats per sequence (the decode step reads xdbl instead)
  w.bcp = off;   off += step ? 0 : round256(static_cast<size_t>(d->batch) * ((T / d->batch + 1) / 2) * 64 * 4);
  w.total = off;
  return w;
}

struct GmuWs {
  size_t h, tail, tail_bytes, total;
};

constexpr int kStepMaxRows = 256;
constexpr int kStepMaxSplits = 8;
// Partial tiles of a prefill GEMM's K-split tail: at most one 256 x 256 fp32
// tile per CTA pair of a 148-SM B200, then the tail units' arrival flags (one
// 8-byte flag per tail unit and CTA of its pair) in an area of their own.
constexpr int kTailUnits = 74;
constexpr size_t kTailSyncBytes = 4096;

// Epochs of the K-split tail's arrival flags: one per launch, from a 48-bit
// sequence that starts at a point drawn from the clock and the process id
// (splitmix64), so that no flag left in reused scratch carries a live epoch.
unsigned long long next_tail_epoch() {
  static const unsigned long long base = [] {
    unsigned long long z = static_cast<unsigned long long>(
                               std::chrono::steady_clock::now().time_since_epoch().count()) ^
                           (static_cast<unsigned long long>(getpid()) << 32);
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }();
  static std::atomic<unsigned long long> seq{0};
  for (;;) {
    const unsigned long long e = (base + seq.fetch_add(1)) & ((1ull << 48) - 1);
    if (e != 0) return e;
  }
}

GmuWs gmu_ws_layout(const sambay_dims* d, long long rows, bool step) {
  GmuWs w{};
  size_t off = 0;
  w.h = off;
  off += round256(static_cast<size_t>(rows) * d->d_inner * io_bytes(d->io));
  if (!step && d->io == SAMBAY_BF16 && rows > 256) {
    // more than one 256-row tile: room for the K-split tail of either GEMM
    w.tail = off;
    w.tail_bytes = static_cast<size_t>(kTailUnits) * 256 * 256 * 4 + kTailSyncBytes;
    off += round256(w.tail_bytes);
  }
  w.total = off;
  return w;
}

// ------------------------------------------------------------ TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D tensor [outer, inner] (inner contiguous, row pitch row_bytes) with a
// box of {box_inner, box_outer} elements whose inner extent is 128 bytes,
// 128-byte swizzle, zero fill out of bounds (loads) / clipping (stores).
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dtype, uint64_t inner,
              uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, dtype, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 operand map, box {64, box_outer}
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
              uint32_t box_outer) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, inner, outer, row_bytes, 64, box_outer);
}

// ------------------------------------------------------------ tensor-core GEMM launch

// An operand in memory: `rows` x `cols` bf16, cols contiguous.
struct Operand {
  const void* ptr;
  long long rows, cols;
};

// The kernels launched between the tensor-core GEMMs ask for the largest
// shared-memory carveout, the configuration the GEMMs need, so the SMs keep
// one L1 / shared-memory split through a whole step instead of switching it
// at kernel boundaries.  Once per call site (kernel) and device; a refusal
// only leaves the default preference.
#define SAMBAY_MAX_CARVEOUT(kern, dev)                                                  \
  do {                                                                                  \
    static bool done_[kMaxDevices] = {};                                                \
    if (!done_[dev]) {                                                                  \
      if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,    \
                               cudaSharedmemCarveoutMaxShared) != cudaSuccess)          \
        (void)cudaGetLastError();                                                       \
      done_[dev] = true;                                                                \
    }                                                                                   \
  } while (0)

// Kernel launch with an optional cluster size and, for `chained` launches,
// programmatic dependent launch: used for every kernel of an entry point
// after its first, whose predecessor on the stream is then one of this
// library's kernels.  Such a kernel may start (set-up, CTA launch) while its
// predecessor finishes; each kernel waits for its predecessor (pdl_wait)
// before touching global memory.  The first kernel of a call is launched
// plainly and so orders after whatever the caller queued before.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     bool chained, int cluster, Args... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute at[2];
  unsigned n = 0;
  if (cluster > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = cluster;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = 1;
    ++n;
  }
  if (chained) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  lc.attrs = at;
  lc.numAttrs = n;
  return cudaLaunchKernelEx(&lc, kern, args...);
}

// Blocks for a grid-stride launch of `threads` threads: enough to cover
// them, at most 16 per SM.
int grid_for(long long threads, int block, int sms) {
  const long long g = (threads + block - 1) / block;
  return static_cast<int>(std::max(1LL, std::min(g, static_cast<long long>(sms) * 16)));
}

// Last-wave balancing of a GEMM without K split: with W whole waves of
// tiles over the SMs and a partial wave of `tail` tiles, the tail tiles are
// cut along N into nsplit units (64 columns at the narrowest) so they spread
// over up to all SMs instead of running on `tail` of them.
struct TailPlan {
  int full, nsplit;
};

TailPlan tail_plan(int tiles, int BN, int slots, int min_width) {
  TailPlan tp{tiles, 1};
  const int waves = tiles / slots, tail = tiles % slots;
  if (waves == 0 || tail == 0) return tp;
  for (int cand = BN / min_width; cand >= 2; cand /= 2)
    if (BN % (cand * min_width) == 0 && tail * cand <= slots) {
      tp.full = waves * slots;
      tp.nsplit = cand;
      break;
    }
  return tp;
}

// K-split tail (pairs only): the partial wave's `ntail` tiles are each cut
// along K into `splits` units of `kbps` k-blocks (ntail * splits <= slots);
// every unit writes an fp32 partial tile; the GEMM's CTAs sum them in a fixed
// order after their last unit and apply the epilogue.
struct KTailPlan {
  int ntail = 0, splits = 1, kbps = 0;
};

KTailPlan ktail_plan(int tiles, int slots, int k_blocks) {
  KTailPlan kp;
  const int waves = tiles / slots, tail = tiles % slots;
  if (waves == 0 || tail == 0) return kp;
  const int s = std::min({slots / tail, k_blocks, sambay::tc::kMaxTailSplits});
  if (s < 2) return kp;
  kp.kbps = (k_blocks + s - 1) / s;
  kp.splits = (k_blocks + kp.kbps - 1) / kp.kbps;
  if (kp.splits >= 2) kp.ntail = tail;
  return kp;
}

// Whether `count` clusters of `s` CTAs of this (non-pair) configuration are
// co-resident on the device; cached per device and cluster size.
template <int BN, bool A_MN, bool B_MN, int KIND, bool TRANS, int EW>
bool cluster_fits(int dev, int sms, int s, int count) {
  using namespace sambay::tc;
  using C = Cfg<BN, A_MN, B_MN, KIND, TRANS, EW, false>;
  static int active[kMaxDevices][9] = {};
  if (active[dev][s] == 0) {
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(s * (sms / s));
    q.blockDim = dim3(gemm_threads(EW));
    q.dynamicSmemBytes = C::kSmem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = s;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    q.attrs = at;
    q.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_kernel<BN, A_MN, B_MN, KIND, TRANS, EW, false>, &q) !=
            cudaSuccess)
      n = -1;
    active[dev][s] = n > 0 ? n : -1;
  }
  return active[dev][s] >= count;
}

// `splits` > 1 splits K into that many contiguous ranges (as computed by
// split_count for the same sizes); `chained`: launched with programmatic
// dependent launch after this library's previous kernel (launch_k);
// `balance_tail` (no K split) applies
// tail_plan, or for pairs with `tail_part` scratch of `tail_bytes` the
// K-split tail when that leaves the shorter last round (a tail unit costs
// 1/splits of a tile plus about a tenth of one for its partial tile and its
// share of the reduction, which the same kernel's CTAs do after their last
// unit).  PAIR: 256-row tiles on CTA pairs (clusters of two).
template <int BN, bool A_MN, bool B_MN, int KIND, bool TRANS, int EW = 4, bool PAIR = false>
sambay_status run_tc(const char* name, int dev, int sms, Operand a, Operand b,
                     sambay::tc::GemmArgs g, int splits, cudaStream_t st, bool chained, bool balance_tail = false,
                     float* tail_part = nullptr, size_t tail_bytes = 0) {
  using namespace sambay::tc;
  using C = Cfg<BN, A_MN, B_MN, KIND, TRANS, EW, PAIR>;
  static bool attr_set[kMaxDevices] = {};
  static int pair_slots[kMaxDevices] = {};   // co-resident clusters of two (PAIR)
  auto kern = tc_gemm_kernel<BN, A_MN, B_MN, KIND, TRANS, EW, PAIR>;
  SAMBAY_MAX_CARVEOUT(kern, dev);
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(C::kSmem)) != cudaSuccess)
      return SAMBAY_ERR_CUDA;
    if (PAIR) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(2 * (sms / 2));
      q.blockDim = dim3(gemm_threads(EW));
      q.dynamicSmemBytes = C::kSmem;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      q.attrs = at;
      q.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n < 1) return SAMBAY_ERR_CUDA;
      pair_slots[dev] = n;
    }
    attr_set[dev] = true;
  }
  CUtensorMap ta, tb;
  // A K-major: [M, K] -> box {64 k, 128 m};  MN-major: [K, M] -> box {64 m, 64 k}
  // B K-major: [N, K] -> box {64 k, kBHalf n} (a pair's CTA loads half the tile's columns)
  if (!make_map(&ta, a.ptr, a.cols, a.rows, a.cols * 2, A_MN ? 64 : BM)) return SAMBAY_ERR_CUDA;
  if (!make_map(&tb, b.ptr, b.cols, b.rows, b.cols * 2, B_MN ? 64 : C::kBHalf)) return SAMBAY_ERR_CUDA;
  // row-major epilogue through TMA when the output columns come in whole
  // blocks: bf16 outputs in 64-column blocks (aux in 128 x 64 boxes, stores in
  // 32 x 64 boxes per warp), f32 outputs in 32 x 32 boxes
  CUtensorMap taux, tout;
  std::memset(&taux, 0, sizeof(taux));
  std::memset(&tout, 0, sizeof(tout));
  g.tma_epi = 0;
  if (C::kTmaEpi && g.ldo % 8 == 0) {
    const bool f32 = KIND == sambay::tc::EPI_SOFTPLUS;
    if (g.N % (f32 ? 32 : 64) == 0) {
      const uint64_t eb = f32 ? 4 : 2;
      bool okm = make_map(&tout, g.out, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                          g.N, g.M, g.ldo * eb, f32 ? 32 : 64, 32);
      if (okm && g.aux != nullptr && !f32)
        okm = make_map(&taux, g.aux, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.N, g.M, g.ldo * 2, 64, BM);
      if (!okm) return SAMBAY_ERR_CUDA;
      g.tma_epi = 1;
    }
  }
  g.m_tiles = (g.M + C::kBMT - 1) / C::kBMT;
  g.n_tiles = (g.N + BN - 1) / BN;
  g.k_blocks = (g.K + BK - 1) / BK;
  if (g.csplit) {
    // cluster split-K: the most splits (<= `splits`) whose clusters of that
    // many CTAs all fit on the GPU at once, about one CTA per SM in total
    const int tiles = g.m_tiles * g.n_tiles;
    int best = 1;
    for (int s = std::min({splits, g.k_blocks, 8}); s >= 2; --s) {
      if (static_cast<long long>(tiles) * s > sms) continue;
      if (cluster_fits<BN, A_MN, B_MN, KIND, TRANS, EW>(dev, sms, s, tiles)) { best = s; break; }
    }
    splits = best;
    if (splits == 1) g.csplit = 0;
  }
  splits = std::max(1, std::min(splits, g.k_blocks));
  g.kb_per_split = (g.k_blocks + splits - 1) / splits;
  g.splits = (g.k_blocks + g.kb_per_split - 1) / g.kb_per_split;
  if (g.splits == 1) g.csplit = 0;
  g.tiles = g.m_tiles * g.n_tiles * g.splits;
  g.full_tiles = g.tiles;
  g.tail_nsplit = 1;
  CUtensorMap tb2 = tb;
  g.tail_ksplit = 1;
  const int slots = PAIR ? pair_slots[dev] : sms;   // work units in flight at once
  if (balance_tail && g.splits == 1) {
    // narrowest unit: 64 columns per CTA's B load (MN-major B: whole 64-column boxes)
    const int min_width = (PAIR && B_MN) ? 128 : 64;
    const TailPlan tp = tail_plan(g.tiles, BN, slots, min_width);
    // (the kernel sums a K-split tail only in its bf16 gate / residual epilogues)
    constexpr bool kTailKind = KIND == sambay::tc::EPI_GATE || KIND == sambay::tc::EPI_RESID;
    const KTailPlan kp = PAIR && kTailKind && tail_part ? ktail_plan(g.tiles, slots, g.k_blocks) : KTailPlan{};
    const double ncost = 1.0 / tp.nsplit, kcost = 1.0 / kp.splits + 0.1;
    if (kp.ntail > 0 && kcost < ncost &&
        static_cast<size_t>(kp.ntail) * kp.splits * C::kBMT * BN * 4 + kTailSyncBytes <= tail_bytes &&
        static_cast<size_t>(kp.ntail) * kp.splits * 2 * sizeof(unsigned long long) <= kTailSyncBytes) {
      g.full_tiles = g.tiles - kp.ntail;
      g.tail_ksplit = kp.splits;
      g.tail_kbps = kp.kbps;
      g.tail_part = tail_part;
      g.tail_flags = reinterpret_cast<unsigned long long*>(reinterpret_cast<uint8_t*>(tail_part) + tail_bytes -
                                                           kTailSyncBytes);
      g.tail_epoch = next_tail_epoch();
      g.tiles = g.full_tiles + kp.ntail * kp.splits;
    } else if (tp.nsplit > 1) {
      const int hb = (BN / tp.nsplit) / (PAIR ? 2 : 1);
      if (!B_MN && !make_map(&tb2, b.ptr, b.cols, b.rows, b.cols * 2, hb)) return SAMBAY_ERR_CUDA;
      g.tiles = tp.full + (g.tiles - tp.full) * tp.nsplit;
      g.full_tiles = tp.full;
      g.tail_nsplit = tp.nsplit;
    }
  }
  const int units = std::min(g.tiles, slots);
  {
    ProfScope ps(name, st);
    // PAIR: one unit per cluster of two; cluster split-K: one cluster of
    // `splits` CTAs per tile; otherwise one unit per CTA
    const int grid = PAIR ? 2 * units : g.csplit ? g.tiles : units;
    const int cluster = PAIR ? 2 : g.csplit ? g.splits : 1;
    if (launch_k(kern, dim3(grid), dim3(gemm_threads(EW)), C::kSmem, st, chained, cluster, ta, tb, tb2, taux,
                 tout, g) != cudaSuccess)
      return SAMBAY_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? SAMBAY_OK : SAMBAY_ERR_CUDA;
}

sambay::tc::GemmArgs tc_args(int M, int N, int K, void* out, long long ldo, const void* aux = nullptr,
                             const float* vec = nullptr, float* partials = nullptr,
                             long long split_stride = 0, int* counters = nullptr) {
  sambay::tc::GemmArgs g{};
  g.M = M;
  g.N = N;
  g.K = K;
  g.out = out;
  g.aux = aux;
  g.vec = vec;
  g.ldo = ldo;
  g.partials = partials;
  g.split_stride = split_stride;
  g.counters = counters;
  return g;
}

// ------------------------------------------------------------ fp32 GEMM launch

template <int KIND>
sambay_status run_simt(const char* name, const sambay::simt::Args& g, cudaStream_t st) {
  dim3 grid((g.N + 63) / 64, (g.M + 63) / 64);
  ProfScope ps(name, st);
  sambay::simt::simt_gemm_kernel<KIND><<<grid, 256, 0, st>>>(g);
  return cudaGetLastError() == cudaSuccess ? SAMBAY_OK : SAMBAY_ERR_CUDA;
}

sambay::simt::Args simt_args(const float* A, long long sam, long long sak, const float* B,
                             long long sbk, long long sbn, int M, int N, int K, float* out,
                             long long ldo, const float* aux = nullptr, const float* vec = nullptr) {
  sambay::simt::Args g{};
  g.A = A; g.sam = sam; g.sak = sak;
  g.B = B; g.sbk = sbk; g.sbn = sbn;
  g.M = M; g.N = N; g.K = K;
  g.out = out; g.ldo = ldo; g.aux = aux; g.vec = vec; g.trans = 0;
  return g;
}

#define SAMBAY_TRY(expr)                 \
  do {                                   \
    const sambay_status _s = (expr);     \
    if (_s != SAMBAY_OK) return _s;      \
  } while (0)

// ------------------------------------------------------------ shared scan pieces

// Which part of the projections a call runs.  A channel-sharded prefill
// stops after x_proj (PROJ_XPROJ: this shard's partial sums over its channels
// into an external xdbl), the caller sums the partials over the shards, and
// PROJ_FINISH takes the summed xdbl from there on.
enum ProjPhase { PROJ_ALL, PROJ_XPROJ, PROJ_FINISH };

// x_proj + dt_proj for `rows` tokens whose conv output is ws.uc:
//   xdbl = uc W_x^T,  dt = softplus(delta W_dt^T + b_dt)
// xdbl_ext: PROJ_XPROJ writes the (partial) xdbl there; PROJ_FINISH reads
// the summed xdbl from there (and uc is not read).
sambay_status projections(int dev, int sms, const sambay_scan_weights* w, const sambay_dims* d,
                          long long rows, uint8_t* ws, const ScanWs& L, cudaStream_t st, bool prefill,
                          ProjPhase phase = PROJ_ALL, float* xdbl_ext = nullptr) {
  const int Di = d->d_inner, R = d->dt_rank, ldx = d->dt_rank + 2 * d->d_state;
  float* xdbl = reinterpret_cast<float*>(ws + L.xdbl);
  float* dt = reinterpret_cast<float*>(ws + L.dt);
  float* bcp = prefill ? reinterpret_cast<float*>(ws + L.bcp) : nullptr;   // B | C segments: prefill only
  if (d->io == SAMBAY_BF16) {
    const bf16* uc = reinterpret_cast<const bf16*>(ws + L.uc);
    bf16* delta = reinterpret_cast<bf16*>(ws + L.delta);
    float* part = reinterpret_cast<float*>(ws + L.part);
    const long long stride = rows * ldx;
    const int Rp = rank_pad(R);
    if (phase != PROJ_FINISH) {
      // x_proj = [uc_hi | uc_lo] [W_x | W_x]^T, split over K: each split writes
      // its partial [rows, ldx] tile set
      auto gx = tc_args(static_cast<int>(rows), ldx, 2 * Di, part, ldx, nullptr, nullptr, nullptr, stride);
      gx.b_k_wrap = Di;
      const Operand a_uc{uc, rows, 2LL * Di}, b_wx{w->x_proj_w, ldx, Di};
      constexpr int P = sambay::tc::EPI_F32_PARTIAL;
      if (rows > 256 && ldx > 128 && ldx <= 192) {
        // prefill: 256-row tiles on CTA pairs, each CTA loading half of the
        // W_x tile (the splits' K ranges as in the single-CTA form)
        SAMBAY_TRY((run_tc<192, false, false, P, false, 4, true>("x_proj", dev, sms, a_uc, b_wx, gx, L.splits, st, true)));
      } else if (ldx <= 64) SAMBAY_TRY((run_tc<64, false, false, P, false>("x_proj", dev, sms, a_uc, b_wx, gx, L.splits, st, true)));
      else if (ldx <= 128) SAMBAY_TRY((run_tc<128, false, false, P, false>("x_proj", dev, sms, a_uc, b_wx, gx, L.splits, st, true)));
      else if (ldx <= 192) SAMBAY_TRY((run_tc<192, false, false, P, false>("x_proj", dev, sms, a_uc, b_wx, gx, L.splits, st, true)));
      else SAMBAY_TRY((run_tc<256, false, false, P, false>("x_proj", dev, sms, a_uc, b_wx, gx, L.splits, st, true)));
    }
    {
      // the split sums in a fixed order -> xdbl, the split delta and B | C
      // pairs; PROJ_XPROJ: xdbl only (into xdbl_ext); PROJ_FINISH: the summed
      // xdbl_ext is the single "split"
      auto k8 = sambay::scan::xdbl_reduce_kernel<8>;
      auto k1 = sambay::scan::xdbl_reduce_kernel<1>;
      SAMBAY_MAX_CARVEOUT(k8, dev);
      SAMBAY_MAX_CARVEOUT(k1, dev);
      const int Lseq = static_cast<int>(rows / d->batch), nrows = static_cast<int>(rows);
      const float* src = phase == PROJ_FINISH ? xdbl_ext : part;
      const int nsplit = phase == PROJ_FINISH ? 1 : L.splits;
      float* dst = phase == PROJ_XPROJ ? xdbl_ext : xdbl;
      bf16* dl = phase == PROJ_XPROJ ? nullptr : delta;
      float* bp = phase == PROJ_XPROJ ? nullptr : bcp;
      ProfScope ps_reduce("xdbl_reduce", st);
      const bool many = nsplit >= 16;
      if (launch_k(many ? k8 : k1, dim3(grid_for(stride / 4 * (many ? 8 : 1), 256, sms)), dim3(256), 0, st, true, 1,
                   src, nsplit, stride, dst, dl, bp, Lseq, nrows, R, Rp, ldx) != cudaSuccess)
        return SAMBAY_ERR_CUDA;
    }
    if (cudaGetLastError() != cudaSuccess) return SAMBAY_ERR_CUDA;
    if (phase == PROJ_XPROJ) return SAMBAY_OK;
    // dt = softplus([delta_hi | delta_lo] [W_dt | W_dt]^T + b_dt); each half of
    // the A operand is padded with zeros to Rp, W_dt reads zeros past R
    auto gd = tc_args(static_cast<int>(rows), Di, 2 * Rp, dt, Di, nullptr, w->dt_bias);
    gd.b_k_wrap = Rp;
    const Operand a_d{delta, rows, 2LL * Rp}, b_wdt{w->dt_proj_w, Di, R};
    if (rows <= sambay::tc::BM)   // one row tile (decode): narrower tiles, more CTAs
      SAMBAY_TRY((run_tc<64, false, false, sambay::tc::EPI_SOFTPLUS, false>("dt_proj", dev, sms, a_d, b_wdt, gd, 1, st, true)));
    else
      SAMBAY_TRY((run_tc<256, false, false, sambay::tc::EPI_SOFTPLUS, false, 8>("dt_proj", dev, sms, a_d, b_wdt, gd, 1, st, true, true)));
  } else {
    const float* uc = reinterpret_cast<const float*>(ws + L.uc);
    if (phase != PROJ_FINISH) {
      float* dst = phase == PROJ_XPROJ ? xdbl_ext : xdbl;
      SAMBAY_TRY(run_simt<sambay::simt::F32_STORE>("x_proj_f32",
          simt_args(uc, Di, 1, static_cast<const float*>(w->x_proj_w), 1, Di, static_cast<int>(rows),
                    ldx, Di, dst, ldx),
          st));
      if (phase == PROJ_XPROJ) return SAMBAY_OK;
    }
    const float* xs = phase == PROJ_FINISH ? xdbl_ext : xdbl;
    if (prefill) {
      ProfScope ps_bc("bc_pairs", st);
      sambay::scan::bc_pairs_kernel<<<grid_for(rows * 2 * d->d_state, 256, 1 << 20), 256, 0, st>>>(
          xs, bcp, static_cast<int>(rows / d->batch), static_cast<int>(rows), R, ldx);
      if (cudaGetLastError() != cudaSuccess) return SAMBAY_ERR_CUDA;
    }
    SAMBAY_TRY(run_simt<sambay::simt::SOFTPLUS>("dt_proj_f32",
        simt_args(xs, ldx, 1, static_cast<const float*>(w->dt_proj_w), 1, R,
                  static_cast<int>(rows), Di, R, dt, Di, nullptr, w->dt_bias),
        st));
  }
  return SAMBAY_OK;
}

// Channel runs of the prefill scan: CTAs per sequence (nblk) chosen so the
// busiest SM carries the fewest channels, i.e. minimising
// ceil(B * nblk / sms) * ceil(quads / nblk) over runs of at most kScanMaxCH
// channels (ties: fewer, larger CTAs).  The split changes only which CTA
// computes a channel, never its arithmetic.
template <typename T>
void scan_partition(sambay::scan::ScanParams<T>& p, int sms) {
  using namespace sambay::scan;
  const long long quads = p.Di / 4;
  const long long lo = (quads + kScanMaxCH / 4 - 1) / (kScanMaxCH / 4);
  long long best = lo, best_cost = -1;
  for (long long nblk = lo; nblk <= quads; ++nblk) {
    const long long cost = ((static_cast<long long>(p.B) * nblk + sms - 1) / sms) * ((quads + nblk - 1) / nblk);
    if (best_cost < 0 || cost < best_cost) { best = nblk; best_cost = cost; }
  }
  p.nblk = static_cast<int>(best);
  p.q_base = static_cast<int>(quads / best);
  p.q_extra = static_cast<int>(quads % best);
  p.chp = 4 * (p.q_base + (p.q_extra ? 1 : 0));
}

template <typename T>
sambay_status launch_scan(int dev, int sms, sambay::scan::ScanParams<T>& p, cudaStream_t st) {
  using namespace sambay::scan;
  auto kern = selective_scan_kernel<T>;
  // Two CTAs fit on an SM (registers and shared memory), which hides more of
  // the recurrence's latency when the grid has more CTAs than SMs.  A grid of
  // at most one CTA per SM asks for more than half an SM's shared memory
  // instead, so that, launched early behind the kernel before it, its CTAs
  // cannot pair up on the SMs that free first while others stay empty.
  constexpr int kSoloSmem = 120 * 1024;
  static bool attr_set[kMaxDevices] = {};
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             std::max(ScanLayout(kScanMaxCH, sizeof(T)).bytes, kSoloSmem)) != cudaSuccess)
      return SAMBAY_ERR_CUDA;
    attr_set[dev] = true;
  }
  SAMBAY_MAX_CARVEOUT(kern, dev);
  scan_partition<T>(p, sms);
  const ScanLayout ly(p.chp, sizeof(T));
  dim3 grid(p.nblk, p.B);
  const bool solo = static_cast<long long>(p.nblk) * p.B <= sms;
  const size_t smem = solo ? std::max(ly.bytes, kSoloSmem) : static_cast<size_t>(ly.bytes);
  ProfScope ps("selective_scan", st);
  return launch_k(kern, grid, dim3(8 * p.chp), smem, st, true, 1, p) == cudaSuccess ? SAMBAY_OK
                                                                   : SAMBAY_ERR_CUDA;
}

template <typename T>
sambay_status scan_prefill_impl(int dev, int sms, const sambay_scan_weights* w,
                                const sambay_dims* d, const void* u, void* M, float* ssm_state,
                                void* conv_state, int zero_init, uint8_t* ws, cudaStream_t st,
                                ProjPhase phase = PROJ_ALL, float* xdbl_ext = nullptr) {
  const long long T_ = static_cast<long long>(d->batch) * d->seqlen;
  const ScanWs L = scan_ws_layout(d, T_);
  T* uc = reinterpret_cast<T*>(ws + L.uc);
  if (phase != PROJ_FINISH) {
    sambay::scan::ConvParams<T> p{static_cast<const T*>(u), static_cast<const T*>(conv_state),
                                  static_cast<const T*>(w->conv_w),
                                  static_cast<const T*>(w->conv_b), uc, d->batch, d->seqlen,
                                  d->d_inner, zero_init};
    using sambay::scan::kConvTT;
    auto c64 = sambay::scan::conv_silu_kernel<T, 64>;
    auto c32 = sambay::scan::conv_silu_kernel<T, 32>;
    SAMBAY_MAX_CARVEOUT(c64, dev);
    SAMBAY_MAX_CARVEOUT(c32, dev);
    ProfScope ps("conv_silu", st);
    if (d->d_inner % 64 == 0) {
      dim3 grid(d->d_inner / 64, (d->seqlen + kConvTT - 1) / kConvTT, d->batch);
      c64<<<grid, 64 / 4 * (kConvTT / 4), 0, st>>>(p);
    } else {
      dim3 grid(d->d_inner / 32, (d->seqlen + kConvTT - 1) / kConvTT, d->batch);
      c32<<<grid, 32 / 4 * (kConvTT / 4), 0, st>>>(p);
    }
    if (cudaGetLastError() != cudaSuccess) return SAMBAY_ERR_CUDA;
  }
  SAMBAY_TRY(projections(dev, sms, w, d, T_, ws, L, st, true, phase, xdbl_ext));
  if (phase == PROJ_XPROJ) return SAMBAY_OK;
  {
    sambay::scan::ScanParams<T> p{};
    p.uc = uc;
    p.dt = reinterpret_cast<const float*>(ws + L.dt);
    p.bcp = reinterpret_cast<const float*>(ws + L.bcp);
    p.A = w->A;
    p.D = w->D;
    p.u = static_cast<const T*>(u);
    p.h = ssm_state;
    p.conv_state = static_cast<T*>(conv_state);
    p.M = static_cast<T*>(M);
    p.B = d->batch;
    p.L = d->seqlen;
    p.Di = d->d_inner;
    p.zero_init = zero_init;
    SAMBAY_TRY(launch_scan<T>(dev, sms, p, st));
    if (cudaGetLastError() != cudaSuccess) return SAMBAY_ERR_CUDA;
  }
  return SAMBAY_OK;
}

sambay_status scan_step_fused(int dev, int sms, const sambay_scan_weights* w, const sambay_dims* d,
                              const StepPlan& sp, const void* u_t, void* m_t, float* ssm_state,
                              void* conv_state, uint8_t* ws, cudaStream_t st) {
  auto kproj = sambay::step::step_proj_kernel;
  auto kred = sambay::step::step_reduce_kernel;
  auto kscan = sambay::step::step_scan_kernel;
  auto kfused = sambay::step::step_fused_kernel;
  static bool attr_set[kMaxDevices] = {};
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kscan, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(kfused, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmemBytes) != cudaSuccess)
      return SAMBAY_ERR_CUDA;
    attr_set[dev] = true;
  }
  SAMBAY_MAX_CARVEOUT(kproj, dev);
  SAMBAY_MAX_CARVEOUT(kred, dev);
  SAMBAY_MAX_CARVEOUT(kscan, dev);
  const StepWs L = step_ws_layout(d, sp);
  sambay::step::StepParams p{};
  p.u_t = static_cast<const bf16*>(u_t);
  p.conv_state = static_cast<bf16*>(conv_state);
  p.conv_w = static_cast<const bf16*>(w->conv_w);
  p.conv_b = static_cast<const bf16*>(w->conv_b);
  p.x_proj_w = static_cast<const bf16*>(w->x_proj_w);
  p.dt_proj_w = static_cast<const bf16*>(w->dt_proj_w);
  p.dt_bias = w->dt_bias;
  p.A = w->A;
  p.D = w->D;
  p.h = ssm_state;
  p.m_t = static_cast<bf16*>(m_t);
  p.uc = reinterpret_cast<float*>(ws + L.uc);
  p.part = reinterpret_cast<float*>(ws + L.part);
  p.dts = reinterpret_cast<bf16*>(ws + L.dts);
  p.bc = reinterpret_cast<float*>(ws + L.bc);
  p.bar = reinterpret_cast<unsigned long long*>(ws + L.bar);
  p.wait_limit = sambay::tc::kWaitCycles;
  p.B = d->batch;
  p.Di = d->d_inner;
  p.R = d->dt_rank;
  p.Rp = sp.Rp;
  p.ldx = d->dt_rank + 2 * d->d_state;
  p.chan = sp.chan;
  p.nslice = sp.nslice;
  p.group = sp.group;
  if (sp.fused && sp.nslice <= sms && sp.nslice <= sambay::step::kMaxMeetCtas) {
    // one kernel; cooperative, so its CTAs (one per slice) are all resident at
    // once, which its grid-wide meeting points need.  The state h viewed as
    // [B][Di / 8][128 floats]: a CTA's slice is the box {128, chan / 8, B}.
    SAMBAY_MAX_CARVEOUT(kfused, dev);
    EncodeTiledFn fn = encode_fn();
    CUtensorMap hmap;
    {
      const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(d->d_inner / 8), static_cast<cuuint64_t>(d->batch)};
      const cuuint64_t strides[2] = {512, static_cast<cuuint64_t>(d->d_inner) * 64};
      const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(sp.chan / 8), static_cast<cuuint32_t>(d->batch)};
      const cuuint32_t es[3] = {1, 1, 1};
      if (!fn || fn(&hmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ssm_state, dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return SAMBAY_ERR_CUDA;
    }
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(sp.nslice);
    lc.blockDim = dim3(sambay::step::kFusedThreads);
    lc.dynamicSmemBytes = sp.fused_smem;
    lc.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    ProfScope ps("step_fused", st);
    return cudaLaunchKernelEx(&lc, kfused, p, hmap) == cudaSuccess ? SAMBAY_OK : SAMBAY_ERR_CUDA;
  }
  const dim3 grid(sp.nslice, (d->batch + sp.group - 1) / sp.group);
  const dim3 block(sambay::step::kThreads);
  {
    ProfScope ps("step_proj", st);
    if (launch_k(kproj, grid, block, 0, st, false, 1, p) != cudaSuccess) return SAMBAY_ERR_CUDA;
  }
  {
    const long long outs = static_cast<long long>(p.ldx) * p.B * sambay::step::kRedLanes;
    ProfScope ps("step_reduce", st);
    if (launch_k(kred, dim3(grid_for(outs, sambay::step::kThreads, sms)), block, 0, st, true, 1, p) != cudaSuccess)
      return SAMBAY_ERR_CUDA;
  }
  ProfScope ps("step_scan", st);
  return launch_k(kscan, grid, block, sp.smem, st, true, 1, p) == cudaSuccess ? SAMBAY_OK : SAMBAY_ERR_CUDA;
}

template <typename T>
sambay_status scan_step_impl(int dev, int sms, const sambay_scan_weights* w, const sambay_dims* d,
                             const void* u_t, void* m_t, float* ssm_state, void* conv_state,
                             uint8_t* ws, cudaStream_t st) {
  const long long B = d->batch;
  if (sizeof(T) == 2) {
    const StepPlan sp = step_plan(d);
    if (sp.ok) return scan_step_fused(dev, sms, w, d, sp, u_t, m_t, ssm_state, conv_state, ws, st);
  }
  const ScanWs L = scan_ws_layout(d, B, true);
  T* uc = reinterpret_cast<T*>(ws + L.uc);
  constexpr int VEC = 16 / sizeof(T);
  auto sc = sambay::scan::step_conv_kernel<T>;
  auto ss = sambay::scan::step_scan_kernel<T>;
  SAMBAY_MAX_CARVEOUT(sc, dev);
  SAMBAY_MAX_CARVEOUT(ss, dev);
  {
    ProfScope ps("step_conv", st);
    sc<<<grid_for(B * (d->d_inner / VEC), 256, 1 << 20), 256, 0, st>>>(
      static_cast<const T*>(u_t), static_cast<T*>(conv_state), static_cast<const T*>(w->conv_w),
      static_cast<const T*>(w->conv_b), uc, d->batch, d->d_inner);
  }
  if (cudaGetLastError() != cudaSuccess) return SAMBAY_ERR_CUDA;
  SAMBAY_TRY(projections(dev, sms, w, d, B, ws, L, st, false));
  ProfScope ps("step_scan", st);
  const cudaError_t e = launch_k(ss, dim3(grid_for(B * d->d_inner * 4, 256, 1 << 20)), dim3(256), 0, st, true, 1,
                                 static_cast<const T*>(uc), reinterpret_cast<const float*>(ws + L.dt),
                                 reinterpret_cast<const float*>(ws + L.xdbl), static_cast<const float*>(w->A),
                                 static_cast<const float*>(w->D), ssm_state, static_cast<T*>(m_t),
                                 static_cast<int>(d->batch), static_cast<int>(d->d_inner),
                                 static_cast<int>(d->dt_rank), static_cast<int>(d->dt_rank + 2 * d->d_state));
  return e == cudaSuccess ? SAMBAY_OK : SAMBAY_ERR_CUDA;
}

// ------------------------------------------------------------ GMU

sambay_status gmu_f32(const sambay_dims* d, long long rows, const void* X, const void* M,
                      const void* W1, const void* W2, const void* residual, void* Y, uint8_t* ws,
                      const GmuWs& L, cudaStream_t st) {
  const int Dm = d->d_model, Di = d->d_inner;
  float* H = reinterpret_cast<float*>(ws + L.h);
  SAMBAY_TRY(run_simt<sambay::simt::GATE>("gmu_gate_f32",
      simt_args(static_cast<const float*>(X), Dm, 1, static_cast<const float*>(W1), 1, Dm,
                static_cast<int>(rows), Di, Dm, H, Di, static_cast<const float*>(M)),
      st));
  SAMBAY_TRY(run_simt<sambay::simt::RESID>("gmu_out_f32",
      simt_args(H, Di, 1, static_cast<const float*>(W2), Dm, 1, static_cast<int>(rows), Dm, Di,
                static_cast<float*>(Y), Dm, static_cast<const float*>(residual)),
      st));
  return SAMBAY_OK;
}

// Y = io(Ysum + residual) over n elements (residual may be null); 4 per
// thread (n is a multiple of 4: d_model is)
template <typename T>
__global__ void __launch_bounds__(256) gmu_finish_kernel(const float* __restrict__ Ysum,
                                                         const T* __restrict__ residual, T* __restrict__ Y,
                                                         long long n4) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 v = reinterpret_cast<const float4*>(Ysum)[i];
    if (residual != nullptr) {
      v.x += sambay::to_f32(residual[4 * i]);
      v.y += sambay::to_f32(residual[4 * i + 1]);
      v.z += sambay::to_f32(residual[4 * i + 2]);
      v.w += sambay::to_f32(residual[4 * i + 3]);
    }
    Y[4 * i] = sambay::from_f32<T>(v.x);
    Y[4 * i + 1] = sambay::from_f32<T>(v.y);
    Y[4 * i + 2] = sambay::from_f32<T>(v.z);
    Y[4 * i + 3] = sambay::from_f32<T>(v.w);
  }
}

sambay_status gmu_common_checks(const sambay_dims* d, int64_t rows, const void* X, const void* M,
                                const void* W1, const void* W2, const void* residual, void* Y) {
  SAMBAY_TRY(check_dims(d, true, false));
  if (rows < 1 || rows > (1LL << 30)) return SAMBAY_ERR_INVALID_ARG;
  SAMBAY_TRY(check_ptrs({X, M, W1, W2, Y}));
  if (residual && !aligned16(residual)) return SAMBAY_ERR_UNSUPPORTED;
  if (Y == M || (Y == X && X != residual)) return SAMBAY_ERR_INVALID_ARG;
  return SAMBAY_OK;
}

// Y [rows, N] = X [rows, K] W^T, W [N, K] (bf16): KIND = EPI_RESID with no aux
// is the plain projection, KIND = EPI_GATE gives Y = aux ⊙ SiLU(X W^T).  Up to
// 256 rows it is the swap-AB decode GEMM (W is the A operand and streams once,
// split-K over a cluster, reduced through distributed shared memory);
// otherwise the CTA-pair GEMM, whose last round of tiles may be split along K
// into `tail`.
template <int KIND>
sambay_status project_tc(int dev, int sms, long long rows, int N, int K, const void* X, const void* W,
                         const void* aux, void* Y, float* tail, size_t tail_bytes, const char* name,
                         cudaStream_t st) {
  if (rows <= kStepMaxRows) {
    auto g = tc_args(N, static_cast<int>(rows), K, Y, N, aux);
    g.csplit = 1;
    const Operand w{W, N, K}, x{X, rows, K};
    if (rows <= 32) return run_tc<32, false, false, KIND, true>(name, dev, sms, w, x, g, kStepMaxSplits, st, false);
    if (rows <= 64) return run_tc<64, false, false, KIND, true>(name, dev, sms, w, x, g, kStepMaxSplits, st, false);
    if (rows <= 128) return run_tc<128, false, false, KIND, true>(name, dev, sms, w, x, g, kStepMaxSplits, st, false);
    if (rows <= 192) return run_tc<192, false, false, KIND, true>(name, dev, sms, w, x, g, kStepMaxSplits, st, false);
    return run_tc<256, false, false, KIND, true>(name, dev, sms, w, x, g, kStepMaxSplits, st, false);
  }
  return run_tc<256, false, false, KIND, false, 8, true>(name, dev, sms, Operand{X, rows, K}, Operand{W, N, K},
                                                         tc_args(static_cast<int>(rows), N, K, Y, N, aux), 1, st,
                                                         false, true, tail, tail_bytes);
}

// Workspace of the projections: the K-split tail's partial tiles (more than
// 256 rows), after an optional [rows, N] io buffer.
struct ProjWs {
  size_t buf, tail, tail_bytes, total;
};

ProjWs proj_ws_layout(const sambay_dims* d, long long rows, bool buffer) {
  ProjWs w{};
  size_t off = 0;
  w.buf = off;
  if (buffer) off += round256(static_cast<size_t>(rows) * d->d_inner * io_bytes(d->io));
  if (d->io == SAMBAY_BF16 && rows > kStepMaxRows) {
    w.tail = off;
    w.tail_bytes = static_cast<size_t>(kTailUnits) * 256 * 256 * 4 + kTailSyncBytes;
    off += round256(w.tail_bytes);
  }
  w.total = off;
  return w;
}

// How a decode GMU layer's kernels chain onto the work before them.
struct StepChain {
  bool chained = false;      // the gate GEMM follows a kernel of this call (PDL)
  bool x_independent = false;  // ... which does not write X: the whole gate main loop may start early
  unsigned long long wait_limit = 0;
  int stall_test = 0;
};

// Decode GMU, bf16: H^T = SiLU(W1 X^T) ⊙ M^T, then Y^T = W2^T H^T (+ residual^T)
// as swap-AB tensor-core GEMMs whose weights are the A operand and stream
// once.  Split-K over clusters of CTAs (csplit): each split keeps its partial
// tile in shared memory; after a cluster barrier each CTA sums a slice of the
// tile's rows over the cluster (distributed shared memory).  The out GEMM is
// launched with programmatic dependent launch and loads its first W2 tiles
// before waiting for the gate GEMM.
sambay_status gmu_step_tc(int dev, int sms, const sambay_dims* d, int64_t rows, const void* X, const void* M,
                          const void* W1, const void* W2, const void* residual, void* Y, uint8_t* Hbuf,
                          const StepChain& ch, cudaStream_t st) {
  const int Dm = d->d_model, Di = d->d_inner, Bn = static_cast<int>(rows);
  bf16* H = reinterpret_cast<bf16*>(Hbuf);
  auto g1 = tc_args(Di, Bn, Dm, H, Di, M);
  auto g2 = tc_args(Dm, Bn, Di, Y, Dm, residual);
  g1.csplit = g2.csplit = 1;
  g1.a_early = ch.chained ? 1 : 0;
  g1.b_early = (ch.chained && ch.x_independent) ? 1 : 0;
  g2.a_early = 1;
  g1.wait_limit = g2.wait_limit = ch.wait_limit;
  g1.stall_test = g2.stall_test = ch.stall_test;
  const Operand w1{W1, Di, Dm}, xr{X, rows, Dm}, w2{W2, Di, Dm}, hr{H, rows, Di};
#define SAMBAY_STEP_GEMMS(BNV)                                                                              \
  SAMBAY_TRY((run_tc<BNV, false, false, sambay::tc::EPI_GATE, true>("gmu_step_gate", dev, sms, w1, xr, g1,   \
                                                                    kStepMaxSplits, st, ch.chained)));       \
  SAMBAY_TRY((run_tc<BNV, true, false, sambay::tc::EPI_RESID, true>("gmu_step_out", dev, sms, w2, hr, g2,    \
                                                                    kStepMaxSplits, st, true)));
  if (Bn <= 32) { SAMBAY_STEP_GEMMS(32) }
  else if (Bn <= 64) { SAMBAY_STEP_GEMMS(64) }
  else if (Bn <= 128) { SAMBAY_STEP_GEMMS(128) }
  else if (Bn <= 192) { SAMBAY_STEP_GEMMS(192) }
  else { SAMBAY_STEP_GEMMS(256) }
#undef SAMBAY_STEP_GEMMS
  return SAMBAY_OK;
}

}  // namespace

// Scratch of sambay_scan_step_noalloc: a fixed array compiled into the
// library, for callers that cannot allocate device memory.  Host code must
// not pass this symbol to a kernel directly (on the host it names a host-side
// stand-in); its device address is looked up per device with
// cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SAMBAY_NOALLOC_SCRATCH_BYTES];

namespace {
// device address of g_noalloc_scratch, per device; host threads racing on a
// device's first call both store the same value
std::atomic<void*> g_noalloc_ptr[kMaxDevices];
}  // namespace

// ====================================================================== C ABI

extern "C" {

const char* sambay_status_string(sambay_status s) {
  switch (s) {
    case SAMBAY_OK: return "ok";
    case SAMBAY_ERR_INVALID_ARG: return "invalid argument";
    case SAMBAY_ERR_UNSUPPORTED: return "unsupported size or alignment";
    case SAMBAY_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SAMBAY_ERR_CUDA: return "CUDA call failed";
    case SAMBAY_ERR_TIMEOUT: return "a kernel's bounded wait ran out";
    case SAMBAY_ERR_DEVICE: return "no sm_100 device current";
  }
  return "unknown status";
}

const char* sambay_version(void) { return "0.1.0"; }

size_t sambay_scan_prefill_workspace(const sambay_dims* d) {
  if (check_dims(d, false, true) != SAMBAY_OK) return 0;
  return scan_ws_layout(d, static_cast<long long>(d->batch) * d->seqlen).total;
}

size_t sambay_scan_step_workspace(const sambay_dims* d) {
  if (!d) return 0;
  sambay_dims e = *d;
  e.seqlen = 1;
  if (check_dims(&e, false, true) != SAMBAY_OK) return 0;
  return scan_ws_layout(&e, e.batch, true).total;
}

size_t gmu_forward_workspace(const sambay_dims* d, int64_t rows) {
  if (check_dims(d, true, false) != SAMBAY_OK || rows < 1) return 0;
  return gmu_ws_layout(d, rows, false).total;
}

size_t gmu_step_workspace(const sambay_dims* d, int64_t rows) {
  if (check_dims(d, true, false) != SAMBAY_OK || rows < 1 || rows > kStepMaxRows) return 0;
  return gmu_ws_layout(d, rows, true).total;
}

sambay_status sambay_scan_prefill(const sambay_scan_weights* w, const sambay_dims* d, const void* u,
                                  void* M, float* ssm_state, void* conv_state, int zero_init_state,
                                  void* ws, size_t ws_bytes, sambay_stream_t stream) {
  SAMBAY_TRY(check_dims(d, false, true));
  SAMBAY_TRY(check_weights(w));
  SAMBAY_TRY(check_ptrs({u, M, ssm_state, conv_state}));
  if (M == u) return SAMBAY_ERR_INVALID_ARG;
  const size_t need = sambay_scan_prefill_workspace(d);
  SAMBAY_TRY(check_ws(ws, ws_bytes, need));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int zi = zero_init_state ? 1 : 0;
  if (d->io == SAMBAY_BF16)
    return scan_prefill_impl<bf16>(dev, sms, w, d, u, M, ssm_state, conv_state, zi, w8, st);
  return scan_prefill_impl<float>(dev, sms, w, d, u, M, ssm_state, conv_state, zi, w8, st);
}

sambay_status sambay_scan_prefill_xproj(const sambay_scan_weights* w, const sambay_dims* d, const void* u,
                                        const void* conv_state, int zero_init_state, float* xdbl, void* ws,
                                        size_t ws_bytes, sambay_stream_t stream) {
  SAMBAY_TRY(check_dims(d, false, true));
  SAMBAY_TRY(check_weights(w));
  SAMBAY_TRY(check_ptrs({u, conv_state, xdbl}));
  SAMBAY_TRY(check_ws(ws, ws_bytes, sambay_scan_prefill_workspace(d)));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int zi = zero_init_state ? 1 : 0;
  void* cs = const_cast<void*>(conv_state);   // read only in this phase
  if (d->io == SAMBAY_BF16)
    return scan_prefill_impl<bf16>(dev, sms, w, d, u, nullptr, nullptr, cs, zi, w8, st, PROJ_XPROJ, xdbl);
  return scan_prefill_impl<float>(dev, sms, w, d, u, nullptr, nullptr, cs, zi, w8, st, PROJ_XPROJ, xdbl);
}

sambay_status sambay_scan_prefill_finish(const sambay_scan_weights* w, const sambay_dims* d, const void* u,
                                         const float* xdbl, void* M, float* ssm_state, void* conv_state,
                                         int zero_init_state, void* ws, size_t ws_bytes, sambay_stream_t stream) {
  SAMBAY_TRY(check_dims(d, false, true));
  SAMBAY_TRY(check_weights(w));
  SAMBAY_TRY(check_ptrs({u, xdbl, M, ssm_state, conv_state}));
  if (M == u) return SAMBAY_ERR_INVALID_ARG;
  SAMBAY_TRY(check_ws(ws, ws_bytes, sambay_scan_prefill_workspace(d)));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int zi = zero_init_state ? 1 : 0;
  float* xs = const_cast<float*>(xdbl);      // read only in this phase
  if (d->io == SAMBAY_BF16)
    return scan_prefill_impl<bf16>(dev, sms, w, d, u, M, ssm_state, conv_state, zi, w8, st, PROJ_FINISH, xs);
  return scan_prefill_impl<float>(dev, sms, w, d, u, M, ssm_state, conv_state, zi, w8, st, PROJ_FINISH, xs);
}

sambay_status sambay_scan_step(const sambay_scan_weights* w, const sambay_dims* d, const void* u_t,
                               void* m_t, float* ssm_state, void* conv_state, void* ws,
                               size_t ws_bytes, sambay_stream_t stream) {
  if (!d) return SAMBAY_ERR_INVALID_ARG;
  sambay_dims e = *d;
  e.seqlen = 1;
  SAMBAY_TRY(check_dims(&e, false, true));
  SAMBAY_TRY(check_weights(w));
  SAMBAY_TRY(check_ptrs({u_t, m_t, ssm_state, conv_state}));
  if (m_t == u_t) return SAMBAY_ERR_INVALID_ARG;
  SAMBAY_TRY(check_ws(ws, ws_bytes, sambay_scan_step_workspace(&e)));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  if (e.io == SAMBAY_BF16)
    return scan_step_impl<bf16>(dev, sms, w, &e, u_t, m_t, ssm_state, conv_state, w8, st);
  return scan_step_impl<float>(dev, sms, w, &e, u_t, m_t, ssm_state, conv_state, w8, st);
}

sambay_status gmu_forward(const sambay_dims* d, int64_t rows, const void* X, const void* M,
                          const void* W1, const void* W2, const void* residual, void* Y, void* ws,
                          size_t ws_bytes, sambay_stream_t stream) {
  SAMBAY_TRY(gmu_common_checks(d, rows, X, M, W1, W2, residual, Y));
  const GmuWs L = gmu_ws_layout(d, rows, false);
  SAMBAY_TRY(check_ws(ws, ws_bytes, L.total));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  if (d->io == SAMBAY_F32) return gmu_f32(d, rows, X, M, W1, W2, residual, Y, w8, L, st);
  const int Dm = d->d_model, Di = d->d_inner, T = static_cast<int>(rows);
  bf16* H = reinterpret_cast<bf16*>(w8 + L.h);
  float* tail = L.tail_bytes ? reinterpret_cast<float*>(w8 + L.tail) : nullptr;
  // G = X W1^T, epilogue H = M ⊙ SiLU(G)
  SAMBAY_TRY((run_tc<256, false, false, sambay::tc::EPI_GATE, false, 4, true>(
      "gmu_gate_gemm", dev, sms, Operand{X, rows, Dm}, Operand{W1, Di, Dm}, tc_args(T, Di, Dm, H, Di, M), 1, st, false,
      true, tail, L.tail_bytes)));
  // Y = H W2 (+ residual); W2 [Di, Dm] is the MN-major B operand
  SAMBAY_TRY((run_tc<256, false, true, sambay::tc::EPI_RESID, false, 4, true>(
      "gmu_out_gemm", dev, sms, Operand{H, rows, Di}, Operand{W2, Di, Dm}, tc_args(T, Dm, Di, Y, Dm, residual), 1,
      st, true, true, tail, L.tail_bytes)));
  return SAMBAY_OK;
}

sambay_status gmu_forward_partial(const sambay_dims* d, int64_t rows, const void* X, const void* M,
                                  const void* W1, const void* W2, float* Y_part, void* ws, size_t ws_bytes,
                                  sambay_stream_t stream) {
  SAMBAY_TRY(gmu_common_checks(d, rows, X, M, W1, W2, nullptr, Y_part));
  if (Y_part == X) return SAMBAY_ERR_INVALID_ARG;
  const GmuWs L = gmu_ws_layout(d, rows, false);
  SAMBAY_TRY(check_ws(ws, ws_bytes, L.total));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  if (d->io == SAMBAY_F32) return gmu_f32(d, rows, X, M, W1, W2, nullptr, Y_part, w8, L, st);
  const int Dm = d->d_model, Di = d->d_inner, T = static_cast<int>(rows);
  bf16* H = reinterpret_cast<bf16*>(w8 + L.h);
  float* tail = L.tail_bytes ? reinterpret_cast<float*>(w8 + L.tail) : nullptr;
  SAMBAY_TRY((run_tc<256, false, false, sambay::tc::EPI_GATE, false, 4, true>(
      "gmu_gate_gemm", dev, sms, Operand{X, rows, Dm}, Operand{W1, Di, Dm}, tc_args(T, Di, Dm, H, Di, M), 1, st, false,
      true, tail, L.tail_bytes)));
  // Y_part = H W2 in fp32: single-CTA 128 x 256 tiles (the CTA-pair form has
  // only the bf16 epilogues), whole tiles only
  SAMBAY_TRY((run_tc<256, false, true, sambay::tc::EPI_F32_PARTIAL, false, 4>(
      "gmu_out_partial", dev, sms, Operand{H, rows, Di}, Operand{W2, Di, Dm}, tc_args(T, Dm, Di, Y_part, Dm), 1, st,
      true, false)));
  return SAMBAY_OK;
}

sambay_status gmu_finish(const sambay_dims* d, int64_t rows, const float* Y_sum, const void* residual, void* Y,
                         sambay_stream_t stream) {
  SAMBAY_TRY(check_dims(d, true, false));
  if (rows < 1 || rows > (1LL << 30)) return SAMBAY_ERR_INVALID_ARG;
  SAMBAY_TRY(check_ptrs({Y_sum, Y}));
  if (residual && !aligned16(residual)) return SAMBAY_ERR_UNSUPPORTED;
  if (Y == static_cast<const void*>(Y_sum)) return SAMBAY_ERR_INVALID_ARG;
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long n4 = rows * d->d_model / 4;
  ProfScope ps("gmu_finish", st);
  if (d->io == SAMBAY_BF16)
    gmu_finish_kernel<bf16><<<grid_for(n4, 256, sms), 256, 0, st>>>(Y_sum, static_cast<const bf16*>(residual),
                                                                    static_cast<bf16*>(Y), n4);
  else
    gmu_finish_kernel<float><<<grid_for(n4, 256, sms), 256, 0, st>>>(Y_sum, static_cast<const float*>(residual),
                                                                     static_cast<float*>(Y), n4);
  return cudaGetLastError() == cudaSuccess ? SAMBAY_OK : SAMBAY_ERR_CUDA;
}

sambay_status gmu_step(const sambay_dims* d, int64_t rows, const void* X, const void* M,
                       const void* W1, const void* W2, const void* residual, void* Y, void* ws,
                       size_t ws_bytes, sambay_stream_t stream) {
  SAMBAY_TRY(gmu_common_checks(d, rows, X, M, W1, W2, residual, Y));
  if (rows > kStepMaxRows) return SAMBAY_ERR_UNSUPPORTED;
  const GmuWs L = gmu_ws_layout(d, rows, true);
  SAMBAY_TRY(check_ws(ws, ws_bytes, L.total));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  if (d->io == SAMBAY_F32) return gmu_f32(d, rows, X, M, W1, W2, residual, Y, w8, L, st);
  return gmu_step_tc(dev, sms, d, rows, X, M, W1, W2, residual, Y, w8 + L.h, StepChain{}, st);
}

size_t sambay_decode_step_workspace(const sambay_dims* d, int32_t n_layers) {
  if (!d || n_layers < 0) return 0;
  sambay_dims e = *d;
  e.seqlen = 1;
  if (check_dims(&e, true, true) != SAMBAY_OK || e.batch > kStepMaxRows) return 0;
  const size_t scan = scan_ws_layout(&e, e.batch, true).total;
  const size_t gmu = n_layers > 0 ? gmu_ws_layout(&e, e.batch, true).total : 0;
  return round256(scan) + gmu;
}

sambay_status sambay_decode_step(const sambay_scan_weights* w, const sambay_dims* d, const void* u_t,
                                 void* m_t, float* ssm_state, void* conv_state, int32_t n_layers,
                                 const sambay_gmu_weights* layers, void* X, void* ws, size_t ws_bytes,
                                 sambay_stream_t stream) {
  if (!d) return SAMBAY_ERR_INVALID_ARG;
  sambay_dims e = *d;
  e.seqlen = 1;
  SAMBAY_TRY(check_dims(&e, true, true));
  SAMBAY_TRY(check_weights(w));
  SAMBAY_TRY(check_ptrs({u_t, m_t, ssm_state, conv_state}));
  if (m_t == u_t) return SAMBAY_ERR_INVALID_ARG;
  if (n_layers < 0 || n_layers > 1024) return SAMBAY_ERR_INVALID_ARG;
  if (e.batch > kStepMaxRows) return SAMBAY_ERR_UNSUPPORTED;
  if (n_layers > 0) {
    if (!layers) return SAMBAY_ERR_INVALID_ARG;
    SAMBAY_TRY(check_ptrs({X}));
    for (int l = 0; l < n_layers; ++l) SAMBAY_TRY(check_ptrs({layers[l].W1, layers[l].W2}));
    if (X == m_t || X == u_t) return SAMBAY_ERR_INVALID_ARG;
  }
  SAMBAY_TRY(check_ws(ws, ws_bytes, sambay_decode_step_workspace(&e, n_layers)));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  if (e.io == SAMBAY_BF16) {
    SAMBAY_TRY(scan_step_impl<bf16>(dev, sms, w, &e, u_t, m_t, ssm_state, conv_state, w8, st));
  } else {
    SAMBAY_TRY(scan_step_impl<float>(dev, sms, w, &e, u_t, m_t, ssm_state, conv_state, w8, st));
  }
  const GmuWs L = gmu_ws_layout(&e, e.batch, true);
  uint8_t* gw8 = w8 + round256(scan_ws_layout(&e, e.batch, true).total);   // H, after the scan scratch
  for (int l = 0; l < n_layers; ++l) {
    if (e.io == SAMBAY_F32) {
      SAMBAY_TRY(gmu_f32(&e, e.batch, X, m_t, layers[l].W1, layers[l].W2, X, X, gw8, L, st));
      continue;
    }
    // layer 0's gate reads the caller's X, untouched by the scan step, so its
    // whole main loop may overlap the scan; later gates read the X the layer
    // before wrote and load only their W1 tiles early
    StepChain ch;
    ch.chained = true;
    ch.x_independent = (l == 0);
    SAMBAY_TRY(gmu_step_tc(dev, sms, &e, e.batch, X, m_t, layers[l].W1, layers[l].W2, X, X, gw8 + L.h, ch, st));
  }
  return SAMBAY_OK;
}

sambay_status sambay_gmu_step_stall_test(const sambay_dims* d, int64_t rows, const void* X, const void* M,
                                         const void* W1, const void* W2, const void* residual, void* Y,
                                         void* ws, size_t ws_bytes, uint64_t wait_limit_cycles,
                                         sambay_stream_t stream) {
  SAMBAY_TRY(gmu_common_checks(d, rows, X, M, W1, W2, residual, Y));
  if (d->io != SAMBAY_BF16) return SAMBAY_ERR_UNSUPPORTED;
  if (rows > kStepMaxRows) return SAMBAY_ERR_UNSUPPORTED;
  if (wait_limit_cycles < 1 || wait_limit_cycles > (1ull << 32)) return SAMBAY_ERR_INVALID_ARG;
  const GmuWs L = gmu_ws_layout(d, rows, true);
  SAMBAY_TRY(check_ws(ws, ws_bytes, L.total));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  StepChain ch;
  ch.wait_limit = wait_limit_cycles;
  ch.stall_test = 1;
  return gmu_step_tc(dev, sms, d, rows, X, M, W1, W2, residual, Y, static_cast<uint8_t*>(ws) + L.h, ch,
                     reinterpret_cast<cudaStream_t>(stream));
}

size_t sambay_in_proj_workspace(const sambay_dims* d, int64_t rows) {
  if (check_dims(d, true, false) != SAMBAY_OK || rows < 1) return 0;
  return proj_ws_layout(d, rows, false).total;
}

sambay_status sambay_in_proj(const sambay_dims* d, int64_t rows, const void* X, const void* W_in, void* u,
                             void* ws, size_t ws_bytes, sambay_stream_t stream) {
  SAMBAY_TRY(check_dims(d, true, false));
  if (rows < 1 || rows > (1LL << 30)) return SAMBAY_ERR_INVALID_ARG;
  SAMBAY_TRY(check_ptrs({X, W_in, u}));
  if (u == X) return SAMBAY_ERR_INVALID_ARG;
  const ProjWs L = proj_ws_layout(d, rows, false);
  SAMBAY_TRY(check_ws(ws, ws_bytes, L.total));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int Dm = d->d_model, Di = d->d_inner;
  if (d->io == SAMBAY_F32)
    return run_simt<sambay::simt::F32_STORE>("in_proj_f32",
        simt_args(static_cast<const float*>(X), Dm, 1, static_cast<const float*>(W_in), 1, Dm,
                  static_cast<int>(rows), Di, Dm, static_cast<float*>(u), Di), st);
  float* tail = L.tail_bytes ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.tail) : nullptr;
  return project_tc<sambay::tc::EPI_RESID>(dev, sms, rows, Di, Dm, X, W_in, nullptr, u, tail, L.tail_bytes,
                                           "in_proj", st);
}

size_t sambay_mlp_memory_workspace(const sambay_dims* d, int64_t rows) {
  if (check_dims(d, true, false) != SAMBAY_OK || rows < 1) return 0;
  return proj_ws_layout(d, rows, true).total;
}

sambay_status sambay_mlp_memory(const sambay_dims* d, int64_t rows, const void* X, const void* W_g,
                                const void* W_u, void* M, void* ws, size_t ws_bytes, sambay_stream_t stream) {
  SAMBAY_TRY(check_dims(d, true, false));
  if (rows < 1 || rows > (1LL << 30)) return SAMBAY_ERR_INVALID_ARG;
  SAMBAY_TRY(check_ptrs({X, W_g, W_u, M}));
  if (M == X) return SAMBAY_ERR_INVALID_ARG;
  const ProjWs L = proj_ws_layout(d, rows, true);
  SAMBAY_TRY(check_ws(ws, ws_bytes, L.total));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int Dm = d->d_model, Df = d->d_inner, T = static_cast<int>(rows);
  if (d->io == SAMBAY_F32) {
    float* U = reinterpret_cast<float*>(w8 + L.buf);
    SAMBAY_TRY(run_simt<sambay::simt::F32_STORE>("mlp_up_f32",
        simt_args(static_cast<const float*>(X), Dm, 1, static_cast<const float*>(W_u), 1, Dm, T, Df, Dm, U, Df), st));
    return run_simt<sambay::simt::GATE>("mlp_gate_f32",
        simt_args(static_cast<const float*>(X), Dm, 1, static_cast<const float*>(W_g), 1, Dm, T, Df, Dm,
                  static_cast<float*>(M), Df, U), st);
  }
  bf16* U = reinterpret_cast<bf16*>(w8 + L.buf);
  float* tail = L.tail_bytes ? reinterpret_cast<float*>(w8 + L.tail) : nullptr;
  // U = X W_u^T, then M = U ⊙ SiLU(X W_g^T): the gate GEMM with U as its aux
  SAMBAY_TRY(project_tc<sambay::tc::EPI_RESID>(dev, sms, rows, Df, Dm, X, W_u, nullptr, U, tail, L.tail_bytes,
                                               "mlp_up", st));
  return project_tc<sambay::tc::EPI_GATE>(dev, sms, rows, Df, Dm, X, W_g, U, M, tail, L.tail_bytes, "mlp_gate",
                                          st);
}

}  // extern "C"

namespace {

// Split-KV plan of the cross-attention decode: enough (sequence, KV head,
// split) CTAs to cover a 148-SM B200 about three times, splits of whole
// 128-token blocks (a function of the sizes only).
struct AttnPlan {
  int splits = 1, chunk = 0;
  size_t o_part = 0, ml_part = 0, total = 0;
};

sambay_status attn_check(const sambay_attn_dims* a) {
  if (!a) return SAMBAY_ERR_INVALID_ARG;
  if (a->batch < 1 || a->kv_len < 1 || a->q_heads < 1 || a->kv_heads < 1 || a->head_dim < 1)
    return SAMBAY_ERR_INVALID_ARG;
  if (a->head_dim != 64 && a->head_dim != 128) return SAMBAY_ERR_UNSUPPORTED;
  if (a->q_heads % a->kv_heads != 0 || a->q_heads / a->kv_heads > 16) return SAMBAY_ERR_UNSUPPORTED;
  return SAMBAY_OK;
}

AttnPlan attn_plan(const sambay_attn_dims* a) {
  AttnPlan pl;
  constexpr int kBlock = sambay::attn::kTile * sambay::attn::kWarps;
  const long long pairs = static_cast<long long>(a->batch) * a->kv_heads;
  const long long blocks = (a->kv_len + kBlock - 1) / kBlock;
  long long splits = std::max(1LL, (3LL * kSplitTarget + pairs - 1) / pairs);
  splits = std::min(splits, blocks);
  pl.chunk = static_cast<int>((blocks + splits - 1) / splits) * kBlock;
  pl.splits = static_cast<int>((a->kv_len + pl.chunk - 1) / pl.chunk);
  if (pl.splits > 1) {
    const size_t qh = static_cast<size_t>(a->batch) * a->q_heads * pl.splits;
    pl.o_part = 0;
    pl.ml_part = round256(qh * a->head_dim * 4);
    pl.total = pl.ml_part + round256(qh * 2 * 4);
  }
  return pl;
}

template <int DH>
sambay_status attn_launch(int dev, int sms, sambay::attn::AttnParams& p, cudaStream_t st) {
  using namespace sambay::attn;
  auto kern = cross_attn_decode_kernel<DH>;
  static bool attr_set[kMaxDevices] = {};
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnLayout<DH>::kBytes) !=
        cudaSuccess)
      return SAMBAY_ERR_CUDA;
    attr_set[dev] = true;
  }
  {
    ProfScope ps("cross_attn_decode", st);
    if (launch_k(kern, dim3(p.splits, p.Hkv, p.B), dim3(kThreads), AttnLayout<DH>::kBytes, st, false, 1, p) !=
        cudaSuccess)
      return SAMBAY_ERR_CUDA;
  }
  if (p.splits > 1) {
    const long long n = static_cast<long long>(p.B) * p.Hq * DH;
    ProfScope ps("cross_attn_combine", st);
    if (launch_k(cross_attn_combine_kernel<DH>, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, st,
                 true, 1, p) != cudaSuccess)
      return SAMBAY_ERR_CUDA;
  }
  return SAMBAY_OK;
}

}  // namespace

extern "C" {

size_t sambay_cross_attn_decode_workspace(const sambay_attn_dims* a) {
  if (attn_check(a) != SAMBAY_OK) return 0;
  return attn_plan(a).total;
}

sambay_status sambay_cross_attn_decode(const sambay_attn_dims* a, const void* q, const void* K, const void* V,
                                       void* out, float scale, void* ws, size_t ws_bytes,
                                       sambay_stream_t stream) {
  SAMBAY_TRY(attn_check(a));
  SAMBAY_TRY(check_ptrs({q, K, V, out}));
  if (out == q || out == K || out == V) return SAMBAY_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || scale > 1e4f) return SAMBAY_ERR_INVALID_ARG;   // also rejects NaN
  const AttnPlan pl = attn_plan(a);
  SAMBAY_TRY(check_ws(ws, ws_bytes, pl.total));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  sambay::attn::AttnParams p{};
  p.q = static_cast<const bf16*>(q);
  p.K = static_cast<const bf16*>(K);
  p.V = static_cast<const bf16*>(V);
  p.out = static_cast<bf16*>(out);
  p.o_part = pl.splits > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.o_part) : nullptr;
  p.ml_part = pl.splits > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.ml_part) : nullptr;
  p.B = a->batch;
  p.N = a->kv_len;
  p.Hq = a->q_heads;
  p.Hkv = a->kv_heads;
  p.G = a->q_heads / a->kv_heads;
  p.splits = pl.splits;
  p.chunk = pl.chunk;
  const float sc = scale > 0.0f ? scale : 1.0f / sqrtf(static_cast<float>(a->head_dim));
  p.scale_log2 = sc * 1.4426950408889634f;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return a->head_dim == 64 ? attn_launch<64>(dev, sms, p, st) : attn_launch<128>(dev, sms, p, st);
}

// ------------------------------------------------------------ SambaY-2 (Mamba-2 SSD)

namespace {

sambay_status ssd_check(const sambay_ssd_dims* d) {
  if (!d) return SAMBAY_ERR_INVALID_ARG;
  if (d->batch <= 0 || d->seqlen <= 0 || d->nheads <= 0 || d->headdim <= 0 || d->d_state <= 0 ||
      d->d_conv <= 0)
    return SAMBAY_ERR_INVALID_ARG;
  if (d->io != SAMBAY_BF16 && d->io != SAMBAY_F32) return SAMBAY_ERR_INVALID_ARG;
  if (d->io != SAMBAY_BF16 || d->headdim != sambay::ssd::kP || (d->d_state != 64 && d->d_state != 128) ||
      d->d_conv != 4)
    return SAMBAY_ERR_UNSUPPORTED;
  const long long C = static_cast<long long>(d->nheads) * d->headdim + 2LL * d->d_state;
  if (C % 32 != 0 || C > (1LL << 24) || static_cast<long long>(d->batch) * d->seqlen > (1LL << 26))
    return SAMBAY_ERR_UNSUPPORTED;
  return SAMBAY_OK;
}

}  // namespace

size_t sambay_ssd_prefill_workspace(const sambay_ssd_dims* d) {
  if (ssd_check(d) != SAMBAY_OK) return 0;
  const size_t C = static_cast<size_t>(d->nheads) * d->headdim + 2 * static_cast<size_t>(d->d_state);
  return round256(static_cast<size_t>(d->batch) * d->seqlen * C * 4);
}

sambay_status sambay_ssd_prefill(const sambay_ssd_weights* w, const sambay_ssd_dims* d, const void* xbc,
                                 const void* dt_raw, void* M, float* ssm_state, void* conv_state, int32_t zero_init,
                                 void* ws, size_t ws_bytes, sambay_stream_t stream) {
  SAMBAY_TRY(ssd_check(d));
  if (!w) return SAMBAY_ERR_INVALID_ARG;
  SAMBAY_TRY(check_ptrs({w->conv_w, w->conv_b, w->dt_bias, w->A, w->D}));
  SAMBAY_TRY(check_ptrs({xbc, dt_raw, M, ssm_state, conv_state}));
  if (M == xbc) return SAMBAY_ERR_INVALID_ARG;
  SAMBAY_TRY(check_ws(ws, ws_bytes, sambay_ssd_prefill_workspace(d)));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int C = d->nheads * d->headdim + 2 * d->d_state;
  bf16* xc = static_cast<bf16*>(ws);
  {
    sambay::scan::ConvParams<bf16> p{static_cast<const bf16*>(xbc), static_cast<const bf16*>(conv_state),
                                     static_cast<const bf16*>(w->conv_w), static_cast<const bf16*>(w->conv_b), xc,
                                     d->batch, d->seqlen, C, zero_init ? 1 : 0};
    using sambay::scan::kConvTT;
    auto c64 = sambay::scan::conv_silu_kernel<bf16, 64>;
    auto c32 = sambay::scan::conv_silu_kernel<bf16, 32>;
    SAMBAY_MAX_CARVEOUT(c64, dev);
    SAMBAY_MAX_CARVEOUT(c32, dev);
    ProfScope ps("ssd_conv_silu", st);
    if (C % 64 == 0) {
      dim3 grid(C / 64, (d->seqlen + kConvTT - 1) / kConvTT, d->batch);
      c64<<<grid, 64 / 4 * (kConvTT / 4), 0, st>>>(p);
    } else {
      dim3 grid(C / 32, (d->seqlen + kConvTT - 1) / kConvTT, d->batch);
      c32<<<grid, 32 / 4 * (kConvTT / 4), 0, st>>>(p);
    }
    if (cudaGetLastError() != cudaSuccess) return SAMBAY_ERR_CUDA;
  }
  {
    auto kern = d->d_state == 128 ? sambay::ssd::ssd_chunk_scan_kernel<128> : sambay::ssd::ssd_chunk_scan_kernel<64>;
    static bool attr_set[kMaxDevices] = {};
    const sambay::ssd::SsdLayout ly(d->d_state);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(sambay::ssd::ssd_chunk_scan_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               sambay::ssd::SsdLayout(128).bytes) != cudaSuccess ||
          cudaFuncSetAttribute(sambay::ssd::ssd_chunk_scan_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               sambay::ssd::SsdLayout(64).bytes) != cudaSuccess)
        return SAMBAY_ERR_CUDA;
      attr_set[dev] = true;
    }
    sambay::ssd::SsdParams p{};
    p.xc = xc;
    p.dt_raw = static_cast<const bf16*>(dt_raw);
    p.dt_bias = w->dt_bias;
    p.A = w->A;
    p.D = w->D;
    p.h = ssm_state;
    p.M = static_cast<bf16*>(M);
    p.Bt = d->batch;
    p.L = d->seqlen;
    p.H = d->nheads;
    p.N = d->d_state;
    p.zero_init = zero_init ? 1 : 0;
    ProfScope ps("ssd_chunk_scan", st);
    if (launch_k(kern, dim3(d->nheads, d->batch), dim3(sambay::ssd::kThreads), ly.bytes, st, true, 1, p) !=
        cudaSuccess)
      return SAMBAY_ERR_CUDA;
  }
  {
    // after the conv has read the old window
    const long long n = static_cast<long long>(d->batch) * C;
    ProfScope ps("ssd_conv_state", st);
    if (launch_k(sambay::ssd::conv_state_update_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0,
                 st, true, 1, static_cast<const bf16*>(xbc), static_cast<bf16*>(conv_state), d->batch, d->seqlen, C,
                 zero_init ? 1 : 0) != cudaSuccess)
      return SAMBAY_ERR_CUDA;
  }
  return SAMBAY_OK;
}

size_t sambay_ssd_step_workspace(const sambay_ssd_dims* d) {
  if (ssd_check(d) != SAMBAY_OK) return 0;
  const size_t C = static_cast<size_t>(d->nheads) * d->headdim + 2 * static_cast<size_t>(d->d_state);
  return round256(static_cast<size_t>(d->batch) * C * 4);
}

sambay_status sambay_ssd_step(const sambay_ssd_weights* w, const sambay_ssd_dims* d, const void* xbc_t,
                              const void* dt_raw_t, void* m_t, float* ssm_state, void* conv_state, void* ws,
                              size_t ws_bytes, sambay_stream_t stream) {
  SAMBAY_TRY(ssd_check(d));
  if (!w) return SAMBAY_ERR_INVALID_ARG;
  SAMBAY_TRY(check_ptrs({w->conv_w, w->conv_b, w->dt_bias, w->A, w->D}));
  SAMBAY_TRY(check_ptrs({xbc_t, dt_raw_t, m_t, ssm_state, conv_state}));
  if (m_t == xbc_t) return SAMBAY_ERR_INVALID_ARG;
  SAMBAY_TRY(check_ws(ws, ws_bytes, sambay_ssd_step_workspace(d)));
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int C = d->nheads * d->headdim + 2 * d->d_state;
  float* xc = static_cast<float*>(ws);
  {
    const long long n = static_cast<long long>(d->batch) * (C / 8);
    ProfScope ps("ssd_step_conv", st);
    sambay::ssd::ssd_step_conv_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
        static_cast<const bf16*>(xbc_t), static_cast<bf16*>(conv_state), static_cast<const bf16*>(w->conv_w),
        static_cast<const bf16*>(w->conv_b), xc, d->batch, C);
    if (cudaGetLastError() != cudaSuccess) return SAMBAY_ERR_CUDA;
  }
  auto kern = d->d_state == 128 ? sambay::ssd::ssd_step_kernel<128> : sambay::ssd::ssd_step_kernel<64>;
  ProfScope ps("ssd_step", st);
  return launch_k(kern, dim3(d->nheads, d->batch), dim3(256), 0, st, true, 1, static_cast<const float*>(xc),
                  static_cast<const bf16*>(dt_raw_t), w->dt_bias, w->A, w->D, ssm_state, static_cast<bf16*>(m_t),
                  d->nheads) == cudaSuccess
             ? SAMBAY_OK
             : SAMBAY_ERR_CUDA;
}

sambay_status sambay_scan_step_noalloc(const sambay_scan_weights* w, const sambay_dims* d,
                                       const void* u_t, void* m_t, float* ssm_state,
                                       void* conv_state, sambay_stream_t stream) {
  if (!d) return SAMBAY_ERR_INVALID_ARG;
  sambay_dims e = *d;
  e.seqlen = 1;
  SAMBAY_TRY(check_dims(&e, false, true));
  SAMBAY_TRY(check_weights(w));
  SAMBAY_TRY(check_ptrs({u_t, m_t, ssm_state, conv_state}));
  if (m_t == u_t) return SAMBAY_ERR_INVALID_ARG;
  if (sambay_scan_step_workspace(&e) > SAMBAY_NOALLOC_SCRATCH_BYTES) return SAMBAY_ERR_UNSUPPORTED;
  int dev, sms;
  SAMBAY_TRY(current_device(&dev, &sms));
  void* scratch = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (scratch == nullptr) {
    // once per device, with that device current
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || scratch == nullptr)
      return SAMBAY_ERR_CUDA;
    g_noalloc_ptr[dev].store(scratch, std::memory_order_release);
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(scratch);
  if (e.io == SAMBAY_BF16)
    return scan_step_impl<bf16>(dev, sms, w, &e, u_t, m_t, ssm_state, conv_state, w8, st);
  return scan_step_impl<float>(dev, sms, w, &e, u_t, m_t, ssm_state, conv_state, w8, st);
}

sambay_status sambay_profile_begin(void* const* events, int32_t capacity) {
  if (!events || capacity < 2) return SAMBAY_ERR_INVALID_ARG;
  ProfState& ps = g_prof_storage;
  ps.ev = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events));
  ps.cap = capacity & ~1;
  ps.n = 0;
  ps.names.clear();
  g_prof = &ps;
  return SAMBAY_OK;
}

int32_t sambay_profile_end(const char** names, int32_t max_names) {
  if (!g_prof) return 0;
  const int launches = g_prof->n / 2;
  for (int i = 0; i < launches && names && i < max_names; ++i) names[i] = g_prof->names[i];
  g_prof = nullptr;
  return launches;
}

sambay_status sambay_device_status(sambay_stream_t stream, int32_t* out_code) {
  if (!out_code) return SAMBAY_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SAMBAY_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, sambay::g_status, sizeof(int)) != cudaSuccess) return SAMBAY_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(sambay::g_status, &zero, sizeof(int)) != cudaSuccess) return SAMBAY_ERR_CUDA;
  *out_code = v;
  return SAMBAY_OK;
}

}  // extern "C"
