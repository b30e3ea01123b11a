// Persistent tcgen05 (5th-gen tensor core) GEMM for sm_100a, bf16 in, fp32
// accumulate in TMEM, operands staged in shared memory by TMA, with fused
// epilogues.  One CTA per SM; warp roles:
//   warp 0        TMA producer (one lane): A and B tiles into a smem ring
//   warp 1        MMA issuer (one lane) + TMEM owner (whole warp allocates)
//   warps 2..     EW epilogue warps (4 or 8): tcgen05.ld TMEM -> registers ->
//                 fused op -> HBM.  Warp w reads TMEM lanes 32 (w % 4) ..; with
//                 8, the two warps of a lane quarter take alternate column blocks
// The accumulator is double-buffered in TMEM so the epilogue of one tile
// overlaps the main loop of the next.  No TMA multicast is used: every CTA
// loads its own tiles.
//
// PAIR mode (cta_group::2): a cluster of two CTAs on two SMs computes one
// 256 x BN tile.  Each CTA loads its own 128 rows of A and its half of B (BN/2
// columns), so a pair moves half the B bytes per flop of two 128 x BN tiles;
// the leader CTA (rank 0) issues the M = 256 MMAs, which read both CTAs'
// shared memory and write each CTA's 128 accumulator rows into that CTA's
// TMEM.  Both CTAs' TMA loads complete on the leader's stage barriers, the
// leader's commits arrive on both CTAs' barriers, and both CTAs' epilogue
// warps hand the accumulator back through the leader's barrier.
//
// D[m, n] = sum_k A[m, k] * B[k, n]
//   A: K-major ([M, K], k contiguous) or MN-major ([K, M], m contiguous)
//   B: K-major ([N, K], k contiguous) or MN-major ([K, N], n contiguous)
// Tile 128 x BN x 64, SWIZZLE_128B smem layout (what TMA writes with a 128-byte
// inner box), UMMA smem descriptors per the sm_100 matrix-descriptor format.
//
// Every mbarrier wait is bounded (clock64), and so is the wait for the K-split
// tail's arrival flags (other CTAs' partial tiles); on expiry the kernel
// records SAMBAY_ERR_TIMEOUT in the device status word, raises a CTA-wide abort
// flag, drains its in-flight TMA loads and MMAs (again bounded), frees TMEM and
// returns.
#pragma once

#include <cuda.h>
#include "common.cuh"

namespace sambay {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;                       // one 128-byte swizzle atom of bf16
__host__ __device__ constexpr int gemm_threads(int EW) { return 64 + 32 * EW; }
constexpr unsigned long long kWaitCycles = 1ull << 34;  // ~8 s at 2 GHz
constexpr unsigned long long kDrainCycles = 1ull << 28;

// ------------------------------------------------------------------ PTX glue

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait.  Returns false if the CTA is aborting (flag already raised by
// another role) or this wait ran out (then it raises the flag itself).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit = kWaitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (static_cast<unsigned long long>(clock64() - t0) > limit) {
      *abort_flag = 1;
      record_status(kStatusTimeout);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// ---- CTA-pair (cta_group::2) forms.  A shared::cta address with the peer
// bit cleared names the same variable in the pair's rank-0 CTA.
constexpr uint32_t kPeerBitMask = 0xFEFFFFFFu;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The shared::cluster address of this CTA's shared variable at `addr` in the
// cluster's CTA `rank`, and a 16-byte load through it (distributed shared memory).
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_dsmem_f32x4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}
// TMA load into this CTA's shared memory whose bytes complete on the
// leader CTA's barrier
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar) & kPeerBitMask), "r"(c0), "r"(c1)
      : "memory");
}
// arrive on the leader CTA's copy of this barrier
__device__ __forceinline__ void mbar_arrive_leader(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(smem_u32(bar) & kPeerBitMask) : "memory");
}

// shared -> global tile store (bulk group); out-of-range rows/columns are clipped
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// generic-proxy shared-memory writes become visible to the async proxy (TMA)
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// the MMAs issued so far by this thread, once complete, arrive on the barrier
// at this offset in both CTAs of the pair
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}\n" ::"r"(
          smem_u32(bar))
      : "memory");
}

// the same, for MMAs issued with cta_group::2, arriving on this CTA only
__device__ __forceinline__ void tc_commit2(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread i of the warp receives row
// (lane base + i), columns [col, col + 32).  The load is asynchronous until
// tmem_ld_wait, which names the destination registers so that no use of
// them can be scheduled before it.
__device__ __forceinline__ void tmem_ld_issue(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                 "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
                 "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
                 "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
                 "+r"(r[31])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld_issue(taddr, r);
  tmem_ld_wait(r);
}

// AND of a predicate over the NT epilogue threads (named barrier 1).
template <int NT>
__device__ __forceinline__ bool epi_agree(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(ok ? 1u : 0u), "n"(NT)
      : "memory");
  return r != 0;
}

// barrier over the NT epilogue threads (named barrier 1)
template <int NT>
__device__ __forceinline__ void named_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

// Shared-memory matrix descriptor, SWIZZLE_128B, sm_100 format (version 1).
//   K-major : 8-row x 128-byte atoms; SBO = 1024 B between 8-row groups.
//   MN-major: 64-element x 8-row atoms; LBO = stride between 64-element MN
//             groups, SBO = 1024 B between 8-row K groups.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= 1ull << 46;  // descriptor version (sm_100)
  d |= 2ull << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                       // D format: f32
         | (1u << 7)                     // A format: bf16
         | (1u << 10)                    // B format: bf16
         | ((a_mn ? 1u : 0u) << 15)      // A major
         | ((b_mn ? 1u : 0u) << 16)      // B major
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------- epilogues

enum EpiKind : int {
  EPI_F32_PARTIAL = 0,  // out(f32)[split][...] = acc     (split-K partials, summed by the caller)
  EPI_GATE = 1,      // out(bf16) = SiLU(acc) * aux      (GMU gate: H = M ⊙ SiLU(X W1^T))
  EPI_RESID = 2,     // out(bf16) = acc (+ aux if given)  (GMU output + residual)
  EPI_SOFTPLUS = 3,  // out(f32) = softplus(acc + vec[n]) (dt_proj)
};

struct GemmArgs {
  int M, N, K;
  int m_tiles, n_tiles, splits, kb_per_split, k_blocks, tiles;
  void* out;          // output base
  const void* aux;    // EPI_GATE: memory readout M; EPI_RESID: residual or NULL
  const float* vec;   // EPI_SOFTPLUS: per-column bias
  long long ldo;      // leading dimension (elements) of out and aux
  long long split_stride;  // elements between consecutive splits' partials
  float* partials;    // split-K partial tiles [splits][split_stride] (f32)
  int* counters;      // split-K arrival counters per (m, n) tile, zero on entry
  int b_k_wrap;       // > 0: B's k coordinate wraps at this multiple of 64, so an A
                      // of [hi | lo] halves meets the same B twice (split-bf16 operand)
  int tma_epi;        // row-major gate / residual / softplus epilogue through TMA
                      // (aux tile in, output tile out); set by the host when the
                      // output's columns come in whole 64 (bf16) / 32 (f32) blocks
  int csplit;         // cluster split-K: the `splits` K ranges of a tile are one
                      // cluster of CTAs (one unit each), which write their partial
                      // tiles, meet at a cluster barrier and then each reduce and
                      // finish a slice of the tile's rows (no counters, no tail
                      // where one CTA sums every partial)
  int full_tiles;     // tail_nsplit > 1: work units [0, full_tiles) are whole tiles,
  int tail_nsplit;    // and every later tile is cut along N into tail_nsplit units
                      // of BN / tail_nsplit columns (wave quantisation: the last,
                      // partial wave of tiles spreads over more SMs; no K split)
  int tail_ksplit;    // > 1 instead: every tile after full_tiles is cut along K into
  int tail_kbps;      // tail_ksplit units of tail_kbps k-blocks, each writing its fp32
  float* tail_part;   // partial tile [tail tile][split][tile rows][BN] to tail_part.
                      // The tail units run first (at most one per CTA pair); before
                      // its first whole tile's epilogue every CTA sums a share of
                      // the tail outputs
  unsigned long long* tail_flags;  // per tail unit and pair rank: the epoch once stored
  unsigned long long tail_epoch;   // this launch's 48-bit epoch (never 0)
  int a_early;        // launched with programmatic dependent launch: the A operand does
                      // not depend on the kernel before this one, so the producer loads
                      // the first pipeline stages' A tiles before griddepcontrol.wait
  int b_early;        // ... and neither does B: the whole main loop may run before the
                      // wait; only the epilogue (aux in, output out) waits
  unsigned long long wait_limit;  // bounded-wait limit in clock64 cycles (0: kWaitCycles)
  int stall_test;     // fault-detector test: the epilogue first waits on a barrier that
                      // nothing arrives at, so that wait runs out after wait_limit
};

// The final op on one element.  `o` is the output's linear index, `a` the aux
// value at o (M for the gate, the residual or 0 for EPI_RESID).
template <int KIND>
__device__ __forceinline__ void epi_store_one(const GemmArgs& g, long long o, int n, float v, float a) {
  if (KIND == EPI_F32_PARTIAL) {
    reinterpret_cast<float*>(g.out)[o] = v;
  } else if (KIND == EPI_GATE) {
    reinterpret_cast<bf16*>(g.out)[o] = __float2bfloat16_rn(silu(v) * a);
  } else if (KIND == EPI_RESID) {
    reinterpret_cast<bf16*>(g.out)[o] = __float2bfloat16_rn(v + a);
  } else {
    reinterpret_cast<float*>(g.out)[o] = softplus(v + g.vec[n]);
  }
}

// Per-warp staging buffer for the epilogue: 32 rows x (128 + 16 pad) bytes.
// The row pitch keeps the per-thread 16-byte row accesses conflict-free.
constexpr int kEpiPitchF32 = 144;   // 32 floats + pad
constexpr int kEpiPitchB16 = 80;    // 32 bf16 + pad
constexpr int kEpiWarpBytes = 32 * kEpiPitchF32;

// One warp's 32 x 32 output block: thread `lane` holds the 32 accumulator
// values of row m = row0 + lane, columns [n0, n0 + 32).  All 32 lanes call
// this together.  A full block of a row-major output is staged through shared
// memory so every global load / store instruction of the warp covers whole
// row segments (8 rows x 64 B of bf16, 4 rows x 128 B of f32) instead of 32
// scattered 16-byte pieces; the aux tile (M, residual) comes in the same way.
// TRANS (swap-AB decode, out[n * ldo + m]) and ragged column edges go element
// by element, which is already coalesced across the warp for TRANS.
template <int KIND, bool TRANS>
__device__ __forceinline__ void epi_chunk(const GemmArgs& g, int row0, int lane, int n0,
                                          const float (&v)[32], uint8_t* stage) {
  const int m = row0 + lane;
  if (!TRANS && n0 + 32 <= g.N && (g.ldo % 8) == 0) {
    if (KIND == EPI_F32_PARTIAL || KIND == EPI_SOFTPLUS) {
      float4* mine = reinterpret_cast<float4*>(stage + lane * kEpiPitchF32);
      const float4* bias = reinterpret_cast<const float4*>(g.vec + n0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 r = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        if (KIND == EPI_SOFTPLUS) {
          const float4 b = bias[j];
          r.x = softplus(r.x + b.x);
          r.y = softplus(r.y + b.y);
          r.z = softplus(r.z + b.z);
          r.w = softplus(r.w + b.w);
        }
        mine[j] = r;
      }
      __syncwarp();
      float* out = reinterpret_cast<float*>(g.out);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = i * 4 + (lane >> 3), seg = lane & 7;
        if (row0 + r < g.M)
          *reinterpret_cast<float4*>(out + static_cast<long long>(row0 + r) * g.ldo + n0 + seg * 4) =
              *reinterpret_cast<const float4*>(stage + r * kEpiPitchF32 + seg * 16);
      }
      __syncwarp();
    } else {
      const bool has_aux = KIND == EPI_GATE || g.aux != nullptr;
      const bf16* aux = reinterpret_cast<const bf16*>(g.aux);
      Pack16 a[4];
      if (has_aux) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = i * 8 + (lane >> 2), seg = lane & 3;
          uint4 x = make_uint4(0u, 0u, 0u, 0u);
          if (row0 + r < g.M)
            x = *reinterpret_cast<const uint4*>(aux + static_cast<long long>(row0 + r) * g.ldo + n0 + seg * 8);
          *reinterpret_cast<uint4*>(stage + r * kEpiPitchB16 + seg * 16) = x;
        }
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j) a[j].u = *reinterpret_cast<const uint4*>(stage + lane * kEpiPitchB16 + j * 16);
        __syncwarp();
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        Pack16 r;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = v[8 * j + 2 * e], x1 = v[8 * j + 2 * e + 1];
          float y0 = x0, y1 = x1;
          if (KIND == EPI_GATE) {
            const float2 mm = __bfloat1622float2(a[j].h2[e]);
            y0 = silu(x0) * mm.x;
            y1 = silu(x1) * mm.y;
          } else if (has_aux) {
            const float2 rr = __bfloat1622float2(a[j].h2[e]);
            y0 = x0 + rr.x;
            y1 = x1 + rr.y;
          }
          r.h2[e] = __floats2bfloat162_rn(y0, y1);
        }
        *reinterpret_cast<uint4*>(stage + lane * kEpiPitchB16 + j * 16) = r.u;
      }
      __syncwarp();
      bf16* out = reinterpret_cast<bf16*>(g.out);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = i * 8 + (lane >> 2), seg = lane & 3;
        if (row0 + r < g.M)
          *reinterpret_cast<uint4*>(out + static_cast<long long>(row0 + r) * g.ldo + n0 + seg * 8) =
              *reinterpret_cast<const uint4*>(stage + r * kEpiPitchB16 + seg * 16);
      }
      __syncwarp();
    }
    return;
  }
  if (m >= g.M) return;
  // element by element (transposed output, or a ragged edge): all aux loads are
  // issued before any store so they overlap; an element's own load still
  // precedes its store, which keeps Y == residual aliasing safe
  float a[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int n = n0 + j;
    const long long o = TRANS ? static_cast<long long>(n) * g.ldo + m
                              : static_cast<long long>(m) * g.ldo + n;
    a[j] = 0.0f;
    if (n < g.N && (KIND == EPI_GATE || (KIND == EPI_RESID && g.aux != nullptr)))
      a[j] = to_f32(reinterpret_cast<const bf16*>(g.aux)[o]);
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int n = n0 + j;
    if (n < g.N) {
      const long long o = TRANS ? static_cast<long long>(n) * g.ldo + m
                                : static_cast<long long>(m) * g.ldo + n;
      epi_store_one<KIND>(g, o, n, v[j], a[j]);
    }
  }
}

// ------------------------------------------------------------------ kernel

constexpr int kSlotBytes = 16384;             // one 128-row x 128-byte epilogue block
constexpr int kMaxDynSmem = 232448;           // 227 KB per CTA on sm_100

template <int BN, bool A_MN, bool B_MN, int KIND, bool TRANS, int EW, bool PAIR>
struct Cfg {
  static constexpr int kBMT = PAIR ? 2 * BM : BM;   // tile rows (a pair: 128 per CTA)
  static constexpr int kBHalf = PAIR ? BN / 2 : BN; // B columns this CTA loads per tile
  static constexpr int kABytes = BM * BK * 2;   // 16 KB
  static constexpr int kBBytes = kBHalf * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  // TMA epilogue: bf16 outputs keep one 128 x 64 block per 64 output columns
  // (the whole tile's aux arrives ahead of the accumulator); f32 outputs
  // double-buffer 128 x 32 blocks per group of 4 epilogue warps
  static constexpr int kHalves = EW / 4;
  static constexpr bool kTmaEpi = !TRANS && (KIND == EPI_GATE || KIND == EPI_RESID || KIND == EPI_SOFTPLUS);
  static constexpr int kSlots = !kTmaEpi ? 0 : (KIND == EPI_SOFTPLUS ? 2 * kHalves : BN / 64);
  // TRANS (swap-AB decode): the element-wise epilogue needs no staging; the area
  // holds the aux of the cluster split-K reduction: for each of the BN output
  // columns, the 8-aligned run of tile rows around the CTA's reduction rows
  // (at most BM / 2 + 14 rows, since splits >= 2), at a pitch of kAuxPitch
  static constexpr int kAuxPitch = 80;
  static constexpr int kStageArea = TRANS ? BN * kAuxPitch * 2
                                          : (kSlots * kSlotBytes > EW * kEpiWarpBytes ? kSlots * kSlotBytes
                                                                                     : EW * kEpiWarpBytes);
  // cluster split-K with tiles of at most 64 columns (decode batches up to 64):
  // the splits push their partial rows into the reducing CTA's receive buffer
  // ([split][row of the CTA's slice][kCsplitPitch], at most BM + 8 rows)
  static constexpr bool kPush = TRANS && BN <= 64;
  static constexpr int kRecvBytes = kPush ? (BM + 8) * (BN + 4) * 4 : 0;
  static constexpr int kEpiBytes = kStageArea + kRecvBytes + (kTmaEpi ? 1024 /*bias*/ : 0);
  static constexpr int kFixed = 1024 /*align slack*/ + 512 /*barriers*/ + kEpiBytes;
  static constexpr int kStagesFit = (kMaxDynSmem - kFixed) / kStageBytes;
  static constexpr int kStageCap = 8;
  static constexpr int kStages = kStagesFit > kStageCap ? kStageCap : kStagesFit;
  static constexpr int kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                   : (2 * BN <= 256) ? 256 : 512;
  static constexpr uint32_t kIdesc = idesc_bf16(kBMT, BN, A_MN, B_MN);
  static constexpr size_t kSmem = static_cast<size_t>(kFixed) + static_cast<size_t>(kStages) * kStageBytes;
  // cluster split-K partial tile in the pipeline stages: BM rows of BN floats
  // at a pitch of BN + 4 (16-byte rows whose starts step by 4 banks)
  static constexpr int kCsplitPitch = BN + 4;
  static constexpr bool kCsplitFits = BM * kCsplitPitch * 4 <= kStages * kStageBytes;
  static_assert(kStages >= 2, "shared memory budget");
  static_assert(kSmem <= kMaxDynSmem, "shared memory budget");
  static_assert(EW == 4 || EW == 8, "one or two epilogue warps per TMEM lane quarter");
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "UMMA N for M=128, whole 32-column epilogue chunks");
  static_assert(!TRANS || EW == 4, "decode epilogue: one warp per TMEM lane quarter");
  static_assert(!B_MN || kBHalf % 64 == 0, "MN-major B tiles are whole 64-element atoms");
  static_assert(!PAIR || (!TRANS && !A_MN), "pairs serve the row-major prefill GEMMs");
};

struct TileCoord {
  int m, n, split, kb0, kb1;
  int n0, bn;          // first output column and width of this unit
  int tailk;           // -1, or the index among the K-split tail tiles
};

template <int BN>
__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& g, int t) {
  TileCoord c;
  c.tailk = -1;
  if (g.tail_ksplit > 1) {
    // K-split tail units come first in the schedule: unit t < nt is tail unit
    // t, the rest are the whole tiles.  With nt <= the number of CTA pairs,
    // each pair meets at most one tail unit, before any whole tile.
    const int nt = g.tiles - g.full_tiles;
    t = t < nt ? g.full_tiles + t : t - nt;
  }
  if (g.tail_ksplit > 1 && t >= g.full_tiles) {
    const int r = t - g.full_tiles;
    c.tailk = r / g.tail_ksplit;
    const int tile = g.full_tiles + c.tailk;
    c.m = tile % g.m_tiles;
    c.n = tile / g.m_tiles;
    c.bn = BN;
    c.n0 = c.n * BN;
    c.split = r % g.tail_ksplit;
    c.kb0 = c.split * g.tail_kbps;
    c.kb1 = min(g.k_blocks, c.kb0 + g.tail_kbps);
    return c;
  }
  if (g.tail_nsplit > 1 && t >= g.full_tiles) {
    const int r = t - g.full_tiles;
    const int tile = g.full_tiles + r / g.tail_nsplit;
    c.m = tile % g.m_tiles;
    c.n = tile / g.m_tiles;
    c.bn = BN / g.tail_nsplit;
    c.n0 = c.n * BN + (r % g.tail_nsplit) * c.bn;
    c.split = 0;
    c.kb0 = 0;
    c.kb1 = g.k_blocks;
    return c;
  }
  if (g.csplit) {             // unit t: split t % splits of tile t / splits
    c.split = t % g.splits;
    const int tile = t / g.splits;
    c.m = tile % g.m_tiles;
    c.n = tile / g.m_tiles;
  } else {
    c.m = t % g.m_tiles;
    const int r = t / g.m_tiles;
    c.n = r % g.n_tiles;
    c.split = r / g.n_tiles;
  }
  c.kb0 = c.split * g.kb_per_split;
  c.kb1 = min(g.k_blocks, c.kb0 + g.kb_per_split);
  c.n0 = c.n * BN;
  c.bn = BN;
  return c;
}

// ---------------------------------------------------------------- K-split tail
//
// Each CTA of a tail unit, once its rows of the partial tile are stored,
// writes this launch's epoch to its own flag in the caller's scratch (no
// atomics: the arrivals of one launch land at the same moment and must not
// queue on one word).  The flags' contents on entry are undefined; epochs come
// from a 48-bit sequence that a process starts at a random point and never
// repeats, so a flag holds the live epoch only once this launch has set it.

constexpr int kMaxTailSplits = 16;
constexpr int kTailLanes = 4;      // lanes summing one output's partials

__device__ __forceinline__ void tail_flag_set(unsigned long long* f, unsigned long long epoch) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(f), "l"(epoch) : "memory");
}

// One warp: bounded wait until all n flags hold the epoch.  False (the same
// in every lane) if the limit ran out (status recorded) or the CTA is aborting.
__device__ __forceinline__ bool tail_flags_wait(const unsigned long long* f, int n, unsigned long long epoch,
                                                volatile int* abort_flag, unsigned long long limit) {
  const int lane = threadIdx.x & 31;
  const long long t0 = clock64();
  for (;;) {
    bool mine = true;
    for (int i = lane; i < n; i += 32) {
      unsigned long long v;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(f + i) : "memory");
      mine &= v == epoch;
    }
    if (__all_sync(0xffffffffu, mine)) return true;
    const bool late = static_cast<unsigned long long>(clock64() - t0) > limit;
    if (__any_sync(0xffffffffu, *abort_flag != 0 || late)) {
      if (lane == 0 && !*abort_flag) {
        *abort_flag = 1;
        record_status(kStatusTimeout);
      }
      return false;
    }
    __nanosleep(128);
  }
}

// Sums the tail tiles' partials and applies the epilogue: output float4 groups
// of kTailLanes lanes, warp w of `warps` taking groups w, w + warps, ...  The
// lanes of a group sum every kTailLanes-th split, then combine by shuffles (a
// fixed order: the result does not depend on which warp runs it).  A few
// warps per SM run this, so each lane keeps the loads of kTailBatch groups in
// flight at once.
constexpr int kTailBatch = 4;

template <int BN, int BMT, int KIND>
__device__ __forceinline__ void tail_reduce_warps(const GemmArgs& g, int ntail, long long w0, long long warps) {
  constexpr int Q = BN / 4, LPG = kTailLanes, PER = kMaxTailSplits / LPG, U = kTailBatch;
  constexpr bool kAuxKind = KIND == EPI_GATE || KIND == EPI_RESID;
  const int lane = threadIdx.x & 31, sub = lane % LPG;
  const long long total = static_cast<long long>(ntail) * BMT * Q;   // output float4s
  for (long long wb = w0; wb * (32 / LPG) < total; wb += U * warps) {
    float4 x[U][PER];
    uint2 aux4[U];
    long long o[U];
    int n[U];
    bool live[U], vec4[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long e = (wb + u * warps) * (32 / LPG) + lane / LPG;
      const int i = static_cast<int>(e / (BMT * Q));
      const int lr = static_cast<int>((e / Q) % BMT), lq = static_cast<int>(e % Q);
      const int tile = g.full_tiles + i;
      const int m = (tile % g.m_tiles) * BMT + lr;
      n[u] = (tile / g.m_tiles) * BN + 4 * lq;
      live[u] = e < total && m < g.M && n[u] < g.N;
      const float* base = g.tail_part + (static_cast<long long>(i) * g.tail_ksplit * BMT + lr) * BN + 4 * lq;
      o[u] = static_cast<long long>(m) * g.ldo + n[u];
      // the aux (M or the residual) of the reducing lane's 4 outputs, loaded
      // together with the partials so the round trips overlap
      vec4[u] = n[u] + 4 <= g.N && (o[u] & 3) == 0;
      aux4[u] = make_uint2(0u, 0u);
      if (kAuxKind && g.aux != nullptr && live[u] && sub == 0 && vec4[u])
        aux4[u] = __ldcg(reinterpret_cast<const uint2*>(reinterpret_cast<const bf16*>(g.aux) + o[u]));
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int sp = sub + j * LPG;
        const bool on = live[u] && sp < g.tail_ksplit;
        x[u][j] = ldcg_or_zero(base + (on ? static_cast<long long>(sp) * BMT * BN : 0), on);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float4 acc = x[u][0];
#pragma unroll
      for (int j = 1; j < PER; ++j) {
        acc.x += x[u][j].x; acc.y += x[u][j].y; acc.z += x[u][j].z; acc.w += x[u][j].w;
      }
#pragma unroll
      for (int off = LPG / 2; off >= 1; off >>= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
      }
      if (!live[u] || sub != 0) continue;
      const float v[4] = {acc.x, acc.y, acc.z, acc.w};
      if (kAuxKind && vec4[u]) {
        // 4 bf16 outputs as one 8-byte store
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&aux4[u]);
        const float2 a01 = __bfloat1622float2(a2[0]), a23 = __bfloat1622float2(a2[1]);
        const float a[4] = {a01.x, a01.y, a23.x, a23.y};
        float r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) r[j] = KIND == EPI_GATE ? silu(v[j]) * a[j] : v[j] + a[j];
        uint2 packed;
        *reinterpret_cast<__nv_bfloat162*>(&packed.x) = __floats2bfloat162_rn(r[0], r[1]);
        *reinterpret_cast<__nv_bfloat162*>(&packed.y) = __floats2bfloat162_rn(r[2], r[3]);
        *reinterpret_cast<uint2*>(reinterpret_cast<bf16*>(g.out) + o[u]) = packed;
        continue;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (n[u] + j >= g.N) break;
        float a = 0.0f;
        if (KIND == EPI_GATE || (KIND == EPI_RESID && g.aux != nullptr))
          a = to_f32(reinterpret_cast<const bf16*>(g.aux)[o[u] + j]);
        epi_store_one<KIND>(g, o[u] + j, n[u] + j, v[j], a);
      }
    }
  }
}

template <int BN, bool A_MN, bool B_MN, int KIND, bool TRANS, int EW, bool PAIR>
__global__ void __launch_bounds__(gemm_threads(EW), 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmAux,
                   const __grid_constant__ CUtensorMap tmOut, const GemmArgs g) {
  using C = Cfg<BN, A_MN, B_MN, KIND, TRANS, EW, PAIR>;
  constexpr int S = C::kStages;
  static_assert(!TRANS || C::kCsplitFits, "cluster split-K partial tile exceeds the pipeline stages");
  // work units: one per CTA, or one per CTA pair (cluster of 2)
  const int rank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const int unit0 = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int ustride = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * C::kABytes;
  uint8_t* epi_area = smem + S * C::kStageBytes;          // 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_area + C::kEpiBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;      // [2]
  uint64_t* tempty = tfull + 2;     // [2]
  uint64_t* drain = tempty + 2;     // [1]
  uint64_t* auxf = drain + 1;       // [4] aux block landed (TMA epilogue)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(auxf + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;
  uint8_t* epi_stage = epi_area;                           // fallback staging, EW x kEpiWarpBytes
  float* epi_vec = reinterpret_cast<float*>(epi_area + C::kStageArea);  // tile's bias

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], PAIR ? 2 * EW : EW);
    }
    mbar_init(drain, 1);
    for (int j = 0; j < 4; ++j) mbar_init(&auxf[j], 1);
    *abort_flag = 0;
    *last_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (g.tail_nsplit > 1 && !B_MN) prefetch_tmap(&tmB2);
    if (C::kTmaEpi && g.tma_epi) {
      if (KIND != EPI_SOFTPLUS && g.aux != nullptr) prefetch_tmap(&tmAux);
      prefetch_tmap(&tmOut);
    }
  }
  if (warp == 1) {
    if (PAIR) {   // warp 1 of both CTAs: the same columns in each CTA's TMEM
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(C::kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(C::kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  if (PAIR) cluster_sync();   // the peer's barriers exist before any load or arrive targets them
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const unsigned long long wl = g.wait_limit ? g.wait_limit : kWaitCycles;
  // the set-up above touched only this CTA's shared memory and TMEM; global
  // reads and writes wait for the kernel before this one on the stream,
  // except the producer's loads of operands flagged independent of it
  // (a_early / b_early), which it orders itself
  if (warp != 0 || !(g.a_early || g.b_early)) pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;  // per stage: outstanding load, its parity
      bool ok = true;
      // a_early: the A tiles of the first S k-blocks (stages that are free from
      // the start) are issued before griddepcontrol.wait, their B tiles after it
      int n_early = 0;
      const bool split_wait = g.a_early && !g.b_early;
      auto load = [&](void* dst, const CUtensorMap* map, int st, int c0, int c1) {
        if (PAIR) tma_load_2d_pair(dst, map, &full[st], c0, c1);
        else tma_load_2d(dst, map, &full[st], c0, c1);
      };
      auto load_a = [&](int st, int arow, int kb) {
        uint8_t* a_dst = sA + st * C::kABytes;
        if (A_MN) {  // [K, M] in memory: boxes of 64 m x 64 k
          load(a_dst, &tmA, st, arow, kb * BK);
          load(a_dst + 8192, &tmA, st, arow + 64, kb * BK);
        } else {     // [M, K]: one box of 64 k x 128 m
          load(a_dst, &tmA, st, kb * BK, arow);
        }
      };
      auto load_b = [&](int st, int hb, int bcol, int kb) {
        uint8_t* b_dst = sB + st * C::kBBytes;
        const int kb_b = g.b_k_wrap > 0 ? (kb * BK) % g.b_k_wrap : kb * BK;
        if (B_MN) {  // [K, N]: boxes of 64 n x 64 k
#pragma unroll
          for (int j = 0; j < C::kBHalf / 64; ++j)
            if (64 * j < hb) load(b_dst + j * 8192, &tmB, st, bcol + 64 * j, kb_b);
        } else {     // [N, K]: one box of 64 k x kBHalf n (tail units: 64 k x hb n)
          load(b_dst, hb == C::kBHalf ? &tmB : &tmB2, st, kb_b, bcol);
        }
      };
      if (split_wait) {
        for (int t = unit0; t < g.tiles && n_early < S; t += ustride) {
          const TileCoord c = tile_coord<BN>(g, t);
          const int hb = PAIR ? c.bn / 2 : c.bn;
          for (int kb = c.kb0; kb < c.kb1 && n_early < S; ++kb, ++n_early) {
            if (rank == 0) mbar_arrive_expect_tx(&full[n_early], (C::kABytes + hb * BK * 2) * (PAIR ? 2 : 1));
            load_a(n_early, c.m * C::kBMT + rank * BM, kb);
          }
        }
      }
      // a_early: wait before the first B tile; b_early: every operand is
      // independent of the previous kernel and the producer never waits
      if (split_wait) pdl_wait();
      int item = 0;                   // position in this CTA's (tile, k-block) sequence
      for (int t = unit0; t < g.tiles && ok; t += ustride) {
        const TileCoord c = tile_coord<BN>(g, t);
        const int arow = c.m * C::kBMT + rank * BM;       // this CTA's A rows
        const int hb = PAIR ? c.bn / 2 : c.bn;            // this CTA's B columns
        const int bcol = c.n0 + rank * hb;
        for (int kb = c.kb0; kb < c.kb1; ++kb, ++item) {
          if (item < n_early) {
            // A already issued and the barrier armed: the B half only (stage == item)
            load_b(stage, hb, bcol, kb);
          } else {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, wl)) { ok = false; break; }
            // the leader's barrier counts the bytes of both CTAs of a pair
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], (C::kABytes + hb * BK * 2) * (PAIR ? 2 : 1));
            load_a(stage, arow, kb);
            load_b(stage, hb, bcol, kb);
          }
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag && rank == 0) {
        // drain: every issued load must land before the CTA's smem goes away
        // (in a pair the leader's barriers count the peer's loads too, and the
        // peer stays resident until the leader reaches the final cluster barrier)
        for (int s = 0; s < S; ++s)
          if (issued_mask & (1u << s)) {
            volatile int dummy = 0;
            mbar_wait(&full[s], (issued_parity >> s) & 1u, &dummy, kDrainCycles);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = unit0; t < g.tiles && ok; t += ustride) {
        const TileCoord c = tile_coord<BN>(g, t);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, wl)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        const uint32_t idesc = c.bn == BN ? C::kIdesc : idesc_bf16(C::kBMT, c.bn, A_MN, B_MN);
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, wl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = A_MN ? sdesc_sw128(a_addr + kk * 2048, 8192, 1024)
                                     : sdesc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? sdesc_sw128(b_addr + kk * 2048, 8192, 1024)
                                     : sdesc_sw128(b_addr + kk * 32, 16, 1024);
            if (PAIR) tc_mma_bf16_pair(d_tmem, ad, bd, idesc, (kb > c.kb0 || kk > 0) ? 1u : 0u);
            else tc_mma_bf16(d_tmem, ad, bd, idesc, (kb > c.kb0 || kk > 0) ? 1u : 0u);
          }
          if (PAIR) tc_commit_pair(&empty[stage]);
          else tc_commit(&empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (PAIR) tc_commit_pair(&tfull[acc]);
        else tc_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // all MMAs issued by this thread complete before TMEM is released
      if (PAIR) tc_commit2(drain);
      else tc_commit(drain);
      volatile int dummy = 0;
      mbar_wait(drain, 0, &dummy, kDrainCycles);
    }
  } else {
    // ------------------------------------------------------ epilogue
    constexpr int H = C::kHalves;            // epilogue warps per TMEM lane quarter
    constexpr int EPI_THREADS = 32 * EW;
    const int quarter = warp & 3;            // TMEM lanes [32*quarter, +32)
    const int ep_tid = threadIdx.x - 64;     // 0 .. 32*EW - 1
    const int half = (warp - 2) / 4;         // which of the quarter's warps: column blocks half, half + H, ...
    uint8_t* my_stage = epi_stage + (warp - 2) * kEpiWarpBytes;
    if (TRANS && g.csplit && g.splits > 1 && KIND != EPI_F32_PARTIAL &&
        (KIND == EPI_GATE || (KIND == EPI_RESID && g.aux != nullptr)) && blockIdx.x < g.tiles) {
      // cluster split-K: the aux values (M or the residual) around the rows this
      // CTA will reduce come into shared memory while the main loop runs.  In
      // memory a column n of the transposed output holds its rows m
      // contiguously, so each thread copies whole 16-byte runs of 8 rows (the
      // rows [ra, rb) are the reduction rows widened to multiples of 8), all
      // of its loads in flight at once.
      const TileCoord c = tile_coord<BN>(g, blockIdx.x);
      const int R = (BM + g.splits - 1) / g.splits;
      const int r0 = c.split * R, r1 = min(BM, r0 + R);
      const int ra = r0 & ~7, rb = min(BM, (r1 + 7) & ~7), nr8 = max(0, rb - ra) / 8;
      const int ncols = min(c.bn, g.N - c.n0);
      const int chunks = ncols * nr8;
      bf16* pre = reinterpret_cast<bf16*>(epi_area);
      const bf16* aux = reinterpret_cast<const bf16*>(g.aux);
      constexpr int kPre = 8;
      for (int c0i = ep_tid; c0i < chunks; c0i += kPre * (32 * EW)) {
        uint4 v[kPre];
#pragma unroll
        for (int u = 0; u < kPre; ++u) {
          const int ch = c0i + u * 32 * EW;
          const int n = ch < chunks ? ch / nr8 : 0, r8 = ch < chunks ? ch % nr8 : 0;
          const int m = c.m * BM + ra + 8 * r8;
          v[u] = make_uint4(0u, 0u, 0u, 0u);
          if (ch < chunks && m + 8 <= g.M)   // M is a multiple of 8: runs are whole or outside
            v[u] = *reinterpret_cast<const uint4*>(aux + static_cast<long long>(c.n0 + n) * g.ldo + m);
        }
#pragma unroll
        for (int u = 0; u < kPre; ++u) {
          const int ch = c0i + u * 32 * EW;
          if (ch < chunks)
            *reinterpret_cast<uint4*>(pre + (ch / nr8) * C::kAuxPitch + 8 * (ch % nr8)) = v[u];
        }
      }
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t aux_phase = 0;    // parity bit per aux slot
    int sp_local = 0;          // softplus chunks this warp has staged (slot double buffering)
    bool tail_summed = false;  // this CTA's share of the K-split tail outputs is done
    // the K-split tail: CTA pairs with a bf16 epilogue (the host plans it for no other)
    constexpr bool kTailCode = PAIR && (KIND == EPI_GATE || KIND == EPI_RESID);
    const bool has_aux = KIND == EPI_GATE || (KIND == EPI_RESID && g.aux != nullptr);
    for (int t = unit0; t < g.tiles; t += ustride) {
      const TileCoord c = tile_coord<BN>(g, t);
      const int arow = c.m * C::kBMT + rank * BM;     // this CTA's first output row
      const bool split = (g.splits > 1 && KIND != EPI_F32_PARTIAL) || c.tailk >= 0;
      const bool tma = C::kTmaEpi && g.tma_epi && !split;
      if (tma) {
        // the tile's aux blocks (M or the residual) and bias are fetched while
        // its main loop still runs; the slots are free because every store of
        // the previous tile has finished reading them (barrier at tile end)
        if (has_aux && ep_tid == 0) {
#pragma unroll
          for (int j = 0; j < C::kSlots; ++j) {
            const int n0 = c.n0 + 64 * j;
            if (64 * j < c.bn && n0 < g.N) {
              mbar_arrive_expect_tx(&auxf[j], kSlotBytes);
              tma_load_2d(epi_area + j * kSlotBytes, &tmAux, &auxf[j], n0, arow);
            }
          }
        }
        if (KIND == EPI_SOFTPLUS)
          for (int i = ep_tid; i < c.bn; i += EPI_THREADS)
            epi_vec[i] = c.n0 + i < g.N ? g.vec[c.n0 + i] : 0.0f;
      }
      if constexpr (kTailCode) if (g.tail_ksplit > 1 && c.tailk < 0 && !tail_summed) {
        // The CTA's first whole tile.  Every CTA pair ran its tail unit (if
        // any) first, so the tail's partials are in or nearly so: once every
        // flag is (both CTAs of every tail unit), this CTA's epilogue warps sum
        // their share of the tail outputs while the tile's main loop runs on
        // the tensor cores.  One warp waits; the barrier hands its verdict (an
        // aborting CTA skips the sum) to the others.
        tail_summed = true;
        const int nt = g.tiles - g.full_tiles;
        named_bar_sync<EPI_THREADS>();
        if (warp == 2) {
          const bool in = tail_flags_wait(g.tail_flags, 2 * nt, g.tail_epoch, abort_flag,
                                          g.wait_limit ? g.wait_limit : kWaitCycles);
          if (lane == 0) *last_flag = in ? 1 : 0;
        }
        named_bar_sync<EPI_THREADS>();
        if (*last_flag) {
          __threadfence();
          tail_reduce_warps<BN, C::kBMT, KIND>(g, nt / g.tail_ksplit,
                                               static_cast<long long>(blockIdx.x) * EW + (warp - 2),
                                               static_cast<long long>(gridDim.x) * EW);
        }
      }
      bool ok = true;
      // stall_test: auxf[3] is never armed in the element-wise (TRANS) epilogue,
      // so this wait can only end by running out of its limit
      if (g.stall_test) ok = mbar_wait(&auxf[3], 0, abort_flag, wl);
      ok = ok && mbar_wait(&tfull[acc], acc_phase, abort_flag, wl);
      // the split-K and TMA paths synchronise the epilogue warps, so they must
      // agree on leaving the loop together (the barrier also publishes epi_vec)
      if (split || tma) ok = epi_agree<EPI_THREADS>(ok);
      if (!ok) break;
      tc_fence_after();
      const int row = arow + quarter * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      if (tma) {
        // rows r of the tile live at r * 128 bytes of a slot, 16-byte chunks
        // 128-byte swizzled (the layout TMA reads and writes)
        const int r = quarter * 32 + lane;
        if (KIND == EPI_SOFTPLUS) {
#pragma unroll 1
          for (int ch = half; ch < c.bn / 32; ch += H) {
            const int n0 = c.n0 + 32 * ch;
            if (n0 >= g.N) break;
            uint8_t* blk = epi_area + (half * 2 + (sp_local & 1)) * kSlotBytes;
            if (sp_local >= 2) {      // this slot's store from two chunks ago has read it
              if (lane == 0) bulk_wait_read<1>();
              __syncwarp();
            }
            ++sp_local;
            uint32_t rr[32];
            tmem_ld_32x32b_x32(t_row + 32 * ch, rr);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float4 b = *reinterpret_cast<const float4*>(epi_vec + 32 * ch + 4 * k);
              float4 o;
              o.x = softplus(__uint_as_float(rr[4 * k + 0]) + b.x);
              o.y = softplus(__uint_as_float(rr[4 * k + 1]) + b.y);
              o.z = softplus(__uint_as_float(rr[4 * k + 2]) + b.z);
              o.w = softplus(__uint_as_float(rr[4 * k + 3]) + b.w);
              *reinterpret_cast<float4*>(blk + r * 128 + ((k ^ (r & 7)) << 4)) = o;
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmOut, blk + quarter * 32 * 128, n0, arow + quarter * 32);
              bulk_commit();
            }
          }
        } else {
          // slot j (64 columns) goes to the quarter's warp j % H; every warp runs
          // the same number of rounds, since each round ends in a barrier
#pragma unroll 1
          for (int j0 = 0; j0 < C::kSlots; j0 += H) {
            const int j = j0 + half;
            const int n0 = c.n0 + 64 * j;
            const bool mine = j < C::kSlots && 64 * j < c.bn && n0 < g.N;
            if (has_aux) {
              ok = mine ? mbar_wait(&auxf[j], (aux_phase >> j) & 1u, abort_flag, wl) : true;
              ok = epi_agree<EPI_THREADS>(ok);
              if (!ok) break;
              if (mine) aux_phase ^= 1u << j;
            }
            if (!mine) continue;
            uint8_t* blk = epi_area + j * kSlotBytes;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
              uint32_t rr[32];
              tmem_ld_32x32b_x32(t_row + 64 * j + 32 * h, rr);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const int k = 4 * h + kk;
                uint4* addr = reinterpret_cast<uint4*>(blk + r * 128 + ((k ^ (r & 7)) << 4));
                Pack16 a, o;
                if (has_aux) a.u = *addr;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float x0 = __uint_as_float(rr[8 * kk + 2 * e]);
                  const float x1 = __uint_as_float(rr[8 * kk + 2 * e + 1]);
                  float y0 = x0, y1 = x1;
                  if (KIND == EPI_GATE) {
                    const float2 mm = __bfloat1622float2(a.h2[e]);
                    y0 = silu(x0) * mm.x;
                    y1 = silu(x1) * mm.y;
                  } else if (has_aux) {
                    const float2 rs = __bfloat1622float2(a.h2[e]);
                    y0 = x0 + rs.x;
                    y1 = x1 + rs.y;
                  }
                  o.h2[e] = __floats2bfloat162_rn(y0, y1);
                }
                *addr = o.u;
              }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmOut, blk + quarter * 32 * 128, n0, arow + quarter * 32);
              bulk_commit();
            }
          }
          if (!ok) break;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR && rank != 0) mbar_arrive_leader(&tempty[acc]);
          else mbar_arrive(&tempty[acc]);
        }
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        // every store of this tile has read its slot before the next tile's
        // aux loads and bias overwrite them
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        sp_local = 0;
        named_bar_sync<EPI_THREADS>();
        continue;
      }
#pragma unroll 1
      for (int ch = half; ch < c.bn / 32; ch += H) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + ch * 32, r);
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        const int n0 = c.n0 + ch * 32;
        if (c.tailk >= 0) {
          // K-split tail unit: this CTA's rows of the partial tile, row-major
          float* part = g.tail_part +
                        ((static_cast<long long>(c.tailk) * g.tail_ksplit + c.split) * C::kBMT +
                         (row - c.m * C::kBMT)) * BN + (n0 - c.n0);
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            __stcg(reinterpret_cast<float4*>(part + j), make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
        } else if (split && g.csplit && C::kPush) {
          // cluster split-K, push: tile row r belongs to the CTA (cluster rank)
          // r / R that reduces it; this split's 32 values of the row go
          // straight into that CTA's receive buffer (distributed shared
          // memory stores, no wait), at [split * R + r % R]
          const int r = quarter * 32 + lane;
          const int R = (BM + g.splits - 1) / g.splits;
          const int owner = r / R;
          const uint32_t local = smem_u32(epi_area + C::kStageArea) +
                                 static_cast<uint32_t>(((c.split * R + r - owner * R) * C::kCsplitPitch + ch * 32) * 4);
          const uint32_t remote = mapa_shared(local, static_cast<uint32_t>(owner));
#pragma unroll
          for (int j = 0; j < 32; j += 4) st_dsmem_f32x4(remote + 4u * j, make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
        } else if (split && g.csplit) {
          // cluster split-K, pull: this split's partial tile stays in this CTA's
          // (now idle) pipeline shared memory, row-major at kCsplitPitch; the
          // cluster's CTAs read it there after the cluster barrier
          float* dst = reinterpret_cast<float*>(smem) + (quarter * 32 + lane) * C::kCsplitPitch + ch * 32;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        } else if (split) {
          // this split's partial tile, summed in split order by the last CTA
          float* part = g.partials + static_cast<long long>(c.split) * g.split_stride;
          if (row < g.M) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int n = n0 + j;
              if (n < g.N) {
                const long long o = TRANS ? static_cast<long long>(n) * g.ldo + row
                                          : static_cast<long long>(row) * g.ldo + n;
                __stcg(part + o, v[j]);
              }
            }
          }
        } else if (KIND == EPI_F32_PARTIAL) {
          GemmArgs gs = g;
          gs.out = reinterpret_cast<float*>(g.out) + static_cast<long long>(c.split) * g.split_stride;
          epi_chunk<KIND, TRANS>(gs, row - lane, lane, n0, v, my_stage);
        } else {
          epi_chunk<KIND, TRANS>(g, row - lane, lane, n0, v, my_stage);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR && rank != 0) mbar_arrive_leader(&tempty[acc]);
        else mbar_arrive(&tempty[acc]);
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }

      if (split && !g.csplit && c.tailk < 0) {
        // The last CTA to finish a split-K tile sums the partials in split
        // order (deterministic), applies the final op and resets the counter.
        __threadfence();
        named_bar_sync<EPI_THREADS>();
        if (ep_tid == 0) {
          const int tile_mn = c.m + g.m_tiles * c.n;
          const int prev = atomicAdd(g.counters + tile_mn, 1);
          const int last = (prev == g.splits - 1);
          if (last) g.counters[tile_mn] = 0;
          *last_flag = last;
        }
        named_bar_sync<EPI_THREADS>();
        if (*last_flag) {
          __threadfence();
#pragma unroll 1
          for (int ch = half; ch < BN / 32; ch += H) {
            const int n0 = c.n0 + ch * 32;
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.0f;
            // split order is fixed; each split's 32 loads are in flight together
#pragma unroll 1
            for (int sp = 0; sp < g.splits; ++sp) {
              const float* part = g.partials + static_cast<long long>(sp) * g.split_stride;
              float x[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int n = n0 + j;
                const long long o = TRANS ? static_cast<long long>(n) * g.ldo + row
                                          : static_cast<long long>(row) * g.ldo + n;
                x[j] = (n < g.N && row < g.M) ? __ldcg(part + o) : 0.0f;
              }
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] += x[j];
            }
            epi_chunk<KIND, TRANS>(g, row - lane, lane, n0, v, my_stage);
          }
        }
        named_bar_sync<EPI_THREADS>();
      }
      if constexpr (kTailCode) if (c.tailk >= 0) {
        // this CTA's rows of a K-split tail unit are stored: publish them
        __threadfence();
        named_bar_sync<EPI_THREADS>();
        if (ep_tid == 0) tail_flag_set(g.tail_flags + 2 * (c.tailk * g.tail_ksplit + c.split) + rank, g.tail_epoch);
      }
    }
  }

  if (C::kTmaEpi && warp >= 2 && lane == 0) bulk_wait_read<0>();   // no store still reading smem
  tc_fence_before();
  // a pair ends together: the leader's MMAs write the peer's TMEM and read its
  // shared memory, and the peer's arrivals target the leader's barriers
  if (PAIR) cluster_sync();
  else __syncthreads();
  tc_fence_after();
  if (!PAIR && C::kPush && g.csplit && g.splits > 1 && KIND != EPI_F32_PARTIAL && blockIdx.x < g.tiles) {
    // cluster split-K, push: every split has stored its rows into the
    // reducing CTAs' receive buffers; after one cluster barrier (which orders
    // those stores) each CTA sums its rows [split * R, +R) locally, in split
    // order, and applies the final op.  Nothing touches a peer's shared
    // memory after the barrier, so no second barrier is needed before exit.
    // Thread: row tid % 64 of the CTA's rows (at most 64: splits >= 2), 4
    // consecutive columns per pass, the CTA's blockDim / 64 threads of a row
    // on every (blockDim / 64)-th column group.
    cluster_sync();
    const TileCoord c = tile_coord<BN>(g, blockIdx.x);
    const int splits = g.splits, gM = g.M, gN = g.N;
    const long long ldo = g.ldo;
    const int R = (BM + splits - 1) / splits;
    const int r0 = c.split * R, r1 = min(BM, r0 + R);
    const int nrows = max(0, r1 - r0), ncols = min(c.bn, gN - c.n0);
    const bool has_aux = KIND == EPI_GATE || (KIND == EPI_RESID && g.aux != nullptr);
    const float* recv = reinterpret_cast<const float*>(epi_area + C::kStageArea);
    const bf16* pre = reinterpret_cast<const bf16*>(epi_area);
    const int ra = r0 & ~7;
    const int lr = threadIdx.x & 63, gstep = blockDim.x >> 6;
    const int mm = c.m * BM + r0 + lr;
    if (lr < nrows && mm < gM) {
      for (int lc = 4 * (threadIdx.x >> 6); lc < ncols; lc += 4 * gstep) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp = 0; sp < splits; ++sp) {
          const float4 x = ld_shared_f4(recv + (sp * R + lr) * C::kCsplitPitch + lc);
          v.x += x.x; v.y += x.y; v.z += x.z; v.w += x.w;
        }
        const float w[4] = {v.x, v.y, v.z, v.w};
        const int nn = c.n0 + lc;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (nn + k >= gN) break;
          const float a = has_aux ? ld_shared_bf16(pre + (lc + k) * C::kAuxPitch + r0 + lr - ra) : 0.0f;
          epi_store_one<KIND>(g, (nn + k) * ldo + mm, nn + k, w[k], a);
        }
      }
    }
  } else if (!PAIR && g.csplit && g.splits > 1 && KIND != EPI_F32_PARTIAL && blockIdx.x < g.tiles) {
    // cluster split-K, pull: every CTA of the cluster holds its partial tile in its
    // shared memory; CTA `split` (cluster rank `split`) sums rows
    // [split * R, +R) of the tile over the splits in split order, reading the
    // peers' tiles 16 bytes at a time through distributed shared memory, and
    // applies the final op.  Thread: 4 consecutive columns of one row,
    // consecutive threads on consecutive rows.
    cluster_sync();
    const TileCoord c = tile_coord<BN>(g, blockIdx.x);
    const int R = (BM + g.splits - 1) / g.splits;
    const int r0 = c.split * R, r1 = min(BM, r0 + R);
    const int nrows = max(0, r1 - r0), ncols = min(c.bn, g.N - c.n0);
    const int total = nrows * ((ncols + 3) / 4);
    const bool has_aux = KIND == EPI_GATE || (KIND == EPI_RESID && g.aux != nullptr);
    const uint32_t base = smem_u32(smem);
    const bf16* pre = reinterpret_cast<const bf16*>(epi_area);   // aux rows (TRANS)
    // kRed elements per thread and pass; every split's loads of a pass are
    // issued before the first add, and the adds run in split order
    constexpr int kRed = 2;
    constexpr int kMaxCsplit = 8;
    const int ra = r0 & ~7;   // first row of the prefetched aux runs (TRANS)
    for (int e0 = threadIdx.x; e0 < total; e0 += kRed * blockDim.x) {
      int mm[kRed], nn[kRed], lrs[kRed], lcs[kRed];
      uint32_t off[kRed];
      bool live[kRed];
      float a[kRed][4];
#pragma unroll
      for (int u = 0; u < kRed; ++u) {
        const int e = e0 + u * static_cast<int>(blockDim.x);
        lrs[u] = e < total ? e % nrows : 0;
        lcs[u] = 4 * (e < total ? e / nrows : 0);
        const int lr = r0 + lrs[u];
        mm[u] = c.m * BM + lr;
        nn[u] = c.n0 + lcs[u];
        live[u] = e < total && mm[u] < g.M;
        off[u] = static_cast<uint32_t>(lr * C::kCsplitPitch + lcs[u]) * 4u;
      }
      float4 x[kMaxCsplit][kRed];
#pragma unroll
      for (int sp = 0; sp < kMaxCsplit; ++sp) {
        if (sp < g.splits) {
          const uint32_t peer = mapa_shared(base, static_cast<uint32_t>(sp));
#pragma unroll
          for (int u = 0; u < kRed; ++u) x[sp][u] = ld_dsmem_f32x4(peer + off[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < kRed; ++u) {
#pragma unroll
        for (int k = 0; k < 4; ++k) a[u][k] = 0.0f;
        if (has_aux && live[u]) {
          if (TRANS) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              a[u][k] = __bfloat162float(pre[(lcs[u] + k) * C::kAuxPitch + r0 + lrs[u] - ra]);
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              if (nn[u] + k < g.N)
                a[u][k] = to_f32(reinterpret_cast<const bf16*>(g.aux)[static_cast<long long>(mm[u]) * g.ldo + nn[u] + k]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kRed; ++u) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int sp = 0; sp < kMaxCsplit; ++sp)
          if (sp < g.splits) { v.x += x[sp][u].x; v.y += x[sp][u].y; v.z += x[sp][u].z; v.w += x[sp][u].w; }
        if (!live[u]) continue;
        const float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (nn[u] + k >= g.N) break;
          const long long o = TRANS ? static_cast<long long>(nn[u] + k) * g.ldo + mm[u]
                                    : static_cast<long long>(mm[u]) * g.ldo + nn[u] + k;
          epi_store_one<KIND>(g, o, nn[u] + k, w[k], a[u][k]);
        }
      }
    }
    // no CTA leaves (and frees its shared memory) while a peer still reads it
    cluster_sync();
  }
  if (warp == 1) {
    if (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(C::kTmemCols)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(C::kTmemCols)
                   : "memory");
  }
}

}  // namespace tc
}  // namespace sambay
