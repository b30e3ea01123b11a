// Mamba selective-scan kernels of the SambaY memory-readout path (sm_100a).
//
// The scan (Gu & Dao 2023, "Mamba", section 3.2 / Algorithm 2) as the
// SambaY self-decoder's last SSM layer computes it; its readout y is the
// memory M that the Gated Memory Unit reuses ("Decoder-Hybrid-Decoder
// Architecture for Efficient Reasoning with Long Generation", Paper-Notes
// page, 方法详解 > 关键设计):
//
//   uc_t  = SiLU(conv_b + sum_k conv_w[k] u_{t-K+1+k})      causal depthwise conv
//   h_t   = exp(dt_t A) h_{t-1} + dt_t B_t uc_t             per (channel, state)
//   M_t   = sum_n C_t[n] h_t[n] + D uc_t
//
// Layouts: u, M [B, L, Di] (channel fastest); dt [B*L, Di] f32;
// xdbl [B*L, R + 2N] f32 holding (delta | B | C); h [B, Di, N] f32;
// conv state [B, Di, K] (last K inputs, oldest first).  N = 16, K = 4.
//
// uc, the conv output, is float32 [B*L, Di] in float32 mode.  In bfloat16
// mode it is kept as a split pair [B*L, 2*Di]: columns [0, Di) hold
// hi = bf16(uc), columns [Di, 2Di) hold lo = bf16(uc - hi).  hi + lo carries
// uc to ~2^-17 relative, so the scan works on (nearly) float32 uc, and the
// x_proj GEMM on bf16 tensor cores sums hi W^T + lo W^T over a K of 2*Di
// without rounding uc to bf16.  The delta operand of dt_proj is split the
// same way.
#pragma once

#include "common.cuh"

namespace sambay {
namespace scan {

constexpr int kN = 16;   // d_state
constexpr int kK = 4;    // d_conv

// ---------------------------------------------------------------- cp.async

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ------------------------------------------------------- conv1d + SiLU (prefill)
//
// One thread: VEC consecutive channels (16 bytes of T) x TT consecutive
// tokens, with a (K-1)-token halo taken from the previous tokens, the caller's
// conv state (continuing prompt) or zeros (fresh prompt).

template <typename T>
struct ConvParams {
  const T* u;            // [B, L, Di]
  const T* conv_state;   // [B, Di, K] (read only here)
  const T* conv_w;       // [Di, K]
  const T* conv_b;       // [Di]
  T* uc;                 // [B*L, Di] (f32) or [B*L, 2*Di] split pair (bf16)
  int B, L, Di;
  int zero_init;
};

// Stores VEC conv outputs of one token row: float32 as is; bf16 as the split
// pair (hi at column c, lo at column Di + c of a 2*Di row).
template <typename T, int VEC>
__device__ __forceinline__ void store_uc(T* uc, long long row, int Di, int c0, const float (&y)[VEC]) {
  static_assert(VEC * sizeof(T) == 16 || VEC * sizeof(T) == 8, "16- or 8-byte vectors");
  if constexpr (sizeof(T) == 2) {
    __nv_bfloat162 hi[VEC / 2], lo[VEC / 2];
#pragma unroll
    for (int v = 0; v < VEC; v += 2) {
      hi[v / 2] = __floats2bfloat162_rn(y[v], y[v + 1]);
      const float2 back = __bfloat1622float2(hi[v / 2]);
      lo[v / 2] = __floats2bfloat162_rn(y[v] - back.x, y[v + 1] - back.y);
    }
    if constexpr (VEC == 8) {
      *reinterpret_cast<uint4*>(uc + row * 2 * Di + c0) = *reinterpret_cast<const uint4*>(hi);
      *reinterpret_cast<uint4*>(uc + row * 2 * Di + Di + c0) = *reinterpret_cast<const uint4*>(lo);
    } else {
      *reinterpret_cast<uint2*>(uc + row * 2 * Di + c0) = *reinterpret_cast<const uint2*>(hi);
      *reinterpret_cast<uint2*>(uc + row * 2 * Di + Di + c0) = *reinterpret_cast<const uint2*>(lo);
    }
  } else {
    if constexpr (VEC == 4) *reinterpret_cast<float4*>(uc + row * Di + c0) = make_float4(y[0], y[1], y[2], y[3]);
    else *reinterpret_cast<float2*>(uc + row * Di + c0) = make_float2(y[0], y[1]);
  }
}

template <typename T, int TT>
__global__ void __launch_bounds__(256) conv_silu_kernel(const ConvParams<T> p) {
  constexpr int VEC = 8 / sizeof(T);
  const int groups = p.Di / VEC;
  const int ttiles = (p.L + TT - 1) / TT;
  const long long total = static_cast<long long>(p.B) * ttiles * groups;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int g = static_cast<int>(idx % groups);
    const long long r = idx / groups;
    const int tt = static_cast<int>(r % ttiles);
    const int b = static_cast<int>(r / ttiles);
    const int c0 = g * VEC;
    const int t0 = tt * TT;
    const long long base = static_cast<long long>(b) * p.L;

    // rows[i] = the VEC inputs of token t0 - (K-1) + i
    uint2 rows[TT + kK - 1];
#pragma unroll
    for (int i = 0; i < TT + kK - 1; ++i) {
      const int t = t0 - (kK - 1) + i;
      rows[i] = make_uint2(0u, 0u);
      if (t >= 0 && t < p.L) rows[i] = *reinterpret_cast<const uint2*>(p.u + (base + t) * p.Di + c0);
    }
    if (t0 == 0 && !p.zero_init) {
      // left context from the conv state: entry K + t of each channel for t < 0
#pragma unroll
      for (int i = 0; i < kK - 1; ++i) {
        T* e = reinterpret_cast<T*>(&rows[i]);
#pragma unroll
        for (int v = 0; v < VEC; ++v)
          e[v] = p.conv_state[(static_cast<long long>(b) * p.Di + c0 + v) * kK + 1 + i];
      }
    }
    // taps in registers: the uc stores below could alias them as far as the
    // compiler knows, so loads inside the token loop would be repeated
    float w[VEC][kK], bias[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      bias[v] = to_f32(p.conv_b[c0 + v]);
#pragma unroll
      for (int k = 0; k < kK; ++k) w[v][k] = to_f32(p.conv_w[(c0 + v) * kK + k]);
    }
#pragma unroll
    for (int i = 0; i < TT; ++i) {
      const int t = t0 + i;
      if (t >= p.L) break;
      float y[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        float acc = bias[v];
#pragma unroll
        for (int k = 0; k < kK; ++k)
          acc = fmaf(w[v][k], to_f32(reinterpret_cast<const T*>(&rows[i + k])[v]), acc);
        y[v] = silu(acc);
      }
      store_uc<T, VEC>(p.uc, base + t, p.Di, c0, y);
    }
  }
}

// ------------------------------------ x_proj split-K reduction (+ split delta)
//
// xdbl = sum of the x_proj split-K partials, added in split order so the
// result does not depend on scheduling.  The delta columns are also written
// as the split bf16 A operand of the dt_proj GEMM: delta2 [rows, 2*Rp] with
// hi in columns [0, R), lo in [Rp, Rp + R) and zeros in the padding up to
// Rp (a multiple of 64).  One thread: 4 consecutive columns.

// LPG lanes per 4-column group: lane `sub` adds splits sub, sub + LPG, ... in
// order, then a fixed xor tree combines the lane sums, so the result is the
// same on every run.  Warps iterate uniformly (shuffles need all lanes).
// LPG = 8 for many splits (single-row-tile decode), 1 otherwise.
template <int LPG>
__global__ void xdbl_reduce_kernel(const float* __restrict__ partials, int splits,
                                   long long split_stride, float* __restrict__ xdbl,
                                   bf16* __restrict__ delta2, int rows, int R, int Rp, int ldx) {
  const long long total4 = static_cast<long long>(rows) * ldx / 4;
  const int lane = threadIdx.x & 31, sub = lane % LPG;
  const long long warps = static_cast<long long>(gridDim.x) * blockDim.x / 32;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long w = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) / 32;
       w * (32 / LPG) < total4; w += warps) {
    const long long i = w * (32 / LPG) + lane / LPG;
    const bool valid = i < total4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (valid) {
#pragma unroll 4
      for (int sp = sub; sp < splits; sp += LPG) {
        const float4 p = reinterpret_cast<const float4*>(partials + sp * split_stride)[i];
        acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
      }
    }
#pragma unroll
    for (int off = LPG / 2; off >= 1; off >>= 1) {  // no iterations for LPG = 1
      acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
      acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
      acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
      acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
    }
    if (!valid || sub != 0) continue;
    reinterpret_cast<float4*>(xdbl)[i] = acc;
    const long long e = i * 4;
    const long long row = e / ldx;
    const int col = static_cast<int>(e % ldx);
    if (col < R) {
      const float a[4] = {acc.x, acc.y, acc.z, acc.w};
      bf16 hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        hi[j] = __float2bfloat16_rn(a[j]);
        lo[j] = __float2bfloat16_rn(a[j] - __bfloat162float(hi[j]));
      }
      bf16* dh = delta2 + row * 2 * Rp + col;
      bf16* dl = dh + Rp;
      reinterpret_cast<__nv_bfloat162*>(dh)[0] = __halves2bfloat162(hi[0], hi[1]);
      reinterpret_cast<__nv_bfloat162*>(dh)[1] = __halves2bfloat162(hi[2], hi[3]);
      reinterpret_cast<__nv_bfloat162*>(dl)[0] = __halves2bfloat162(lo[0], lo[1]);
      reinterpret_cast<__nv_bfloat162*>(dl)[1] = __halves2bfloat162(lo[2], lo[3]);
    }
  }
  // zero padding columns [R, Rp) of both halves
  const int pad4 = (Rp - R) / 4;
  const long long totalp = static_cast<long long>(rows) * pad4 * 2;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < totalp;
       i += stride) {
    const long long row = i / (2 * pad4);
    const int r = static_cast<int>(i % (2 * pad4));
    const int half = r / pad4;
    const int col = R + (r % pad4) * 4;
    *reinterpret_cast<uint2*>(delta2 + row * 2 * Rp + half * Rp + col) = make_uint2(0u, 0u);
  }
}

// ------------------------------------------------------- selective scan (prefill)
//
// CTA = CH channels of one sequence, 128 threads: thread (channel cl, lane q
// of LANES = 16 / SPT) owns states q*SPT .. q*SPT + SPT-1 of channel cl, in
// registers, for the whole sequence.  Tokens stream through shared memory in
// chunks of TC, double buffered with cp.async; each lane's B and C values of
// a token land side by side so one vector load fetches them.  Per chunk:
//   prepass  (dt, dt*uc) and D*uc per (token, channel), once instead of once
//     per lane;
//   groups of 8 tokens: phase 1 issues every exp(dt A) and dt*uc*B of the
//     group (independent of the state, so they overlap on the SFU), phase 2
//     runs the dependent recurrence and this lane's share of each readout;
//     a LANES-lane butterfly reduce-scatter then leaves lane q with the full
//     readout of token (group base + q), which adds D*uc;
//   the chunk's M rows leave with coalesced 16-byte stores.
// Every shared-memory access is one wavefront of an SM-wide pipe, against
// SPT exps per lane on the per-sub-partition SFU: SPT = 4 keeps the shared
// memory pipe below the SFU.

template <typename T>
struct ScanParams {
  const T* uc;          // [B*L, Di] (f32) or split pair [B*L, 2*Di] (bf16)
  const float* dt;      // [B*L, Di]
  const float* xdbl;    // [B*L, ldx]: B at column R, C at column R + N
  const float* A;       // [Di, N]
  const float* D;       // [Di]
  const T* u;           // [B, L, Di] raw scan input (for the new conv state)
  float* h;             // [B, Di, N] in/out
  T* conv_state;        // [B, Di, K] in/out
  T* M;                 // [B, L, Di] out
  int B, L, Di, R, ldx;
  int zero_init;
};

constexpr int kScanThreads = 128;
constexpr int kScanTC = 32;     // tokens per chunk
constexpr int kScanPG = 8;      // tokens per pipeline group

// number of uc parts per element: the bf16 split pair (hi, lo) or one f32
template <typename T>
__host__ __device__ constexpr int uc_parts() { return sizeof(T) == 2 ? 2 : 1; }

template <typename T>
__device__ __forceinline__ long long uc_ld(int Di) { return static_cast<long long>(Di) * uc_parts<T>(); }

template <typename T, int SPT>
struct ScanSmem {
  static constexpr int LANES = kN / SPT;
  static constexpr int CH = kScanThreads / LANES;
  float dt[2][kScanTC][CH];
  T uc[2][uc_parts<T>()][kScanTC][CH];
  float bcq[2][kScanTC][LANES][2 * SPT];   // lane q: B[q*SPT ..], then C[q*SPT ..]
  float2 dtdu[kScanTC][CH];                // (dt, dt * uc) of the current chunk
  // rows padded: in the readout the lanes of a channel touch different tokens,
  // and unpadded 128-byte rows would put them all on one bank
  float dx[kScanTC][CH + 8];               // D * uc of the current chunk
  T out[kScanTC][CH + 16 / sizeof(T)];
};

template <typename T, int SPT>
__device__ __forceinline__ float uc_value(const ScanSmem<T, SPT>& s, int buf, int t, int cl) {
  if constexpr (sizeof(T) == 2) return to_f32(s.uc[buf][0][t][cl]) + to_f32(s.uc[buf][1][t][cl]);
  else return s.uc[buf][0][t][cl];
}

__device__ __forceinline__ void cp_async8(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(gmem_src) : "memory");
}

template <typename T, int SPT>
__device__ __forceinline__ void scan_load_chunk(const ScanParams<T>& p, ScanSmem<T, SPT>& s, int buf,
                                                int b, int c0, int t0, int nt) {
  constexpr int CH = ScanSmem<T, SPT>::CH;
  constexpr int LANES = ScanSmem<T, SPT>::LANES;
  const int tid = threadIdx.x;
  const long long row0 = static_cast<long long>(b) * p.L + t0;
  constexpr int DTP = CH * 4 / 16;           // 16-byte pieces of a dt row
  for (int i = tid; i < kScanTC * DTP; i += kScanThreads) {
    const int t = i / DTP, piece = i % DTP;
    float* d = &s.dt[buf][t][piece * 4];
    if (t < nt) cp_async16(d, p.dt + (row0 + t) * p.Di + c0 + piece * 4);
    else *reinterpret_cast<float4*>(d) = make_float4(0.f, 0.f, 0.f, 0.f);  // dt = 0: h unchanged
  }
  // B and C of each lane's SPT states: two SPT-float pieces per (token, lane)
  for (int i = tid; i < kScanTC * LANES * 2; i += kScanThreads) {
    const int t = i / (LANES * 2), r = i % (LANES * 2);
    const int q = r >> 1, which = r & 1;     // which: 0 = B, 1 = C
    float* d = &s.bcq[buf][t][q][which * SPT];
    const float* src = p.xdbl + (row0 + t) * p.ldx + p.R + which * kN + q * SPT;
    if (t < nt) {
      if constexpr (SPT == 4) cp_async16(d, src);
      else cp_async8(d, src);
    } else {
#pragma unroll
      for (int j = 0; j < SPT; ++j) d[j] = 0.0f;
    }
  }
  constexpr int UP = CH * sizeof(T) / 16;    // 16-byte pieces of a uc row part
  constexpr int NP = uc_parts<T>();
  for (int i = tid; i < kScanTC * UP * NP; i += kScanThreads) {
    const int part = i / (kScanTC * UP);
    const int r = i % (kScanTC * UP);
    const int t = r / UP, piece = r % UP;
    T* d = &s.uc[buf][part][t][piece * (16 / sizeof(T))];
    if (t < nt)
      cp_async16(d, p.uc + (row0 + t) * uc_ld<T>(p.Di) + part * p.Di + c0 + piece * (16 / sizeof(T)));
    else
      *reinterpret_cast<uint4*>(d) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Butterfly reduce-scatter over the LANES lanes of a channel: on entry v[i]
// is this lane's partial for token i of the group; on return v[0] is the sum
// over all lanes for token q (this lane's index among the LANES).
template <int LANES>
__device__ __forceinline__ float reduce_scatter(float (&v)[LANES], int q) {
#pragma unroll
  for (int off = LANES / 2; off >= 1; off >>= 1) {
    const bool upper = (q & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

template <typename T, int SPT>
__global__ void __launch_bounds__(kScanThreads) selective_scan_kernel(const ScanParams<T> p) {
  using Smem = ScanSmem<T, SPT>;
  constexpr int LANES = Smem::LANES;
  constexpr int CH = Smem::CH;
  extern __shared__ __align__(16) uint8_t scan_smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(scan_smem_raw);
  const int cl = threadIdx.x / LANES;
  const int q = threadIdx.x % LANES;
  const int c0 = blockIdx.x * CH;
  const int c = c0 + cl;
  const int b = blockIdx.y;

  float a2[SPT], h[SPT];
#pragma unroll
  for (int j = 0; j < SPT; ++j) {
    a2[j] = p.A[c * kN + q * SPT + j] * kLog2e;
    h[j] = p.zero_init ? 0.0f : p.h[(static_cast<long long>(b) * p.Di + c) * kN + q * SPT + j];
  }
  const int nchunks = (p.L + kScanTC - 1) / kScanTC;

  scan_load_chunk<T, SPT>(p, s, 0, b, c0, 0, min(kScanTC, p.L));
  cp_async_commit();

  for (int ck = 0; ck < nchunks; ++ck) {
    const int buf = ck & 1;
    const int t0 = ck * kScanTC;
    const int nt = min(kScanTC, p.L - t0);
    if (ck + 1 < nchunks) {
      const int t1 = t0 + kScanTC;
      scan_load_chunk<T, SPT>(p, s, buf ^ 1, b, c0, t1, min(kScanTC, p.L - t1));
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    // prepass: (dt, dt * uc) and D * uc per (token, channel); the thread's
    // channel is the same on every iteration (kScanThreads % CH == 0)
    {
      const int cc = threadIdx.x % CH;
      const float Dcc = p.D[c0 + cc];
      for (int t = threadIdx.x / CH; t < kScanTC; t += kScanThreads / CH) {
        const float d = s.dt[buf][t][cc];
        const float uu = uc_value<T, SPT>(s, buf, t, cc);
        s.dtdu[t][cc] = make_float2(d, d * uu);
        s.dx[t][cc] = Dcc * uu;
      }
    }
    __syncthreads();

#pragma unroll
    for (int tg = 0; tg < kScanTC; tg += kScanPG) {
      // phase 1: decays and inputs of the group's tokens
      float da[kScanPG][SPT], bu[kScanPG][SPT], cv[kScanPG][SPT];
#pragma unroll
      for (int i = 0; i < kScanPG; ++i) {
        const int t = tg + i;
        const float2 dd = s.dtdu[t][cl];
        float bc[2 * SPT];
#pragma unroll
        for (int j = 0; j < 2 * SPT; j += 4)
          *reinterpret_cast<float4*>(&bc[j]) = *reinterpret_cast<const float4*>(&s.bcq[buf][t][q][j]);
#pragma unroll
        for (int j = 0; j < SPT; ++j) {
          da[i][j] = ex2_approx(dd.x * a2[j]);
          bu[i][j] = dd.y * bc[j];
          cv[i][j] = bc[SPT + j];
        }
      }
      // phase 2: the recurrence and this lane's share of each readout
      float part[kScanPG];
#pragma unroll
      for (int i = 0; i < kScanPG; ++i) {
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < SPT; ++j) {
          h[j] = fmaf(da[i][j], h[j], bu[i][j]);
          acc = fmaf(cv[i][j], h[j], acc);
        }
        part[i] = acc;
      }
      // readout: reduce-scatter over the channel's lanes, LANES tokens at a time
#pragma unroll
      for (int r0 = 0; r0 < kScanPG; r0 += LANES) {
        float v[LANES];
#pragma unroll
        for (int i = 0; i < LANES; ++i) v[i] = part[r0 + i];
        const float y = reduce_scatter<LANES>(v, q);
        const int t = tg + r0 + q;
        s.out[t][cl] = from_f32<T>(y + s.dx[t][cl]);
      }
    }
    __syncthreads();
    // coalesced write-out of the chunk's readout rows
    {
      constexpr int PIECES = CH * sizeof(T) / 16;
      const long long row0 = static_cast<long long>(b) * p.L + t0;
      for (int i = threadIdx.x; i < nt * PIECES; i += kScanThreads) {
        const int t = i / PIECES, piece = i % PIECES;
        *reinterpret_cast<uint4*>(p.M + (row0 + t) * p.Di + c0 + piece * (16 / sizeof(T))) =
            *reinterpret_cast<const uint4*>(&s.out[t][piece * (16 / sizeof(T))]);
      }
    }
    // the next chunk's prefetch overwrites buf only after its first barrier,
    // which every thread reaches after finishing this write-out
  }

#pragma unroll
  for (int j = 0; j < SPT; ++j) p.h[(static_cast<long long>(b) * p.Di + c) * kN + q * SPT + j] = h[j];
  // new conv state: the last K raw inputs (older ones from the previous state
  // when the prompt is shorter than K)
  if (q == 0) {
    T* cs = p.conv_state + (static_cast<long long>(b) * p.Di + c) * kK;
    T nw[kK];
#pragma unroll
    for (int k = 0; k < kK; ++k) {
      const int t = p.L - kK + k;
      if (t >= 0) nw[k] = p.u[(static_cast<long long>(b) * p.L + t) * p.Di + c];
      else if (!p.zero_init) nw[k] = cs[kK + t];  // token t < 0 of the previous state
      else nw[k] = from_f32<T>(0.0f);
    }
#pragma unroll
    for (int k = 0; k < kK; ++k) cs[k] = nw[k];
  }
}

// ------------------------------------------------------------ decode step

// conv window shift + conv + SiLU for one token of every sequence, in place
// on the conv state.  Thread: VEC channels of one sequence; the channels'
// K-entry windows (and taps) are contiguous, so they move as 16-byte vectors.
template <typename T>
__global__ void __launch_bounds__(256) step_conv_kernel(const T* __restrict__ u_t,
                                                        T* __restrict__ conv_state,
                                                        const T* __restrict__ conv_w,
                                                        const T* __restrict__ conv_b,
                                                        T* __restrict__ uc, int B, int Di) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int WV = VEC * kK * sizeof(T) / 16;   // 16-byte vectors per VEC windows
  const int groups = Di / VEC;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * groups) return;
  const int b = idx / groups;
  const int c0 = (idx % groups) * VEC;
  const long long off = static_cast<long long>(b) * Di + c0;
  Pack16 in, bias_v, st[WV], wt[WV];
  in.u = *reinterpret_cast<const uint4*>(u_t + off);
  bias_v.u = *reinterpret_cast<const uint4*>(conv_b + c0);
  uint4* sp = reinterpret_cast<uint4*>(conv_state + off * kK);
  const uint4* wp = reinterpret_cast<const uint4*>(conv_w + static_cast<long long>(c0) * kK);
#pragma unroll
  for (int i = 0; i < WV; ++i) {
    st[i].u = sp[i];
    wt[i].u = wp[i];
  }
  T* sw = reinterpret_cast<T*>(st);              // [VEC][K], oldest first
  const T* ww = reinterpret_cast<const T*>(wt);  // [VEC][K]
  float y[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) {
    T x;
    float b0;
    if constexpr (sizeof(T) == 2) { x = in.h[v]; b0 = __bfloat162float(bias_v.h[v]); }
    else { x = in.f[v]; b0 = bias_v.f[v]; }
#pragma unroll
    for (int k = 0; k < kK - 1; ++k) sw[v * kK + k] = sw[v * kK + k + 1];
    sw[v * kK + kK - 1] = x;
    float acc = b0;
#pragma unroll
    for (int k = 0; k < kK; ++k) acc = fmaf(to_f32(ww[v * kK + k]), to_f32(sw[v * kK + k]), acc);
    y[v] = silu(acc);
  }
#pragma unroll
  for (int i = 0; i < WV; ++i) sp[i] = st[i].u;
  store_uc<T, VEC>(uc, b, Di, c0, y);
}

// state update + readout for one token: thread (b, c, q) owns states
// 4q..4q+3 of channel c of sequence b, updated in place.
template <typename T>
__global__ void __launch_bounds__(256) step_scan_kernel(const T* __restrict__ uc,
                                                        const float* __restrict__ dt,
                                                        const float* __restrict__ xdbl,
                                                        const float* __restrict__ A,
                                                        const float* __restrict__ D,
                                                        float* __restrict__ h, T* __restrict__ m_t,
                                                        int B, int Di, int R, int ldx) {
  const long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  const long long pair = idx >> 2;      // (b, c)
  const int q = static_cast<int>(idx & 3);
  const bool live = pair < static_cast<long long>(B) * Di;
  const long long pc = live ? pair : 0;
  const int b = static_cast<int>(pc / Di);
  const int c = static_cast<int>(pc % Di);
  const float d = dt[pc];
  float u;
  if constexpr (sizeof(T) == 2) u = to_f32(uc[b * 2LL * Di + c]) + to_f32(uc[b * 2LL * Di + Di + c]);
  else u = uc[pc];
  const float du = d * u;
  const float4 av = *reinterpret_cast<const float4*>(A + c * kN + 4 * q);
  const float4 bv = *reinterpret_cast<const float4*>(xdbl + static_cast<long long>(b) * ldx + R + 4 * q);
  const float4 cv = *reinterpret_cast<const float4*>(xdbl + static_cast<long long>(b) * ldx + R + kN + 4 * q);
  float* hp = h + pc * kN + 4 * q;
  float4 hv = *reinterpret_cast<const float4*>(hp);
  hv.x = fmaf(ex2_approx(d * av.x * kLog2e), hv.x, du * bv.x);
  hv.y = fmaf(ex2_approx(d * av.y * kLog2e), hv.y, du * bv.y);
  hv.z = fmaf(ex2_approx(d * av.z * kLog2e), hv.z, du * bv.z);
  hv.w = fmaf(ex2_approx(d * av.w * kLog2e), hv.w, du * bv.w);
  float y = cv.x * hv.x;
  y = fmaf(cv.y, hv.y, y);
  y = fmaf(cv.z, hv.z, y);
  y = fmaf(cv.w, hv.w, y);
  y += __shfl_xor_sync(0xffffffffu, y, 1);
  y += __shfl_xor_sync(0xffffffffu, y, 2);
  if (live) {
    *reinterpret_cast<float4*>(hp) = hv;
    if (q == 0) m_t[pc] = from_f32<T>(fmaf(D[c], u, y));
  }
}

}  // namespace scan
}  // namespace sambay
