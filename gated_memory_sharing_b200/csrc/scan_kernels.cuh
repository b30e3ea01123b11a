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
  if constexpr (sizeof(T) == 2) {
    Pack16 hi, lo;
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      hi.h[v] = __float2bfloat16_rn(y[v]);
      lo.h[v] = __float2bfloat16_rn(y[v] - __bfloat162float(hi.h[v]));
    }
    *reinterpret_cast<uint4*>(uc + row * 2 * Di + c0) = hi.u;
    *reinterpret_cast<uint4*>(uc + row * 2 * Di + Di + c0) = lo.u;
  } else {
    Pack16 o;
#pragma unroll
    for (int v = 0; v < VEC; ++v) o.f[v] = y[v];
    *reinterpret_cast<uint4*>(uc + row * Di + c0) = o.u;
  }
}

template <typename T, int TT>
__global__ void __launch_bounds__(256) conv_silu_kernel(const ConvParams<T> p) {
  constexpr int VEC = 16 / sizeof(T);
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

    float w[VEC][kK], bias[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      bias[v] = to_f32(p.conv_b[c0 + v]);
#pragma unroll
      for (int k = 0; k < kK; ++k) w[v][k] = to_f32(p.conv_w[(c0 + v) * kK + k]);
    }
    // window[k] holds token t - (K-1) + k
    float win[kK][VEC];
#pragma unroll
    for (int k = 0; k < kK - 1; ++k) {
      const int t = t0 - (kK - 1) + k;
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        float x = 0.0f;
        if (t >= 0) {
          x = to_f32(p.u[(static_cast<long long>(b) * p.L + t) * p.Di + c0 + v]);
        } else if (!p.zero_init) {
          x = to_f32(p.conv_state[(static_cast<long long>(b) * p.Di + c0 + v) * kK + (kK + t)]);
        }
        win[k + 1][v] = x;  // shifted into place below
      }
    }
    const int t_end = min(p.L, t0 + TT);
    for (int t = t0; t < t_end; ++t) {
      const long long off = (static_cast<long long>(b) * p.L + t) * p.Di + c0;
      Pack16 in;
      in.u = *reinterpret_cast<const uint4*>(p.u + off);
#pragma unroll
      for (int k = 0; k < kK - 1; ++k)
#pragma unroll
        for (int v = 0; v < VEC; ++v) win[k][v] = win[k + 1][v];
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        if constexpr (sizeof(T) == 2) win[kK - 1][v] = __bfloat162float(in.h[v]);
        else win[kK - 1][v] = in.f[v];
      }
      float y[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        float acc = bias[v];
#pragma unroll
        for (int k = 0; k < kK; ++k) acc = fmaf(w[v][k], win[k][v], acc);
        y[v] = silu(acc);
      }
      store_uc<T, VEC>(p.uc, static_cast<long long>(b) * p.L + t, p.Di, c0, y);
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

__global__ void xdbl_reduce_kernel(const float* __restrict__ partials, int splits,
                                   long long split_stride, float* __restrict__ xdbl,
                                   bf16* __restrict__ delta2, int rows, int R, int Rp, int ldx) {
  const long long total4 = static_cast<long long>(rows) * ldx / 4;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total4;
       i += stride) {
    float4 acc = reinterpret_cast<const float4*>(partials)[i];
    for (int sp = 1; sp < splits; ++sp) {
      const float4 p = reinterpret_cast<const float4*>(partials + sp * split_stride)[i];
      acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
    }
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
// CTA = 32 channels of one sequence, 128 threads: thread (channel cl, quarter
// q) owns states 4q..4q+3 of channel cl, in registers, for the whole
// sequence.  Tokens stream through shared memory in chunks of TC, double
// buffered with cp.async.  Each token's readout sum over the 16 states is a
// 4-lane reduce-scatter done every 4 tokens, so lane q ends up holding the
// output of token 4j + q.

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

constexpr int kScanCh = 32;     // channels per CTA
constexpr int kScanTC = 32;     // tokens per chunk

// number of uc parts per element: the bf16 split pair (hi, lo) or one f32
template <typename T>
__host__ __device__ constexpr int uc_parts() { return sizeof(T) == 2 ? 2 : 1; }

template <typename T>
__device__ __forceinline__ long long uc_ld(int Di) { return static_cast<long long>(Di) * uc_parts<T>(); }

template <typename T>
struct ScanSmem {
  float dt[2][kScanTC][kScanCh];
  float bc[2][kScanTC][2 * kN];
  T uc[2][uc_parts<T>()][kScanTC][kScanCh];
  T out[kScanTC][kScanCh];
};

template <typename T>
__device__ __forceinline__ float uc_value(const ScanSmem<T>& s, int buf, int t, int cl) {
  if constexpr (sizeof(T) == 2) return to_f32(s.uc[buf][0][t][cl]) + to_f32(s.uc[buf][1][t][cl]);
  else return s.uc[buf][0][t][cl];
}

template <typename T>
__device__ __forceinline__ void scan_load_chunk(const ScanParams<T>& p, ScanSmem<T>& s, int buf,
                                                int b, int c0, int t0, int nt) {
  const int tid = threadIdx.x;
  const long long row0 = static_cast<long long>(b) * p.L + t0;
  // dt and B|C: rows of 32 floats = 8 x 16 bytes; 256 pieces each
  for (int i = tid; i < kScanTC * 8; i += blockDim.x) {
    const int t = i >> 3, piece = i & 7;
    float* d_dt = &s.dt[buf][t][piece * 4];
    float* d_bc = &s.bc[buf][t][piece * 4];
    if (t < nt) {
      cp_async16(d_dt, p.dt + (row0 + t) * p.Di + c0 + piece * 4);
      cp_async16(d_bc, p.xdbl + (row0 + t) * p.ldx + p.R + piece * 4);
    } else {  // ragged tail: dt = 0 leaves h unchanged
      *reinterpret_cast<float4*>(d_dt) = make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(d_bc) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  constexpr int PIECES = kScanCh * sizeof(T) / 16;  // per token row and part
  constexpr int NP = uc_parts<T>();
  for (int i = tid; i < kScanTC * PIECES * NP; i += blockDim.x) {
    const int part = i / (kScanTC * PIECES);
    const int r = i % (kScanTC * PIECES);
    const int t = r / PIECES, piece = r % PIECES;
    T* d_u = &s.uc[buf][part][t][piece * (16 / sizeof(T))];
    if (t < nt)
      cp_async16(d_u, p.uc + (row0 + t) * uc_ld<T>(p.Di) + part * p.Di + c0 + piece * (16 / sizeof(T)));
    else
      *reinterpret_cast<uint4*>(d_u) = make_uint4(0u, 0u, 0u, 0u);
  }
}

template <typename T>
__global__ void __launch_bounds__(128) selective_scan_kernel(const ScanParams<T> p) {
  __shared__ __align__(16) ScanSmem<T> s;
  const int cl = threadIdx.x >> 2;
  const int q = threadIdx.x & 3;
  const int c0 = blockIdx.x * kScanCh;
  const int c = c0 + cl;
  const int b = blockIdx.y;

  float a2[4], h[4];
  {
    const float4 av = *reinterpret_cast<const float4*>(p.A + c * kN + 4 * q);
    a2[0] = av.x * kLog2e; a2[1] = av.y * kLog2e; a2[2] = av.z * kLog2e; a2[3] = av.w * kLog2e;
    float* hp = p.h + (static_cast<long long>(b) * p.Di + c) * kN + 4 * q;
    if (p.zero_init) {
      h[0] = h[1] = h[2] = h[3] = 0.0f;
    } else {
      const float4 hv = *reinterpret_cast<const float4*>(hp);
      h[0] = hv.x; h[1] = hv.y; h[2] = hv.z; h[3] = hv.w;
    }
  }
  const float Dc = p.D[c];
  const int nchunks = (p.L + kScanTC - 1) / kScanTC;

  scan_load_chunk(p, s, 0, b, c0, 0, min(kScanTC, p.L));
  cp_async_commit();

  for (int ck = 0; ck < nchunks; ++ck) {
    const int buf = ck & 1;
    const int t0 = ck * kScanTC;
    const int nt = min(kScanTC, p.L - t0);
    if (ck + 1 < nchunks) {
      const int t1 = t0 + kScanTC;
      scan_load_chunk(p, s, buf ^ 1, b, c0, t1, min(kScanTC, p.L - t1));
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

#pragma unroll 1
    for (int tq = 0; tq < kScanTC; tq += 4) {
      float part[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int t = tq + j;
        const float d = s.dt[buf][t][cl];
        const float du = d * uc_value(s, buf, t, cl);
        const float4 bv = *reinterpret_cast<const float4*>(&s.bc[buf][t][4 * q]);
        const float4 cv = *reinterpret_cast<const float4*>(&s.bc[buf][t][kN + 4 * q]);
        const float da0 = ex2_approx(d * a2[0]);
        const float da1 = ex2_approx(d * a2[1]);
        const float da2 = ex2_approx(d * a2[2]);
        const float da3 = ex2_approx(d * a2[3]);
        h[0] = fmaf(da0, h[0], du * bv.x);
        h[1] = fmaf(da1, h[1], du * bv.y);
        h[2] = fmaf(da2, h[2], du * bv.z);
        h[3] = fmaf(da3, h[3], du * bv.w);
        part[j] = cv.x * h[0];
        part[j] = fmaf(cv.y, h[1], part[j]);
        part[j] = fmaf(cv.z, h[2], part[j]);
        part[j] = fmaf(cv.w, h[3], part[j]);
      }
      // 4-lane reduce-scatter: lane q collects the full sum of token tq + q
      const bool hi2 = (q & 2) != 0;
      float s0 = hi2 ? part[0] : part[2];
      float s1 = hi2 ? part[1] : part[3];
      float k0 = hi2 ? part[2] : part[0];
      float k1 = hi2 ? part[3] : part[1];
      k0 += __shfl_xor_sync(0xffffffffu, s0, 2);
      k1 += __shfl_xor_sync(0xffffffffu, s1, 2);
      const bool hi1 = (q & 1) != 0;
      const float snd = hi1 ? k0 : k1;
      float y = hi1 ? k1 : k0;
      y += __shfl_xor_sync(0xffffffffu, snd, 1);
      const int t = tq + q;
      y = fmaf(Dc, uc_value(s, buf, t, cl), y);
      s.out[t][cl] = from_f32<T>(y);
    }
    __syncthreads();
    // coalesced write-out of the chunk's readout rows
    {
      constexpr int PIECES = kScanCh * sizeof(T) / 16;
      const long long row0 = static_cast<long long>(b) * p.L + t0;
      for (int i = threadIdx.x; i < nt * PIECES; i += blockDim.x) {
        const int t = i / PIECES, piece = i % PIECES;
        *reinterpret_cast<uint4*>(p.M + (row0 + t) * p.Di + c0 + piece * (16 / sizeof(T))) =
            *reinterpret_cast<const uint4*>(&s.out[t][piece * (16 / sizeof(T))]);
      }
    }
    // the next iteration's prefetch overwrites buf; s.out is rewritten only
    // after that iteration's first __syncthreads
  }

  {
    float* hp = p.h + (static_cast<long long>(b) * p.Di + c) * kN + 4 * q;
    *reinterpret_cast<float4*>(hp) = make_float4(h[0], h[1], h[2], h[3]);
  }
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
// on the conv state.  Thread: VEC channels of one sequence.
template <typename T>
__global__ void __launch_bounds__(256) step_conv_kernel(const T* __restrict__ u_t,
                                                        T* __restrict__ conv_state,
                                                        const T* __restrict__ conv_w,
                                                        const T* __restrict__ conv_b,
                                                        T* __restrict__ uc, int B, int Di) {
  constexpr int VEC = 16 / sizeof(T);
  const int groups = Di / VEC;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * groups) return;
  const int b = idx / groups;
  const int c0 = (idx % groups) * VEC;
  const long long off = static_cast<long long>(b) * Di + c0;
  Pack16 in;
  in.u = *reinterpret_cast<const uint4*>(u_t + off);
  float y[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) {
    T* cs = conv_state + (off + v) * kK;
    float win[kK];
#pragma unroll
    for (int k = 0; k < kK - 1; ++k) win[k] = to_f32(cs[k + 1]);
    T x;
    if constexpr (sizeof(T) == 2) x = in.h[v];
    else x = in.f[v];
    win[kK - 1] = to_f32(x);
#pragma unroll
    for (int k = 0; k < kK - 1; ++k) cs[k] = cs[k + 1];
    cs[kK - 1] = x;
    float acc = to_f32(conv_b[c0 + v]);
#pragma unroll
    for (int k = 0; k < kK; ++k) acc = fmaf(to_f32(conv_w[(c0 + v) * kK + k]), win[k], acc);
    y[v] = silu(acc);
  }
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
