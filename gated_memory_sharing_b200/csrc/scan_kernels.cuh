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

// B and C of each token pair, as the scan reads them: float index of B (which
// = 0) or C (which = 1) of state n at token t of sequence b, Lh = ceil(L / 2)
// pairs per sequence:
//   [b * Lh + t / 2][which][n / 2][(t, n even), (t+1, n even), (t, n odd), (t+1, n odd)]
__host__ __device__ inline long long bc_pair_index(int b, int t, int which, int n, int Lh) {
  return (static_cast<long long>(b) * Lh + (t >> 1)) * 64 + which * 32 + (n >> 1) * 4 + (n & 1) * 2 + (t & 1);
}


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
// CTA: CB (64 or 32) consecutive channels x kConvTT (64) consecutive tokens of
// one sequence.  The input rows t0-3 .. t0+63 of those channels land in shared
// memory with 16-byte copies (the 3-row halo comes from the previous tokens,
// the caller's conv state for a continuing prompt, or zeros for a fresh one),
// so each input is read from HBM about once.  Thread: 4 consecutive channels x
// 4 consecutive tokens, taps and bias in registers (few enough for four CTAs
// per SM, whose loads then overlap one another's arithmetic); the outputs
// leave as 8-byte stores (bf16: the split pair's hi row and lo row), 16
// threads per 64-channel row.

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

constexpr int kConvTT = 64;                   // tokens per CTA

// N (4 or 8) conv outputs of one token row: float32 as is; bf16 as the split
// pair (hi at column c, lo at column Di + c of a 2*Di row).
template <typename T, int N>
__device__ __forceinline__ void store_uc(T* uc, long long row, int Di, int c0, const float (&y)[N]) {
  static_assert(N == 4 || N == 8, "4 or 8 outputs");
  if constexpr (sizeof(T) == 2) {
    __nv_bfloat162 hi[N / 2], lo[N / 2];
#pragma unroll
    for (int v = 0; v < N; v += 2) {
      hi[v / 2] = __floats2bfloat162_rn(y[v], y[v + 1]);
      const float2 back = __bfloat1622float2(hi[v / 2]);
      lo[v / 2] = __floats2bfloat162_rn(y[v] - back.x, y[v + 1] - back.y);
    }
    if constexpr (N == 8) {
      *reinterpret_cast<uint4*>(uc + row * 2 * Di + c0) = *reinterpret_cast<const uint4*>(hi);
      *reinterpret_cast<uint4*>(uc + row * 2 * Di + Di + c0) = *reinterpret_cast<const uint4*>(lo);
    } else {
      *reinterpret_cast<uint2*>(uc + row * 2 * Di + c0) = *reinterpret_cast<const uint2*>(hi);
      *reinterpret_cast<uint2*>(uc + row * 2 * Di + Di + c0) = *reinterpret_cast<const uint2*>(lo);
    }
  } else {
#pragma unroll
    for (int v = 0; v < N; v += 4)
      *reinterpret_cast<float4*>(uc + row * Di + c0 + v) = make_float4(y[v], y[v + 1], y[v + 2], y[v + 3]);
  }
}

// 4 conv outputs at `dst` (a row of uc, column c): float32 as is; bf16 as
// the split pair, hi at dst and lo Di elements further
template <typename T>
__device__ __forceinline__ void store_uc_row(T* dst, int Di, const float (&y)[4]) {
  if constexpr (sizeof(T) == 2) {
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]), h1 = __floats2bfloat162_rn(y[2], y[3]);
    const float2 b0 = __bfloat1622float2(h0), b1 = __bfloat1622float2(h1);
    const __nv_bfloat162 l0 = __floats2bfloat162_rn(y[0] - b0.x, y[1] - b0.y);
    const __nv_bfloat162 l1 = __floats2bfloat162_rn(y[2] - b1.x, y[3] - b1.y);
    uint2 hi, lo;
    hi.x = *reinterpret_cast<const uint32_t*>(&h0);
    hi.y = *reinterpret_cast<const uint32_t*>(&h1);
    lo.x = *reinterpret_cast<const uint32_t*>(&l0);
    lo.y = *reinterpret_cast<const uint32_t*>(&l1);
    *reinterpret_cast<uint2*>(dst) = hi;
    *reinterpret_cast<uint2*>(dst + Di) = lo;
  } else {
    *reinterpret_cast<float4*>(dst) = make_float4(y[0], y[1], y[2], y[3]);
  }
}

// 4 consecutive values of T at p (8- or 16-byte aligned) as floats
template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&x)[4]) {
  if constexpr (sizeof(T) == 2) {
    const uint2 r = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  } else {
    const float4 r = *reinterpret_cast<const float4*>(p);
    x[0] = r.x; x[1] = r.y; x[2] = r.z; x[3] = r.w;
  }
}

template <typename T, int CB>
__global__ void __launch_bounds__(CB / 4 * (kConvTT / 4), 4) conv_silu_kernel(const ConvParams<T> p) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int ROWS = kConvTT + kK - 1;
  constexpr int EP = 16 / sizeof(T);          // elements per 16-byte piece
  constexpr int PPR = CB / EP;                // pieces per row
  constexpr int NT = CB / 4 * (kConvTT / 4);  // threads
  __shared__ __align__(16) T tile[ROWS][CB];
  const int c0 = blockIdx.x * CB;
  const int t0 = blockIdx.y * kConvTT;
  const int b = blockIdx.z;
  const long long base = static_cast<long long>(b) * p.L;

  for (int i = threadIdx.x; i < ROWS * PPR; i += NT) {
    const int r = i / PPR, piece = i % PPR;
    const int t = t0 - (kK - 1) + r;
    T* d = &tile[r][piece * EP];
    if (t >= 0 && t < p.L) {
      cp_async16(d, p.u + (base + t) * p.Di + c0 + piece * EP);
    } else if (t < 0 && !p.zero_init) {
      // left context: entry K + t of each channel's conv state
#pragma unroll
      for (int e = 0; e < EP; ++e)
        d[e] = p.conv_state[(static_cast<long long>(b) * p.Di + c0 + piece * EP + e) * kK + kK + t];
    } else {
      *reinterpret_cast<uint4*>(d) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  cp_async_commit();

  const int j = threadIdx.x % (CB / 4);       // channels c0 + 4j .. + 3
  const int tq = threadIdx.x / (CB / 4);      // tokens t0 + 4tq .. + 3
  const int cj = c0 + 4 * j;
  float w[4][kK], bias[4];
  {
    // 4 channels x K taps are 4K contiguous values
#pragma unroll
    for (int v = 0; v < 4; ++v) load4<T>(p.conv_w + static_cast<long long>(cj + v) * kK, w[v]);
    load4<T>(p.conv_b + cj, bias);
  }
  cp_async_wait<0>();
  __syncthreads();

  // output token t0 + 4tq + i reads tile rows 4tq + i .. 4tq + i + K - 1
  // (tile row r is token t0 - K + 1 + r): the thread's 4 + K - 1 rows are
  // read and converted once, and its output rows are one pointer step apart
  float x[4 + kK - 1][4];
#pragma unroll
  for (int r = 0; r < 4 + kK - 1; ++r) load4<T>(&tile[4 * tq + r][4 * j], x[r]);
  const long long ld = static_cast<long long>(p.Di) * (sizeof(T) == 2 ? 2 : 1);   // uc row: split pair or f32
  T* dst = p.uc + (base + t0 + 4 * tq) * ld + cj;
  const int nt = min(4, p.L - (t0 + 4 * tq));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (i >= nt) break;
    float y[4] = {bias[0], bias[1], bias[2], bias[3]};
#pragma unroll
    for (int k = 0; k < kK; ++k)
#pragma unroll
      for (int v = 0; v < 4; ++v) y[v] = fmaf(w[v][k], x[i + k][v], y[v]);
#pragma unroll
    for (int v = 0; v < 4; ++v) y[v] = silu(y[v]);
    store_uc_row<T>(dst + i * ld, p.Di, y);
  }
}

// ------------------------------------ x_proj split-K reduction (+ split delta)
//
// xdbl = sum of the x_proj split-K partials, added in split order so the
// result does not depend on scheduling.  The delta columns are also written
// as the split bf16 A operand of the dt_proj GEMM: delta2 [rows, 2*Rp] with
// hi in columns [0, R), lo in [Rp, Rp + R) and zeros in the padding up to
// Rp (a multiple of 64).  One thread: 4 consecutive columns.  delta2 and bcp
// may be null: xdbl only.

// LPG lanes per 4-column group: lane `sub` adds splits sub, sub + LPG, ... in
// order, then a fixed xor tree combines the lane sums, so the result is the
// same on every run.  Warps iterate uniformly (shuffles need all lanes).
// LPG = 8 for 16 or more splits (single-row-tile decode), 1 otherwise.
template <int LPG>
__global__ void xdbl_reduce_kernel(const float* __restrict__ partials, int splits,
                                   long long split_stride, float* __restrict__ xdbl,
                                   bf16* __restrict__ delta2, float* __restrict__ bcp, int L,
                                   int rows, int R, int Rp, int ldx) {
  pdl_wait();
  pdl_launch_dependents();
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
      // a batch of this lane's splits loaded together (with one lane per
      // group, all of them: fewer than 16 splits), then added in order
      constexpr int kBatch = LPG == 1 ? 16 : 4;
#pragma unroll 1
      for (int s0 = sub; s0 < splits; s0 += kBatch * LPG) {
        float4 p[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const int sp = s0 + j * LPG;
          p[j] = ldcg_or_zero(partials + (sp < splits ? sp * split_stride + 4 * i : 0), sp < splits);
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          acc.x += p[j].x; acc.y += p[j].y; acc.z += p[j].z; acc.w += p[j].w;
        }
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
      if (delta2 == nullptr) continue;   // xdbl only (a shard's partial sums)
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
    } else if (bcp != nullptr) {
      // B | C columns, also regrouped into token pairs for the prefill scan
      const float a[4] = {acc.x, acc.y, acc.z, acc.w};
      const int rr = static_cast<int>(row), b = rr / L, t = rr % L, Lh = (L + 1) >> 1;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = col + j - R;
        const long long k = bc_pair_index(b, t, cc / kN, cc % kN, Lh);
        bcp[k] = a[j];
        if ((L & 1) && t == L - 1) bcp[k + 1] = 0.0f;   // the missing second token of the last pair
      }
    }
  }
  // zero padding columns [R, Rp) of both halves
  if (delta2 == nullptr) return;
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

// B | C columns of xdbl regrouped into token pairs (bc_pair_index), for the
// float32 path whose x_proj writes xdbl directly.  Thread: one (row, column).
__global__ void bc_pairs_kernel(const float* __restrict__ xdbl, float* __restrict__ bcp, int L, int rows,
                                int R, int ldx) {
  pdl_wait();
  pdl_launch_dependents();
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i >= static_cast<long long>(rows) * 2 * kN) return;
  const int row = static_cast<int>(i / (2 * kN)), cc = static_cast<int>(i % (2 * kN));
  const int b = row / L, t = row % L, Lh = (L + 1) >> 1;
  const long long k = bc_pair_index(b, t, cc / kN, cc % kN, Lh);
  bcp[k] = xdbl[static_cast<long long>(row) * ldx + R + cc];
  if ((L & 1) && t == L - 1) bcp[k + 1] = 0.0f;
}

// ------------------------------------------------------- selective scan (prefill)
//
// Lane (channel c, quad q) of the 8 lanes of a channel owns states 2q, 2q+1
// of c in registers for the whole sequence.  Costs that set the design, per
// SM and clock on B200: 16 exp2 on the SFUs (one warp instruction holds an
// SFU pipe for 8 clocks whatever its active mask), one shared-memory
// wavefront (32 lanes x 32 bits: a 16-byte load per lane is 4 wavefronts),
// and several warp shuffles.  Per token the 8 lanes of a channel need B and C
// of their states (4 words each: shared memory), and dt, dt*uc of the channel
// (2 words all 8 lanes share: one lane loads them for 8 tokens at a time and
// shuffles hand them out), so shared memory stays below the SFUs.
//
// CTAs are sized per SM: a sequence's channels are cut into ScanParams::nblk
// runs of 4-channel quads (q_base or q_base + 1 each), so at batch 1 one CTA
// per SM holds 32 or 36 of the 5120 channels (8 or 9 warps).  Tokens stream
// through shared memory in chunks of kScanTC, three in flight (cp.async): dt
// and uc rows of the CTA's channels, and B, C as the x_proj reduction
// regrouped them (bc_pair_index): one 16-byte load returns (B_t, B_t+1) of
// states 2q and 2q+1, and likewise C.  Each thread's copies (one 4-element
// piece of a dt, uc and output row) are fixed for the whole sequence, so the
// chunk loop does no index arithmetic beyond a pointer step.  Token pairs run on the paired fp32 units (mul/fma .f32x2).
// The readout sum over the 16 states is an 8-lane butterfly reduce-scatter
// per 8 tokens, after which lane q holds token (base + q); it adds D*uc,
// which the same lane preloaded, and the chunk's rows leave from a staging
// tile.  One CTA barrier per chunk.

template <typename T>
struct ScanParams {
  const T* uc;          // [B*L, Di] (f32) or split pair [B*L, 2*Di] (bf16)
  const float* dt;      // [B*L, Di]
  const float* bcp;     // [B * Lh * 64]: B and C per token pair (bc_pair_index)
  const float* A;       // [Di, N]
  const float* D;       // [Di]
  const T* u;           // [B, L, Di] raw scan input (for the new conv state)
  float* h;             // [B, Di, N] in/out
  T* conv_state;        // [B, Di, K] in/out
  T* M;                 // [B, L, Di] out
  int B, L, Di;
  int zero_init;
  int nblk;             // CTAs per sequence (gridDim.x)
  int q_base, q_extra;  // CTA i covers q_base (+1 if i < q_extra) quads of 4 channels
  int chp;              // most channels of any CTA
};

constexpr int kScanTC = 32;     // tokens per chunk
constexpr int kScanStages = 3;  // chunks in flight
constexpr int kScanMaxCH = 36;  // channels per CTA at most (9 warps)
constexpr int kScanMaxThreads = 8 * kScanMaxCH;

// number of uc parts per element: the bf16 split pair (hi, lo) or one f32
template <typename T>
__host__ __device__ constexpr int uc_parts() { return sizeof(T) == 2 ? 2 : 1; }

template <typename T>
__device__ __forceinline__ long long uc_ld(int Di) { return static_cast<long long>(Di) * uc_parts<T>(); }

// Dynamic shared memory of one CTA.  Rows of the channel tiles are
// kScanPitch = 36 elements (at least the kScanMaxCH channels of any CTA, and
// 4 mod 32: a warp's 8-token x 4-channel preload then touches 32 distinct
// banks).  A compile-time pitch lets the chunk loop address its tiles with
// immediate offsets.
constexpr int kScanPitch = 36;
static_assert(kScanPitch >= kScanMaxCH && kScanPitch % 32 == 4, "scan tile pitch");

struct ScanLayout {
  int pitch, dt, uc, bc, out, bytes;
  __host__ __device__ ScanLayout(int chp, int tsize) {
    (void)chp;
    pitch = kScanPitch;
    const int parts = tsize == 2 ? 2 : 1;
    dt = 0;
    uc = dt + kScanStages * kScanTC * pitch * 4;
    bc = uc + kScanStages * parts * kScanTC * pitch * tsize;
    bc = (bc + 15) & ~15;
    out = bc + kScanStages * kScanTC * 2 * kN * 4;
    bytes = out + 2 * kScanTC * pitch * tsize;
  }
};

__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async8(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(gmem_src) : "memory");
}

// Paired fp32 arithmetic: two independent round-to-nearest operations.
__device__ __forceinline__ unsigned long long f2_pack(float2 a) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a.x), "f"(a.y));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(unsigned long long r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_pack(a)), "l"(f2_pack(b)));
  return f2_unpack(r);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_pack(a)), "l"(f2_pack(b)));
  return f2_unpack(r);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(f2_pack(a)), "l"(f2_pack(b)), "l"(f2_pack(c)));
  return f2_unpack(r);
}

// One thread's share of every chunk's copies: a 4-element piece (row td,
// columns 4 pd ..) of the dt row, of each uc part row and of the output row,
// and 16-byte pieces of the chunk's B/C pairs.
struct ScanPiece {
  bool live;          // tid < 8 * CH: this thread owns a row piece
  int soff;           // element offset of the piece within a stage's row tile
  long long goff;     // element offset of the piece's token-0 position, [B*L, Di] layout
  long long uoff;     // the same in the uc layout [B*L, parts * Di]
};

// Chunk loads.  Tokens past the end read as zeros: dt = 0 leaves h
// unchanged and adds nothing.
template <typename T>
__device__ __forceinline__ void scan_load_chunk(const ScanParams<T>& p, uint8_t* smem, const ScanLayout& ly,
                                                const ScanPiece& pc, int td, int st, int b, int t0) {
  const int pitch = ly.pitch;
  if (pc.live) {
    const bool in = t0 + td < p.L;
    const long long g = pc.goff + static_cast<long long>(t0) * p.Di;
    float* d = reinterpret_cast<float*>(smem + ly.dt) + st * kScanTC * pitch + pc.soff;
    if (in) cp_async16(d, p.dt + g);
    else *reinterpret_cast<float4*>(d) = make_float4(0.f, 0.f, 0.f, 0.f);
    constexpr int NP = uc_parts<T>();
    T* u = reinterpret_cast<T*>(smem + ly.uc) + st * NP * kScanTC * pitch + pc.soff;
    const long long gu = pc.uoff + static_cast<long long>(t0) * NP * p.Di;
#pragma unroll
    for (int part = 0; part < NP; ++part) {
      T* dp = u + part * kScanTC * pitch;
      const T* src = p.uc + gu + part * p.Di;
      if constexpr (sizeof(T) == 2) {
        if (in) cp_async8(dp, src);
        else *reinterpret_cast<uint2*>(dp) = make_uint2(0u, 0u);
      } else {
        if (in) cp_async16(dp, src);
        else *reinterpret_cast<float4*>(dp) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  // B/C: the chunk's kScanTC / 2 pairs are 64 floats each, contiguous
  const int Lh = (p.L + 1) >> 1;
  const int pr0 = t0 >> 1;
  float* s_bc = reinterpret_cast<float*>(smem + ly.bc) + st * kScanTC * 32;
  const float* g_bc = p.bcp + (static_cast<long long>(b) * Lh + pr0) * 64;
  for (int i = threadIdx.x; i < kScanTC * 8; i += blockDim.x) {
    float* d = s_bc + 4 * i;
    if (pr0 + (i >> 4) < Lh) cp_async16(d, g_bc + 4 * i);
    else *reinterpret_cast<float4*>(d) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Butterfly reduce-scatter over the 8 lanes of a channel (lanes 4q + c, q =
// 0..7): on entry v[i] is this lane's partial for token i of the group; on
// return the sum over the 8 lanes for token q.
__device__ __forceinline__ float reduce_scatter8(float (&v)[8], int q) {
#pragma unroll
  for (int off = 4; off >= 1; off >>= 1) {
    const bool upper = (q & off) != 0;
    float keep[4], got[4];
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      keep[i] = upper ? v[i + off] : v[i];
      got[i] = __shfl_xor_sync(0xffffffffu, send, off << 2);
    }
    if (off >= 2) {
#pragma unroll
      for (int i = 0; i < off; i += 2) {
        const float2 r = add2(make_float2(keep[i], keep[i + 1]), make_float2(got[i], got[i + 1]));
        v[i] = r.x;
        v[i + 1] = r.y;
      }
    } else {
      v[0] = keep[0] + got[0];
    }
  }
  return v[0];
}

// the chunk's readout rows from staging to M: this thread's 4-element piece
template <typename T>
__device__ __forceinline__ void scan_write_piece(const ScanParams<T>& p, const T* s_out, const ScanPiece& pc,
                                                 int td, int t0, int nt) {
  if (!pc.live || td >= nt) return;
  T* dst = p.M + pc.goff + static_cast<long long>(t0) * p.Di;
  if constexpr (sizeof(T) == 2) *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(s_out + pc.soff);
  else *reinterpret_cast<float4*>(dst) = *reinterpret_cast<const float4*>(s_out + pc.soff);
}

template <typename T>
__global__ void __launch_bounds__(kScanMaxThreads, 2) selective_scan_kernel(const ScanParams<T> p) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t scan_smem_raw[];
  uint8_t* smem = scan_smem_raw;
  const ScanLayout ly(p.chp, sizeof(T));
  constexpr int pitch = kScanPitch;
  const int blk = blockIdx.x, b = blockIdx.y;
  const int CH = 4 * (p.q_base + (blk < p.q_extra ? 1 : 0));
  const int c0 = 4 * (blk * p.q_base + min(blk, p.q_extra));
  // warp w: channels 4w .. 4w+3; lane 4q + c: states 2q, 2q+1 of channel 4w + c.
  // State-major lanes: a half-warp's B/C loads touch 4 distinct 16-byte words.
  const int lane = threadIdx.x & 31;
  const int cl = (threadIdx.x >> 5) * 4 + (lane & 3), q = lane >> 2;
  const bool active = cl < CH;
  // lanes past CH (a CTA narrower than chp) read their global parameters as
  // channel c0 and run on the tile columns [CH, chp), which no copy fills or
  // empties: their results stay in staging columns that never reach M
  const int col = cl;
  const int c = c0 + (active ? cl : 0);
  const float a2_0 = p.A[static_cast<long long>(c) * kN + 2 * q] * kLog2e;
  const float a2_1 = p.A[static_cast<long long>(c) * kN + 2 * q + 1] * kLog2e;
  float* hp = p.h + (static_cast<long long>(b) * p.Di + c) * kN + 2 * q;
  float h0 = p.zero_init ? 0.0f : hp[0];
  float h1 = p.zero_init ? 0.0f : hp[1];
  const float Dc = p.D[c];
  const float* s_dt = reinterpret_cast<const float*>(smem + ly.dt);
  const T* s_uc = reinterpret_cast<const T*>(smem + ly.uc);
  const float4* s_bc = reinterpret_cast<const float4*>(smem + ly.bc);
  T* s_out = reinterpret_cast<T*>(smem + ly.out);
  const int nchunks = (p.L + kScanTC - 1) / kScanTC;
  // this thread's row piece: row td, columns 4 pd .. 4 pd + 3 of the CTA's channels
  ScanPiece pc;
  const int quads = CH >> 2;
  pc.live = threadIdx.x < kScanTC * quads;
  const int td = pc.live ? threadIdx.x / quads : 0;
  const int pd = pc.live ? threadIdx.x % quads : 0;
  pc.soff = td * pitch + 4 * pd;
  pc.goff = (static_cast<long long>(b) * p.L + td) * p.Di + c0 + 4 * pd;
  pc.uoff = (static_cast<long long>(b) * p.L + td) * uc_parts<T>() * p.Di + c0 + 4 * pd;

  scan_load_chunk<T>(p, smem, ly, pc, td, 0, b, 0);
  cp_async_commit();
  if (nchunks > 1) scan_load_chunk<T>(p, smem, ly, pc, td, 1, b, kScanTC);
  cp_async_commit();

  for (int ck = 0; ck < nchunks; ++ck) {
    const int st = ck % kScanStages, ob = ck & 1;
    cp_async_wait<1>();          // chunk ck has landed (this thread's copies)
    __syncthreads();             // ... everyone's; chunk ck-1 fully consumed
    if (ck > 0) scan_write_piece<T>(p, s_out + (ob ^ 1) * kScanTC * pitch, pc, td, (ck - 1) * kScanTC, kScanTC);
    if (ck + 2 < nchunks) scan_load_chunk<T>(p, smem, ly, pc, td, (ck + 2) % kScanStages, b, (ck + 2) * kScanTC);
    cp_async_commit();

    const float* dtc = s_dt + st * kScanTC * pitch + col;
    const T* ucc = s_uc + st * uc_parts<T>() * kScanTC * pitch + col;
    const float4* bcc = s_bc + st * (kScanTC / 2) * 16 + q;
#pragma unroll
    for (int g = 0; g < kScanTC; g += 8) {
      // this lane's token g+q: dt, uc, dt*uc
      const int tq = g + q;
      const float dq = dtc[tq * pitch];
      float uq;
      if constexpr (sizeof(T) == 2) uq = to_f32(ucc[tq * pitch]) + to_f32(ucc[(kScanTC + tq) * pitch]);
      else uq = ucc[tq * pitch];
      const float duq = dq * uq;
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const int pr = (g + i) >> 1;                          // token pair (g+i, g+i+1)
        const int src = 4 * i + (lane & 3);                  // lane holding token g+i of this channel
        const float2 dtp = make_float2(__shfl_sync(0xffffffffu, dq, src), __shfl_sync(0xffffffffu, dq, src + 4));
        const float2 dup = make_float2(__shfl_sync(0xffffffffu, duq, src), __shfl_sync(0xffffffffu, duq, src + 4));
        const float4 bb = bcc[pr * 16];                        // B(t,2q) B(t+1,2q) B(t,2q+1) B(t+1,2q+1)
        const float4 cc = bcc[pr * 16 + 8];                    // the same for C
        const float2 x0 = mul2(dtp, make_float2(a2_0, a2_0));
        const float2 x1 = mul2(dtp, make_float2(a2_1, a2_1));
        const float2 bu0 = mul2(dup, make_float2(bb.x, bb.y));
        const float2 bu1 = mul2(dup, make_float2(bb.z, bb.w));
        const float h0a = fmaf(ex2_approx(x0.x), h0, bu0.x);
        h0 = fmaf(ex2_approx(x0.y), h0a, bu0.y);
        const float h1a = fmaf(ex2_approx(x1.x), h1, bu1.x);
        h1 = fmaf(ex2_approx(x1.y), h1a, bu1.y);
        const float2 pr2 = fma2(make_float2(cc.z, cc.w), make_float2(h1a, h1),
                                mul2(make_float2(cc.x, cc.y), make_float2(h0a, h0)));
        v[i] = pr2.x;
        v[i + 1] = pr2.y;
      }
      const float y = fmaf(Dc, uq, reduce_scatter8(v, q));
      s_out[(ob * kScanTC + tq) * pitch + col] = from_f32<T>(y);
    }
  }
  __syncthreads();
  {
    const int ck = nchunks - 1;
    scan_write_piece<T>(p, s_out + (ck & 1) * kScanTC * pitch, pc, td, ck * kScanTC, p.L - ck * kScanTC);
  }

  if (active) {
    hp[0] = h0;
    hp[1] = h1;
  }
  // new conv state: the last K raw inputs (older ones from the previous state
  // when the prompt is shorter than K)
  if (active && q == 0) {
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
  pdl_wait();
  pdl_launch_dependents();
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
  pdl_wait();
  pdl_launch_dependents();
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
