// Decode step of the selective scan (bfloat16 I/O): three short kernels per
// token of every sequence, chained with programmatic dependent launch.
//
// The decode step of the Mamba layer whose readout is the memory M reused by
// the Gated Memory Units ("Decoder-Hybrid-Decoder Architecture for Efficient
// Reasoning with Long Generation", Paper-Notes page, 方法详解 > 关键设计:
// decoding keeps a constant-size state; Gu & Dao 2023, "Mamba", section 3.2
// and Algorithm 2 with L = 1):
//
//   window <- [window[1:], u_t];  uc = SiLU(conv_b + sum_k conv_w[k] window[k])
//   [delta | B | C] = uc W_x^T;   dt = softplus(delta W_dt^T + b_dt)
//   h = exp(dt A) h + dt B uc;    m_t = C . h + D uc
//
// with the conv window and h updated in place.  Work is split by channel:
// CTA (slice, group) owns `chan` consecutive channels (Di / chan slices, about
// one per SM) of up to 64 sequences, so every weight element is read once per
// step.  x_proj sums over all channels, hence the three kernels:
//
//   step_proj     conv + SiLU of the slice (conv window updated in place; uc
//                 kept as fp32 for step_scan) and the slice's partial x_proj
//                 sums part[slice][j][seq]
//   step_reduce   [delta | B | C][seq][j] = sum over slices, in slice order
//                 (8 lanes per output, a fixed xor tree: run-to-run
//                 identical); delta leaves as the split pair that step_scan's
//                 MMA reads, B and C as fp32
//   step_scan     dt = softplus(delta W_dt^T + b_dt) for the slice, then the
//                 state update and readout.  Its h, W_dt, A, b_dt and D slices
//                 do not depend on the two kernels before it, so they are
//                 copied into shared memory BEFORE griddepcontrol.wait, while
//                 step_proj / step_reduce still run.
//
// The two projections are small contractions with N = 2 x sequences (the hi
// and lo halves of a split operand) and run as m16n8k16 bf16 MMAs with fp32
// accumulation.  The conv output and delta are split into bf16 pairs (x = hi +
// lo, hi = bf16(x), lo = bf16(x - hi)), which carries them to ~2^-17 relative
// into the tensor core; the weights are bf16 already, so no term is lost.
//
// K-permutation of the MMA operands: a lane of the m16n8k16 fragment layout
// holds the logical k = 2t, 2t+1 (first register) and 2t+8, 2t+9 (second)
// of its row; the dot product does not depend on the order of k, so logical
// (2t, 2t+1, 2t+8, 2t+9) is mapped to physical (4t, 4t+1, 4t+2, 4t+3) for
// both operands, which makes each pair of registers one 8-byte load.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace sambay {
namespace step {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxChan = 48;     // channels per slice (3 MMA k-steps / row tiles)
constexpr int kMaxGroup = 64;    // sequences per CTA (MMA N = 128: 16 n-blocks)
constexpr int kStateN = 16;      // d_state
constexpr int kConvK = 4;        // d_conv
constexpr int kRedLanes = 8;     // lanes per output in step_reduce
constexpr int kMaxPerLane = 19;  // slices per lane (148 slices at most)

struct StepParams {
  const bf16* u_t;        // [B, Di]
  bf16* conv_state;       // [B, Di, K] in/out
  const bf16* conv_w;     // [Di, K]
  const bf16* conv_b;     // [Di]
  const bf16* x_proj_w;   // [ldx, Di]
  const bf16* dt_proj_w;  // [Di, R]
  const float* dt_bias;   // [Di]
  const float* A;         // [Di, N]
  const float* D;         // [Di]
  float* h;               // [B, Di, N] in/out
  bf16* m_t;              // [B, Di] out
  // scratch (workspace)
  float* uc;              // [B, Di]            conv output
  float* part;            // [nslice][ldx][B]   x_proj partial sums
  bf16* dts;              // [2B][Rp]           delta split pair (row 2s: hi, 2s + 1: lo)
  float* bc;              // [B][2N]            B | C
  unsigned long long* bar;  // [1 + 2 * nslice]  step_fused: generation word, arrival flags
  unsigned long long wait_limit;  // step_fused: bounded-wait limit (clock64 cycles)
  int B, Di, R, Rp, ldx;
  int chan, nslice;       // channels per slice (multiple of 8, <= kMaxChan), slices
  int group;              // sequences per CTA (<= kMaxGroup)
};

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }
// a bf16 row pitch (elements) whose 32-bit word count is 8 (mod 16): the
// fragment loads of rows g = 0..7 (8 bytes at column 4t) then fall in distinct
// banks within each half-warp
__host__ __device__ constexpr int frag_pitch(int cols) {
  return round_up(cols, 16) + ((round_up(cols, 16) / 2) % 16 == 8 ? 0 : 16);
}

// step_proj's split conv output: [2 * kMaxGroup rows][frag_pitch(48)] bf16
constexpr int kUcsPitch = frag_pitch(kMaxChan);

// Dynamic shared memory of step_scan (byte offsets).
struct ScanStepLayout {
  int mtl, dp;           // dt_proj row tiles, W_dt row pitch (bf16 elements)
  int h, w, a, bias, dv, uc, bc, dt, bytes;
  __host__ __device__ ScanStepLayout(int chan, int group, int Rp) {
    mtl = (chan + 15) / 16;
    dp = frag_pitch(Rp);
    h = 0;                                             // f32 [group][chan][N]
    w = h + group * chan * kStateN * 4;                // bf16 [mtl*16][dp] W_dt rows
    a = w + round_up(mtl * 16 * dp * 2, 16);           // f32 [chan][N]
    bias = a + chan * kStateN * 4;                     // f32 [chan]
    dv = bias + round_up(chan * 4, 16);                // f32 [chan]
    uc = dv + round_up(chan * 4, 16);                  // f32 [group][chan]
    bc = uc + group * chan * 4;                        // f32 [group][2N]
    dt = bc + group * 2 * kStateN * 4;                 // f32 [group][chan]
    bytes = dt + group * chan * 4;
  }
};

// ------------------------------------------------------------------ PTX glue

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// D += A B for one m16n8k16 tile: bf16 operands, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint2 lds64(const bf16* p) { return *reinterpret_cast<const uint2*>(p); }

// hi = bf16(x), lo = bf16(x - hi)
__device__ __forceinline__ void split_bf16(float x, bf16& hi, bf16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// ------------------------------------------------------------------ step_proj

// grid (nslice, groups): conv + SiLU of the slice's channels for the group's
// sequences, then partial x_proj sums over those channels.
__global__ void __launch_bounds__(kThreads) step_proj_kernel(const StepParams p) {
  __shared__ __align__(16) bf16 ucs[2 * kMaxGroup * kUcsPitch];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int chan = p.chan, c0 = blockIdx.x * chan;
  const int s0 = blockIdx.y * p.group, ns = min(p.group, p.B - s0);
  const int nblk = (ns + 3) / 4;                 // MMA n-blocks: 4 sequences x (hi, lo) each
  const int kc = round_up(chan, 16);
  const int Di = p.Di, ldx = p.ldx;

  // conv: one item = 8 channels of one sequence; rows n = 2s (hi), 2s + 1 (lo)
  const int vpc = chan / 8;
  for (int it = tid; it < 4 * nblk * vpc; it += kThreads) {   // 4 sequences per n-block
    const int s = it / vpc, cl = (it % vpc) * 8;
    float y[8];
    if (s < ns) {
      const long long off = static_cast<long long>(s0 + s) * Di + c0 + cl;
      Pack16 in, bias, win[4], wt[4];
      in.u = *reinterpret_cast<const uint4*>(p.u_t + off);
      bias.u = *reinterpret_cast<const uint4*>(p.conv_b + c0 + cl);
      uint4* wp = reinterpret_cast<uint4*>(p.conv_state + off * kConvK);
      const uint4* kp = reinterpret_cast<const uint4*>(p.conv_w + static_cast<long long>(c0 + cl) * kConvK);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        win[j].u = wp[j];
        wt[j].u = kp[j];
      }
      bf16* wv = reinterpret_cast<bf16*>(win);            // [8 channels][K], oldest first
      const bf16* kv = reinterpret_cast<const bf16*>(wt);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
#pragma unroll
        for (int k = 0; k < kConvK - 1; ++k) wv[e * kConvK + k] = wv[e * kConvK + k + 1];
        wv[e * kConvK + kConvK - 1] = in.h[e];
        float acc = __bfloat162float(bias.h[e]);
#pragma unroll
        for (int k = 0; k < kConvK; ++k)
          acc = fmaf(__bfloat162float(kv[e * kConvK + k]), __bfloat162float(wv[e * kConvK + k]), acc);
        y[e] = silu(acc);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) wp[j] = win[j].u;
      float4* ug = reinterpret_cast<float4*>(p.uc + off);
      ug[0] = make_float4(y[0], y[1], y[2], y[3]);
      ug[1] = make_float4(y[4], y[5], y[6], y[7]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = 0.0f;
    }
    Pack16 hi, lo;
#pragma unroll
    for (int e = 0; e < 8; ++e) split_bf16(y[e], hi.h[e], lo.h[e]);
    *reinterpret_cast<uint4*>(ucs + (2 * s) * kUcsPitch + cl) = hi.u;
    *reinterpret_cast<uint4*>(ucs + (2 * s + 1) * kUcsPitch + cl) = lo.u;
  }
  // k-padding columns [chan, kc) of every row the MMAs read
  for (int it = tid; it < 8 * nblk * (kc - chan); it += kThreads) {
    const int r = it / (kc - chan), c = chan + it % (kc - chan);
    ucs[r * kUcsPitch + c] = __float2bfloat16_rn(0.0f);
  }
  __syncthreads();

  // partial x_proj: D[j][n] = sum_{c in slice} W_x[j][c] ucs[n][c]; warp takes
  // row tiles warp, warp + 8, ...; A fragments straight from W_x (L2)
  const int mtiles = (ldx + 15) / 16, ksteps = kc / 16;
  for (int mt = warp; mt < mtiles; mt += kWarps) {
    uint32_t a[3][4];
#pragma unroll
    for (int ks = 0; ks < 3; ++ks) {
      const int col = c0 + ks * 16 + 4 * t;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int j = mt * 16 + g + 8 * half;
        uint2 v = make_uint2(0u, 0u);
        if (ks < ksteps && j < ldx && col + 3 < Di)
          v = *reinterpret_cast<const uint2*>(p.x_proj_w + static_cast<long long>(j) * Di + col);
        a[ks][half] = v.x;          // logical k 2t, 2t+1
        a[ks][2 + half] = v.y;      // logical k 2t+8, 2t+9
      }
    }
    float acc[16][4];
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.0f;
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) {
      if (nb >= nblk) break;
#pragma unroll
      for (int ks = 0; ks < 3; ++ks) {
        if (ks >= ksteps) break;
        const uint2 b = lds64(ucs + (8 * nb + g) * kUcsPitch + ks * 16 + 4 * t);
        mma16816(acc[nb], a[ks][0], a[ks][1], a[ks][2], a[ks][3], b.x, b.y);
      }
    }
    // D[j][8nb + 2t + {0, 1}] = (hi, lo) of sequence 4nb + t
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) {
      if (nb >= nblk) break;
      const int s = 4 * nb + t;
      if (s >= ns) continue;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int j = mt * 16 + g + 8 * half;
        if (j < ldx)
          p.part[(static_cast<long long>(blockIdx.x) * ldx + j) * p.B + s0 + s] =
              acc[nb][2 * half] + acc[nb][2 * half + 1];
      }
    }
  }
}

// ------------------------------------------------------------------ step_reduce

// [delta | B | C] = sum of the slices' partials, in slice order.  8 lanes per
// output: lane `sub` adds slices sub, sub + 8, ... in order, then a fixed xor
// tree combines the lanes.  Warps iterate uniformly (shuffles need all lanes).
__global__ void __launch_bounds__(kThreads) step_reduce_kernel(const StepParams p) {
  pdl_launch_dependents();   // step_scan may start copying its independent inputs
  pdl_wait();
  const int lane = threadIdx.x & 31, sub = lane % kRedLanes;
  const long long total = static_cast<long long>(p.ldx) * p.B;
  const long long slice_stride = static_cast<long long>(p.ldx) * p.B;
  const long long warps = static_cast<long long>(gridDim.x) * kWarps;
  for (long long w = (blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x) / 32;
       w * (32 / kRedLanes) < total; w += warps) {
    const long long o = w * (32 / kRedLanes) + lane / kRedLanes;   // = j * B + s
    const bool valid = o < total;
    // every load of the lane in flight at once (nslice <= 8 * kMaxPerLane),
    // then the adds in slice order
    float x[kMaxPerLane];
#pragma unroll
    for (int k = 0; k < kMaxPerLane; ++k) {
      const int sl = sub + k * kRedLanes;
      x[k] = (valid && sl < p.nslice) ? __ldcg(p.part + sl * slice_stride + o) : 0.0f;
    }
    float acc = 0.0f;
#pragma unroll
    for (int k = 0; k < kMaxPerLane; ++k) acc += x[k];
#pragma unroll
    for (int off = kRedLanes / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (!valid || sub != 0) continue;
    const int j = static_cast<int>(o / p.B), s = static_cast<int>(o % p.B);
    if (j < p.R) {
      bf16 hi, lo;
      split_bf16(acc, hi, lo);
      p.dts[(2LL * s) * p.Rp + j] = hi;
      p.dts[(2LL * s + 1) * p.Rp + j] = lo;
    } else {
      p.bc[static_cast<long long>(s) * 2 * kStateN + (j - p.R)] = acc;
    }
  }
  // zero the k-padding columns [R, Rp) of the split pair
  const int pad = p.Rp - p.R;
  for (long long i = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x; i < 2LL * p.B * pad;
       i += static_cast<long long>(gridDim.x) * kThreads)
    p.dts[(i / pad) * p.Rp + p.R + i % pad] = __float2bfloat16_rn(0.0f);
}

// ------------------------------------------------------------------ step_scan

// grid (nslice, groups): dt for the slice's channels, then the state update
// and readout of the group's sequences.
__global__ void __launch_bounds__(kThreads, 1) step_scan_kernel(const StepParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int chan = p.chan, c0 = blockIdx.x * chan;
  const int s0 = blockIdx.y * p.group, ns = min(p.group, p.B - s0);
  const int Di = p.Di, R = p.R, Rp = p.Rp;
  const ScanStepLayout ly(chan, p.group, Rp);
  float* h_s = reinterpret_cast<float*>(smem + ly.h);
  bf16* w_s = reinterpret_cast<bf16*>(smem + ly.w);
  float* a_s = reinterpret_cast<float*>(smem + ly.a);
  float* bias_s = reinterpret_cast<float*>(smem + ly.bias);
  float* d_s = reinterpret_cast<float*>(smem + ly.dv);
  float* uc_s = reinterpret_cast<float*>(smem + ly.uc);
  float* bc_s = reinterpret_cast<float*>(smem + ly.bc);
  float* dt_s = reinterpret_cast<float*>(smem + ly.dt);

  // ---- inputs that do not depend on the kernels before this one: the state,
  // W_dt, A, b_dt and D slices (the caller's tensors; nothing in this call
  // writes them before this kernel)
  for (int i = tid; i < (ly.mtl * 16 - chan) * ly.dp; i += kThreads)   // W_dt rows past the slice
    w_s[chan * ly.dp + i] = __float2bfloat16_rn(0.0f);
  for (int i = tid; i < chan * (Rp - R); i += kThreads)                   // k padding
    w_s[(i / (Rp - R)) * ly.dp + R + i % (Rp - R)] = __float2bfloat16_rn(0.0f);
  {
    const int hc = chan * kStateN / 4;                        // 16-byte chunks per sequence
    for (int i = tid; i < ns * hc; i += kThreads) {
      const int s = i / hc, k = i % hc;
      cp_async16(h_s + (s * chan) * kStateN + 4 * k, p.h + (static_cast<long long>(s0 + s) * Di + c0) * kStateN + 4 * k);
    }
    const int rc = R / 8;
    for (int i = tid; i < chan * rc; i += kThreads) {
      const int r = i / rc, k = i % rc;
      cp_async16(w_s + r * ly.dp + 8 * k, p.dt_proj_w + static_cast<long long>(c0 + r) * R + 8 * k);
    }
    for (int i = tid; i < chan * kStateN / 4; i += kThreads)
      cp_async16(a_s + 4 * i, p.A + static_cast<long long>(c0) * kStateN + 4 * i);
    for (int i = tid; i < chan / 4; i += kThreads) {
      cp_async16(bias_s + 4 * i, p.dt_bias + c0 + 4 * i);
      cp_async16(d_s + 4 * i, p.D + c0 + 4 * i);
    }
    cp_async_commit();
  }
  pdl_wait();   // step_proj (uc) and step_reduce (delta, B, C) are complete
  for (int i = tid; i < ns * (chan / 4); i += kThreads) {
    const int s = i / (chan / 4), k = i % (chan / 4);
    cp_async16(uc_s + s * chan + 4 * k, p.uc + static_cast<long long>(s0 + s) * Di + c0 + 4 * k);
  }
  for (int i = tid; i < ns * 2 * kStateN / 4; i += kThreads)
    cp_async16(bc_s + 4 * i, p.bc + static_cast<long long>(s0) * 2 * kStateN + 4 * i);
  cp_async_commit();

  // dt_proj: D[c][n] = sum_r W_dt[c][r] dts[n][r]; warp w takes n-blocks 2w,
  // 2w + 1 of the group (B fragments straight from the split pair in L2)
  const int nblk = (ns + 3) / 4, ksteps = Rp / 16;
  uint32_t bfr[2][14][2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int nb = 2 * warp + k;
    const long long row = 2LL * s0 + 8 * nb + g;          // global split-pair row
    const bool live = nb < nblk && row < 2LL * (s0 + ns);
#pragma unroll
    for (int ks = 0; ks < 14; ++ks) {
      uint2 v = make_uint2(0u, 0u);
      if (live && ks < ksteps) v = *reinterpret_cast<const uint2*>(p.dts + row * Rp + ks * 16 + 4 * t);
      bfr[k][ks][0] = v.x;
      bfr[k][ks][1] = v.y;
    }
  }
  cp_async_wait<0>();
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int nb = 2 * warp + k;
    if (nb >= nblk) break;
    for (int mt = 0; mt < ly.mtl; ++mt) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 14; ++ks) {
        if (ks >= ksteps) break;
        const uint2 a_lo = lds64(w_s + (mt * 16 + g) * ly.dp + ks * 16 + 4 * t);
        const uint2 a_hi = lds64(w_s + (mt * 16 + g + 8) * ly.dp + ks * 16 + 4 * t);
        mma16816(acc, a_lo.x, a_hi.x, a_lo.y, a_hi.y, bfr[k][ks][0], bfr[k][ks][1]);
      }
      const int s = 4 * nb + t;
      if (s < ns) {
        const int c = mt * 16 + g;
        if (c < chan) dt_s[s * chan + c] = softplus(acc[0] + acc[1] + bias_s[c]);
        if (c + 8 < chan) dt_s[s * chan + c + 8] = softplus(acc[2] + acc[3] + bias_s[c + 8]);
      }
    }
  }
  __syncthreads();

  // state update and readout: item (s, c, quarter q) owns states 4q .. 4q+3;
  // the 4 quarters of a channel are 4 consecutive lanes, and every warp runs
  // the same number of items (ns * chan * 4 is a multiple of 32)
  const int total = ns * chan * 4;
  int s = 0, c = tid >> 2;
  while (c >= chan) { c -= chan; ++s; }
  const int q = tid & 3;
  for (int it = tid; it < total; it += kThreads) {
    const float4 hv = *reinterpret_cast<const float4*>(h_s + (s * chan + c) * kStateN + 4 * q);
    const float4 av = *reinterpret_cast<const float4*>(a_s + c * kStateN + 4 * q);
    const float d = dt_s[s * chan + c];
    const float uu = uc_s[s * chan + c];
    const float4 bv = *reinterpret_cast<const float4*>(bc_s + s * 2 * kStateN + 4 * q);
    const float4 cv = *reinterpret_cast<const float4*>(bc_s + s * 2 * kStateN + kStateN + 4 * q);
    const float dl = d * kLog2e, du = d * uu;
    float4 hn;
    hn.x = fmaf(ex2_approx(dl * av.x), hv.x, du * bv.x);
    hn.y = fmaf(ex2_approx(dl * av.y), hv.y, du * bv.y);
    hn.z = fmaf(ex2_approx(dl * av.z), hv.z, du * bv.z);
    hn.w = fmaf(ex2_approx(dl * av.w), hv.w, du * bv.w);
    float y = cv.x * hn.x;
    y = fmaf(cv.y, hn.y, y);
    y = fmaf(cv.z, hn.z, y);
    y = fmaf(cv.w, hn.w, y);
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 2);
    const long long hc = static_cast<long long>(s0 + s) * Di + c0 + c;
    *reinterpret_cast<float4*>(p.h + hc * kStateN + 4 * q) = hn;
    if (q == 0) p.m_t[hc] = __float2bfloat16_rn(fmaf(d_s[c], uu, y));
    c += kThreads / 4;
    while (c >= chan) { c -= chan; ++s; }
  }
}

// ------------------------------------------------------------------ step_fused

// The same step as ONE kernel when every slice fits one CTA of all sequences
// (batch <= 64) and the slices fit the GPU at one CTA per SM: launched
// cooperatively, so all CTAs are resident together, and the two points where
// the step needs every slice's result (the x_proj sum over channels, then its
// use by every slice) are grid-wide meeting points instead of kernel
// boundaries.  The slice's W_dt, A, b_dt and D slices arrive by cp.async
// behind the conv's own loads, and its state as one tensor copy issued once
// the conv is done; both land under the partial x_proj and the meetings.
//
//   phase 0   conv of the slice (uc stays in shared memory), partial x_proj
//             sums part[slice][seq][j] (m16n8k16)
//   meet 1
//   phase 1   CTA k sums outputs [k per, (k + 1) per) of [delta | B | C] over
//             the slices: warp w adds slices [w spw, (w + 1) spw) in order,
//             then the warps' sums are added in warp order (a fixed order)
//   meet 2
//   phase 2   dt = softplus(delta W_dt^T + b_dt) for the slice (m16n8k16), the
//             state update and readout
//
// Meeting points: after a CTA barrier, CTA b stores `target` into its own
// flag with release semantics (cumulative over the CTA's writes ordered
// before it by the barrier), and one warp of every CTA reads all flags
// (relaxed) until each holds `target`, then fences (acquire) before the CTA
// barrier that releases the other warps.  Each flag has a 128-byte line of
// its own, so the reads spread over the L2.  `target` = the generation word +
// 1; CTA 0 advances the generation word after the second meeting, when every
// CTA has read it, so flags left by an earlier call never match whatever the
// words held before.  Waits are bounded (wait_limit cycles); a CTA whose wait
// runs out records the timeout status, lets its copies in flight land and
// returns.
constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kMaxSpw = 10;       // slices per warp in phase 1 (148 slices / 16 warps)
constexpr int kFlagStride = 16;   // u64 words between flags (one 128-byte line each)
constexpr int kMaxMeetCtas = 160; // CTAs a meeting point's polling warp covers (5 flags per lane)
static_assert(kMaxGroup * (kMaxChan / 8) <= kFusedThreads, "one conv item per thread");

__host__ __device__ constexpr int fused_per_cta(int ldx, int B, int nslice) {
  return (ldx * B + nslice - 1) / nslice;
}
__host__ __device__ constexpr int max_i(int a, int b) { return a > b ? a : b; }
// meeting words: generation (own line), then two arrays of nslice flags
__host__ __device__ constexpr long long fused_bar_words(int nslice) {
  return static_cast<long long>(kFlagStride) * (1 + 2 * nslice);
}

// Dynamic shared memory of step_fused (byte offsets).
struct FusedStepLayout {
  int mtl, dp, per;
  int h, w, a, bias, dv, uc, bc, un, misc, bytes;
  __host__ __device__ FusedStepLayout(int chan, int B, int Rp, int ldx, int nslice) {
    mtl = (chan + 15) / 16;
    dp = frag_pitch(Rp);
    per = fused_per_cta(ldx, B, nslice);
    h = 0;                                             // f32 [B][chan][N]
    w = h + B * chan * kStateN * 4;                    // bf16 [mtl*16][dp] W_dt rows
    a = w + round_up(mtl * 16 * dp * 2, 16);           // f32 [chan][N]
    bias = a + chan * kStateN * 4;                     // f32 [chan]
    dv = bias + round_up(chan * 4, 16);                // f32 [chan]
    uc = dv + round_up(chan * 4, 16);                  // f32 [B][chan]
    bc = uc + round_up(B * chan * 4, 16);              // f32 [B][2N]
    un = bc + B * 2 * kStateN * 4;                     // one of, by phase:
    const int ucs_b = 2 * round_up(B, 4) * kUcsPitch * 2;   //   bf16 conv output split pair
    const int red_b = kFusedWarps * per * 4;                 //   f32 [warps][per] phase-1 sums
    const int dt_b = B * chan * 4;                           //   f32 [B][chan] dt
    misc = un + round_up(max_i(ucs_b, max_i(red_b, dt_b)), 16);   // u64 generation, int ok, u64 mbarrier
    bytes = misc + 24;
  }
};

// mbarrier and bulk-copy glue (non-multicast forms only)
__device__ __forceinline__ uint32_t sh_addr(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}
__device__ __forceinline__ void mb_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(sh_addr(bar)), "r"(count));
}
__device__ __forceinline__ void mb_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sh_addr(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mb_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(ok)
      : "r"(sh_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait for phase `parity` of `bar`
__device__ __forceinline__ bool mb_wait(uint64_t* bar, uint32_t parity, unsigned long long limit) {
  if (mb_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mb_try_wait(bar, parity))
    if (static_cast<unsigned long long>(clock64() - t0) > limit) return false;
  return true;
}
// 3-D tensor copy global -> shared completing on `bar` (no multicast)
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          sh_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(sh_addr(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* ptr) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ptr) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u64(unsigned long long* ptr, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(ptr), "l"(v) : "memory");
}

// Grid-wide meeting point (see above).  Every thread of the CTA returns the
// same answer: false if some flag did not arrive in time.
__device__ bool grid_meet(unsigned long long* flags, unsigned long long target, unsigned long long limit,
                          int* ok_s) {
  __syncthreads();   // the CTA's writes before the release below (cumulative)
  if (threadIdx.x == 0) st_release_u64(flags + static_cast<long long>(blockIdx.x) * kFlagStride, target);
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const long long t0 = clock64();
    while (true) {
      // all of the lane's flags (at most 5 of 148) read at once, then compared
      unsigned long long v[5];
#pragma unroll
      for (int k = 0; k < 5; ++k) {
        const int i = lane + 32 * k;
        v[k] = i < static_cast<int>(gridDim.x) ? ld_relaxed_u64(flags + static_cast<long long>(i) * kFlagStride)
                                                : target;
      }
      bool mine = true;
#pragma unroll
      for (int k = 0; k < 5; ++k) mine = mine && v[k] == target;
      if (__all_sync(0xffffffffu, mine)) break;
      if (static_cast<unsigned long long>(clock64() - t0) > limit) {
        if (lane == 0) {
          *reinterpret_cast<volatile int*>(ok_s) = 0;
          record_status(kStatusTimeout);
        }
        break;
      }
      __nanosleep(32);
    }
    asm volatile("fence.acq_rel.gpu;" ::: "memory");   // later reads of other CTAs' data see their writes
  }
  __syncthreads();
  return *reinterpret_cast<volatile int*>(ok_s) != 0;
}

__global__ void __launch_bounds__(kFusedThreads, 1) step_fused_kernel(const StepParams p,
                                                                     const __grid_constant__ CUtensorMap hmap) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int chan = p.chan, c0 = blockIdx.x * chan, B = p.B;
  const int Di = p.Di, R = p.R, Rp = p.Rp, ldx = p.ldx, nslice = p.nslice;
  const FusedStepLayout ly(chan, B, Rp, ldx, nslice);
  float* h_s = reinterpret_cast<float*>(smem + ly.h);
  bf16* w_s = reinterpret_cast<bf16*>(smem + ly.w);
  float* a_s = reinterpret_cast<float*>(smem + ly.a);
  float* bias_s = reinterpret_cast<float*>(smem + ly.bias);
  float* d_s = reinterpret_cast<float*>(smem + ly.dv);
  float* uc_s = reinterpret_cast<float*>(smem + ly.uc);
  float* bc_s = reinterpret_cast<float*>(smem + ly.bc);
  bf16* ucs = reinterpret_cast<bf16*>(smem + ly.un);
  float* red_s = reinterpret_cast<float*>(smem + ly.un);
  float* dt_s = reinterpret_cast<float*>(smem + ly.un);
  unsigned long long& gen_s = *reinterpret_cast<unsigned long long*>(smem + ly.misc);
  int& ok_s = *reinterpret_cast<int*>(smem + ly.misc + 8);
  uint64_t* mb = reinterpret_cast<uint64_t*>(smem + ly.misc + 16);
  if (tid == 0) {
    ok_s = 1;
    gen_s = *reinterpret_cast<volatile unsigned long long*>(p.bar);
    mb_init(mb, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_smem();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&hmap)) : "memory");
  }
  pdl_launch_dependents();
  __syncthreads();

  // ---- phase 0a: what the conv and the partial x_proj need first, to
  // registers: the W_x fragments of the warp's first row tile, and the
  // thread's conv item (8 channels of one sequence; 4 nblk vpc <= 384 items,
  // at most one per thread)
  const int kc = round_up(chan, 16), ksteps = kc / 16;
  const int mtiles = (ldx + 15) / 16;
  auto load_wx = [&](int mt, uint32_t (&a)[3][4]) {
#pragma unroll
    for (int ks = 0; ks < 3; ++ks) {
      const int col = c0 + ks * 16 + 4 * t;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int j = mt * 16 + g + 8 * half;
        uint2 v = make_uint2(0u, 0u);
        if (ks < ksteps && j < ldx && col + 3 < Di)
          v = *reinterpret_cast<const uint2*>(p.x_proj_w + static_cast<long long>(j) * Di + col);
        a[ks][half] = v.x;          // logical k 2t, 2t+1
        a[ks][2 + half] = v.y;      // logical k 2t+8, 2t+9
      }
    }
  };
  uint32_t afr[3][4];
  if (warp < mtiles) load_wx(warp, afr);
  const int nblk = (B + 3) / 4;
  const int vpc = chan / 8;
  const int cs = tid / vpc, cl = (tid % vpc) * 8;     // conv item: sequence cs, channels cl .. cl+7
  const bool conv_item = tid < 4 * nblk * vpc;
  const bool conv_live = conv_item && cs < B;
  const long long coff = static_cast<long long>(cs) * Di + c0 + cl;
  Pack16 in, cbias, win[4], wt[4];
  if (conv_live) {
    in.u = *reinterpret_cast<const uint4*>(p.u_t + coff);
    cbias.u = *reinterpret_cast<const uint4*>(p.conv_b + c0 + cl);
    const uint4* wp = reinterpret_cast<const uint4*>(p.conv_state + coff * kConvK);
    const uint4* kp = reinterpret_cast<const uint4*>(p.conv_w + static_cast<long long>(c0 + cl) * kConvK);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      win[j].u = wp[j];
      wt[j].u = kp[j];
    }
  }

  // ---- phase 0b, behind those loads: the W_dt rows, A, b_dt and D slices
  // (cp.async), landing while the conv, the x_proj and both meetings run.
  // The slice's state follows after the conv as ONE tensor copy (box {128
  // floats, chan / 8, B} of h viewed as [B][Di / 8][128]) landing on `mb`.
  {
    const int rc = R / 8;
    for (int i = tid; i < chan * rc; i += kFusedThreads) {
      const int r = i / rc, k = i % rc;
      cp_async16(w_s + r * ly.dp + 8 * k, p.dt_proj_w + static_cast<long long>(c0 + r) * R + 8 * k);
    }
    for (int i = tid; i < chan * kStateN / 4; i += kFusedThreads)
      cp_async16(a_s + 4 * i, p.A + static_cast<long long>(c0) * kStateN + 4 * i);
    for (int i = tid; i < chan / 4; i += kFusedThreads) {
      cp_async16(bias_s + 4 * i, p.dt_bias + c0 + 4 * i);
      cp_async16(d_s + 4 * i, p.D + c0 + 4 * i);
    }
    cp_async_commit();
  }
  for (int i = tid; i < (ly.mtl * 16 - chan) * ly.dp; i += kFusedThreads)   // W_dt rows past the slice
    w_s[chan * ly.dp + i] = __float2bfloat16_rn(0.0f);
  for (int i = tid; i < chan * (Rp - R); i += kFusedThreads)                   // k padding
    w_s[(i / (Rp - R)) * ly.dp + R + i % (Rp - R)] = __float2bfloat16_rn(0.0f);

  // ---- phase 0c: conv + SiLU (window shifted in place)
  if (conv_item) {
    float y[8];
    if (conv_live) {
      bf16* wv = reinterpret_cast<bf16*>(win);            // [8 channels][K], oldest first
      const bf16* kv = reinterpret_cast<const bf16*>(wt);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
#pragma unroll
        for (int k = 0; k < kConvK - 1; ++k) wv[e * kConvK + k] = wv[e * kConvK + k + 1];
        wv[e * kConvK + kConvK - 1] = in.h[e];
        float acc = __bfloat162float(cbias.h[e]);
#pragma unroll
        for (int k = 0; k < kConvK; ++k)
          acc = fmaf(__bfloat162float(kv[e * kConvK + k]), __bfloat162float(wv[e * kConvK + k]), acc);
        y[e] = silu(acc);
      }
      uint4* wp = reinterpret_cast<uint4*>(p.conv_state + coff * kConvK);
#pragma unroll
      for (int j = 0; j < 4; ++j) wp[j] = win[j].u;
      float4* us = reinterpret_cast<float4*>(uc_s + cs * chan + cl);
      us[0] = make_float4(y[0], y[1], y[2], y[3]);
      us[1] = make_float4(y[4], y[5], y[6], y[7]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = 0.0f;
    }
    Pack16 hi, lo;
#pragma unroll
    for (int e = 0; e < 8; ++e) split_bf16(y[e], hi.h[e], lo.h[e]);
    *reinterpret_cast<uint4*>(ucs + (2 * cs) * kUcsPitch + cl) = hi.u;
    *reinterpret_cast<uint4*>(ucs + (2 * cs + 1) * kUcsPitch + cl) = lo.u;
  }
  for (int it = tid; it < 8 * nblk * (kc - chan); it += kFusedThreads) {   // k padding
    const int r = it / (kc - chan), c = chan + it % (kc - chan);
    ucs[r * kUcsPitch + c] = __float2bfloat16_rn(0.0f);
  }
  __syncthreads();
  // the slice's state, once the conv's own reads are done (so they did not
  // queue behind it); it lands under the x_proj and both meetings
  if (tid == 0) {
    mb_expect_tx(mb, static_cast<uint32_t>(B) * chan * kStateN * 4);
    tma_load_3d(h_s, &hmap, mb, 0, c0 / 8, 0);
  }

  // ---- phase 0d: partial x_proj D[j][n] = sum_{c in slice} W_x[j][c] ucs[n][c],
  // stored as part[slice][seq][j]
  for (int mt = warp; mt < mtiles; mt += kFusedWarps) {
    if (mt != warp) load_wx(mt, afr);
    float acc[16][4];
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.0f;
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) {
      if (nb >= nblk) break;
#pragma unroll
      for (int ks = 0; ks < 3; ++ks) {
        if (ks >= ksteps) break;
        const uint2 b = lds64(ucs + (8 * nb + g) * kUcsPitch + ks * 16 + 4 * t);
        mma16816(acc[nb], afr[ks][0], afr[ks][1], afr[ks][2], afr[ks][3], b.x, b.y);
      }
    }
    float* part = p.part + static_cast<long long>(blockIdx.x) * B * ldx;
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) {            // D[j][8nb + 2t + {0, 1}]: (hi, lo) of sequence 4nb + t
      if (nb >= nblk) break;
      const int s = 4 * nb + t;
      if (s >= B) continue;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int j = mt * 16 + g + 8 * half;
        if (j < ldx) part[s * ldx + j] = acc[nb][2 * half] + acc[nb][2 * half + 1];
      }
    }
  }

  const unsigned long long target = gen_s + 1;
  unsigned long long* flags1 = p.bar + kFlagStride;
  unsigned long long* flags2 = flags1 + static_cast<long long>(nslice) * kFlagStride;
  if (!grid_meet(flags1, target, p.wait_limit, &ok_s)) {
    cp_async_wait<0>();
    mb_wait(mb, 0, p.wait_limit);   // copies into this CTA's shared memory land before it leaves
    return;
  }

  // ---- phase 1: outputs [o0, o1) of [delta | B | C] (o = seq * ldx + j);
  // every load of a lane (kRounds rounds of 32 outputs x its slices) in flight
  // at once, then the adds in slice order
  {
    constexpr int kRounds = 4;
    const int per = ly.per, total = ldx * B;
    const int o0 = blockIdx.x * per, o1 = min(total, o0 + per);
    const int spw = (nslice + kFusedWarps - 1) / kFusedWarps;
    const int sl0 = warp * spw, sl1 = min(nslice, sl0 + spw);
    const long long sstride = static_cast<long long>(ldx) * B;
    for (int r0 = 0; r0 * 32 < per; r0 += kRounds) {
      float x[kRounds][kMaxSpw];
#pragma unroll
      for (int rr = 0; rr < kRounds; ++rr) {
        const int oi = (r0 + rr) * 32 + lane, o = o0 + oi;
        const bool valid = oi < per && o < o1;
#pragma unroll
        for (int k = 0; k < kMaxSpw; ++k)
          x[rr][k] = (valid && sl0 + k < sl1) ? __ldcg(p.part + (sl0 + k) * sstride + o) : 0.0f;
      }
#pragma unroll
      for (int rr = 0; rr < kRounds; ++rr) {
        const int oi = (r0 + rr) * 32 + lane;
        float acc = 0.0f;
#pragma unroll
        for (int k = 0; k < kMaxSpw; ++k) acc += x[rr][k];
        if (oi < per) red_s[warp * per + oi] = acc;
      }
    }
    __syncthreads();
    for (int i = tid; i < o1 - o0; i += kFusedThreads) {
      float acc = 0.0f;
      for (int w2 = 0; w2 < kFusedWarps; ++w2) acc += red_s[w2 * per + i];
      const int o = o0 + i, s = o / ldx, j = o % ldx;
      if (j < R) {
        bf16 hi, lo;
        split_bf16(acc, hi, lo);
        p.dts[(2LL * s) * Rp + j] = hi;
        p.dts[(2LL * s + 1) * Rp + j] = lo;
      } else {
        p.bc[static_cast<long long>(s) * 2 * kStateN + (j - R)] = acc;
      }
    }
    if (blockIdx.x == 0)
      for (int i = tid; i < 2 * B * (Rp - R); i += kFusedThreads)
        p.dts[(i / (Rp - R)) * Rp + R + i % (Rp - R)] = __float2bfloat16_rn(0.0f);
  }

  if (!grid_meet(flags2, target, p.wait_limit, &ok_s)) {
    cp_async_wait<0>();
    mb_wait(mb, 0, p.wait_limit);
    return;
  }
  if (blockIdx.x == 0 && tid == 0) *reinterpret_cast<volatile unsigned long long*>(p.bar) = target;

  // ---- phase 2: B | C of every sequence, delta fragments, dt, state update
  for (int i = tid; i < B * 2 * kStateN / 4; i += kFusedThreads) cp_async16(bc_s + 4 * i, p.bc + 4 * i);
  cp_async_commit();
  const int kst = Rp / 16;
  uint32_t bfr[14][2];
  {
    const int row = 8 * warp + g;                       // split-pair row of n-block `warp`
    const bool live = warp < nblk && row < 2 * B;
#pragma unroll
    for (int ks = 0; ks < 14; ++ks) {
      uint2 v = make_uint2(0u, 0u);
      if (live && ks < kst)
        v = __ldcg(reinterpret_cast<const uint2*>(p.dts + static_cast<long long>(row) * Rp + ks * 16 + 4 * t));
      bfr[ks][0] = v.x;
      bfr[ks][1] = v.y;
    }
  }
  cp_async_wait<0>();
  if (!mb_wait(mb, 0, p.wait_limit)) {
    *reinterpret_cast<volatile int*>(&ok_s) = 0;
    record_status(kStatusTimeout);
  }
  __syncthreads();
  if (!*reinterpret_cast<volatile int*>(&ok_s)) return;
  if (warp < nblk) {          // n-block `warp`, the slice's (at most 3) row tiles side by side
    float acc[3][4] = {};
#pragma unroll
    for (int ks = 0; ks < 14; ++ks) {
      if (ks >= kst) break;
#pragma unroll
      for (int mt = 0; mt < 3; ++mt) {
        if (mt >= ly.mtl) break;
        const uint2 a_lo = lds64(w_s + (mt * 16 + g) * ly.dp + ks * 16 + 4 * t);
        const uint2 a_hi = lds64(w_s + (mt * 16 + g + 8) * ly.dp + ks * 16 + 4 * t);
        mma16816(acc[mt], a_lo.x, a_hi.x, a_lo.y, a_hi.y, bfr[ks][0], bfr[ks][1]);
      }
    }
    const int s = 4 * warp + t;
    if (s < B) {
#pragma unroll
      for (int mt = 0; mt < 3; ++mt) {
        if (mt >= ly.mtl) break;
        const int c = mt * 16 + g;
        if (c < chan) dt_s[s * chan + c] = softplus(acc[mt][0] + acc[mt][1] + bias_s[c]);
        if (c + 8 < chan) dt_s[s * chan + c + 8] = softplus(acc[mt][2] + acc[mt][3] + bias_s[c + 8]);
      }
    }
  }
  __syncthreads();

  // state update and readout: thread (row, c, quarter q) owns states 4q ..
  // 4q+3 of channel c for sequences row, row + rows, ...; chan * 4 threads
  // per row (a multiple of 32: warps never straddle rows), the quarters of a
  // channel on 4 consecutive lanes
  const int per_row = chan * 4, rows = kFusedThreads / per_row;
  if (tid < rows * per_row) {
    const int row = tid / per_row, c = (tid % per_row) >> 2, q = tid & 3;
    const float4 av = *reinterpret_cast<const float4*>(a_s + c * kStateN + 4 * q);
    const float4 al = make_float4(av.x * kLog2e, av.y * kLog2e, av.z * kLog2e, av.w * kLog2e);
    const float dd = d_s[c];
#pragma unroll 2
    for (int s = row; s < B; s += rows) {
      const float4 hv = ld_shared_f4(h_s + (s * chan + c) * kStateN + 4 * q);
      const float d = ld_shared_f32(dt_s + s * chan + c);
      const float uu = ld_shared_f32(uc_s + s * chan + c);
      const float4 bv = ld_shared_f4(bc_s + s * 2 * kStateN + 4 * q);
      const float4 cv = ld_shared_f4(bc_s + s * 2 * kStateN + kStateN + 4 * q);
      const float du = d * uu;
      float4 hn;
      hn.x = fmaf(ex2_approx(d * al.x), hv.x, du * bv.x);
      hn.y = fmaf(ex2_approx(d * al.y), hv.y, du * bv.y);
      hn.z = fmaf(ex2_approx(d * al.z), hv.z, du * bv.z);
      hn.w = fmaf(ex2_approx(d * al.w), hv.w, du * bv.w);
      float y = cv.x * hn.x;
      y = fmaf(cv.y, hn.y, y);
      y = fmaf(cv.z, hn.z, y);
      y = fmaf(cv.w, hn.w, y);
      y += __shfl_xor_sync(0xffffffffu, y, 1);
      y += __shfl_xor_sync(0xffffffffu, y, 2);
      const long long hc = static_cast<long long>(s) * Di + c0 + c;
      *reinterpret_cast<float4*>(p.h + hc * kStateN + 4 * q) = hn;
      if (q == 0) p.m_t[hc] = __float2bfloat16_rn(fmaf(dd, uu, y));
    }
  }
}

}  // namespace step
}  // namespace sambay
