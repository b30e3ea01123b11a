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

}  // namespace step
}  // namespace sambay
