// SambaY-2 memory readout: the Mamba-2 SSD scan, chunked on the tensor cores
// (sm_100a, m16n8k16 bf16 MMAs with fp32 accumulation).
//
// The SambaY-2 row of the ablation table ("Decoder-Hybrid-Decoder
// Architecture for Efficient Reasoning with Long Generation", Paper-Notes
// page, 实验关键数据 > 消融实验) replaces Mamba by Mamba-2, whose forget gate
// is one scalar per head (Dao & Gu 2024, "Transformers are SSMs", SSD):
//
//   H_t = exp(dt_t A_h) H_{t-1} + dt_t x_t B_t^T     H in R^{P x N} per head
//   y_t = H_t C_t + D_h x_t                          B_t, C_t shared by heads
//
// Chunked form, chunk of kQ = 64 tokens, c_t = A_h sum_{k <= t} dt_k within
// the chunk:
//   y_t = exp(c_t) C_t . H_in                                  (carry)
//       + sum_{s <= t} (C_t . B_s) exp(c_t - c_s) dt_s x_s     (intra-chunk)
//       + D x_t
//   H_out = exp(c_end) H_in + sum_s exp(c_end - c_s) dt_s x_s B_s^T
// All four products are small GEMMs: G = C B^T (64 x 64, K = N), Y = W X
// with W = G masked and scaled (64 x P, K = 64), C H_in (64 x P, K = N) and
// S = (B scaled)^T X (N x P, K = 64).
//
// CTA: one (sequence, head), 4 warps, the chunks in order.  Warp w owns the
// output rows t in [16 w, 16 w + 16) of the chunk and the state rows n in
// [N w / 4, N (w + 1) / 4); the fp32 state lives in its MMA accumulator
// registers across chunks, with a bf16 copy in shared memory for the carry
// product.  Operands come from shared memory by ldmatrix (.trans where the
// stored tile is K-major for the operand); W goes from accumulator fragments
// straight into A fragments.  Operands are bf16 (x, B, C: the hi half of the
// conv output's split pair; W and the state copy rounded), accumulation and
// the state fp32.
#pragma once

#include "common.cuh"

namespace sambay {
namespace ssd {

constexpr int kQ = 64;          // tokens per chunk
constexpr int kP = 64;          // head dim
constexpr int kThreads = 128;   // 4 warps
constexpr int kMaxN = 128;      // d_state

struct SsdParams {
  const bf16* xc;        // [Bt*L, 2*C] conv output split pair (hi | lo), C = H*P + 2N
  const bf16* dt_raw;    // [Bt*L, H]
  const float* dt_bias;  // [H]
  const float* A;        // [H]
  const float* D;        // [H]
  float* h;              // [Bt, H, P, N] in/out
  bf16* M;               // [Bt*L, H*P] out
  int Bt, L, H, N;
  int zero_init;
};

// shared-memory tile pitches (bf16 elements): rows 16 bytes past a multiple of
// 128 so the 8 row addresses of an ldmatrix hit distinct bank groups
constexpr int kPitchP = kP + 8;          // x tiles, state copy
__host__ __device__ constexpr int pitch_n(int N) { return N + 8; }

struct SsdLayout {
  int x, xl, b, c, hs, dt, cs, bytes;
  __host__ __device__ SsdLayout(int N) {
    x = 0;                                   // bf16 [kQ][kPitchP]  x hi
    xl = x + kQ * kPitchP * 2;               // bf16 [kQ][kPitchP]  x lo
    b = xl + kQ * kPitchP * 2;               // bf16 [kQ][pitch_n]  B, then B scaled
    c = b + kQ * pitch_n(N) * 2;             // bf16 [kQ][pitch_n]  C
    hs = c + kQ * pitch_n(N) * 2;            // bf16 [N][kPitchP]   state copy
    dt = hs + N * kPitchP * 2;               // f32 [kQ]
    cs = dt + kQ * 4;                        // f32 [kQ] c_t log2(e)
    bytes = cs + kQ * 4;
  }
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

// A fragment (16 x 16 at row r0, column k0) of a row-major [rows][pitch] tile
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], const bf16* tile, int pitch, int r0, int k0, int lane) {
  const int j = lane >> 3, i = lane & 7;
  ldsm_x4(a, tile + (r0 + (j & 1) * 8 + i) * pitch + k0 + (j >> 1) * 8);
}
// A fragment of a tile stored K-major ([k][pitch], m contiguous)
__device__ __forceinline__ void frag_a_t(uint32_t (&a)[4], const bf16* tile, int pitch, int m0, int k0, int lane) {
  const int j = lane >> 3, i = lane & 7;
  ldsm_x4_t(a, tile + (k0 + (j >> 1) * 8 + i) * pitch + m0 + (j & 1) * 8);
}
// B fragments of two n8 tiles (n0, n0 + 8), one k16 step at k0, from a tile
// stored N-major ([n][pitch], k contiguous): b[0], b[1] tile n0; b[2], b[3] n0 + 8
__device__ __forceinline__ void frag_b(uint32_t (&b)[4], const bf16* tile, int pitch, int n0, int k0, int lane) {
  const int j = lane >> 3, i = lane & 7;
  ldsm_x4(b, tile + (n0 + (j >> 1) * 8 + i) * pitch + k0 + (j & 1) * 8);
}
// the same from a tile stored K-major ([k][pitch], n contiguous)
__device__ __forceinline__ void frag_b_t(uint32_t (&b)[4], const bf16* tile, int pitch, int n0, int k0, int lane) {
  const int j = lane >> 3, i = lane & 7;
  ldsm_x4_t(b, tile + (k0 + (j & 1) * 8 + i) * pitch + n0 + (j >> 1) * 8);
}

__global__ void __launch_bounds__(kThreads) ssd_chunk_scan_kernel(const SsdParams p) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(128) uint8_t smem[];
  const int N = p.N, H = p.H, L = p.L;
  const int PN = pitch_n(N);
  const SsdLayout ly(N);
  bf16* xs = reinterpret_cast<bf16*>(smem + ly.x);
  bf16* xl = reinterpret_cast<bf16*>(smem + ly.xl);
  bf16* bs = reinterpret_cast<bf16*>(smem + ly.b);
  bf16* cs_t = reinterpret_cast<bf16*>(smem + ly.c);
  bf16* hs = reinterpret_cast<bf16*>(smem + ly.hs);
  float* dts = reinterpret_cast<float*>(smem + ly.dt);
  float* c2 = reinterpret_cast<float*>(smem + ly.cs);
  const int b = blockIdx.y, hd = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int C = H * kP + 2 * N;                  // conv channels
  const long long ldx = 2LL * C;                  // split-pair row pitch
  const float A2 = p.A[hd] * kLog2e, Dh = p.D[hd], bias = p.dt_bias[hd];
  const int nrow = N / 4;                         // state rows per warp
  const int ntm = nrow / 16;                      // their m16 tiles (1 or 2)
  float* hglob = p.h + (static_cast<long long>(b) * H + hd) * kP * N;   // [P][N]

  // the state, fp32 in this warp's accumulators: tile (mi, pj) holds rows
  // n = n0 + 16 mi + {g, g + 8}, columns p = 8 pj + 2 t4 + {0, 1}
  float st[2][8][4];
  const int n0 = warp * nrow;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int pj = 0; pj < 8; ++pj)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int n = n0 + 16 * mi + g + (e >> 1) * 8, pp = 8 * pj + 2 * t4 + (e & 1);
        st[mi][pj][e] = (mi < ntm && !p.zero_init) ? hglob[pp * N + n] : 0.0f;
      }
  auto store_state_copy = [&]() {
#pragma unroll
    for (int mi = 0; mi < 2; ++mi) {
      if (mi >= ntm) break;
#pragma unroll
      for (int pj = 0; pj < 8; ++pj) {
        const int n = n0 + 16 * mi + g, pp = 8 * pj + 2 * t4;
        *reinterpret_cast<uint32_t*>(hs + n * kPitchP + pp) = pack2(st[mi][pj][0], st[mi][pj][1]);
        *reinterpret_cast<uint32_t*>(hs + (n + 8) * kPitchP + pp) = pack2(st[mi][pj][2], st[mi][pj][3]);
      }
    }
  };
  store_state_copy();

  const int nchunks = (L + kQ - 1) / kQ;
  for (int ck = 0; ck < nchunks; ++ck) {
    const int t0 = ck * kQ, nt = min(kQ, L - t0);
    // ---- the chunk's x (hi, lo), B, C (hi) rows; rows past L as zeros
    {
      const long long row0 = static_cast<long long>(b) * L + t0;
      for (int i = tid; i < kQ * (kP / 8); i += kThreads) {          // x: 8 pieces of 8 per row
        const int r = i / (kP / 8), k = i % (kP / 8);
        if (r < nt) {
          const bf16* src = p.xc + (row0 + r) * ldx + hd * kP + 8 * k;
          cp16(xs + r * kPitchP + 8 * k, src);
          cp16(xl + r * kPitchP + 8 * k, src + C);
        } else {
          *reinterpret_cast<uint4*>(xs + r * kPitchP + 8 * k) = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(xl + r * kPitchP + 8 * k) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      const int np = N / 8;
      for (int i = tid; i < kQ * np; i += kThreads) {                // B, C
        const int r = i / np, k = i % np;
        if (r < nt) {
          const bf16* src = p.xc + (row0 + r) * ldx + H * kP + 8 * k;
          cp16(bs + r * PN + 8 * k, src);
          cp16(cs_t + r * PN + 8 * k, src + N);
        } else {
          *reinterpret_cast<uint4*>(bs + r * PN + 8 * k) = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(cs_t + r * PN + 8 * k) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      if (warp == 0) {
        // dt = softplus(dt_raw + bias), c_t log2(e) = A log2(e) cumsum(dt):
        // lane holds tokens 2 lane, 2 lane + 1
        float d[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = 2 * lane + e;
          d[e] = r < nt ? softplus(__bfloat162float(p.dt_raw[(row0 + r) * H + hd]) + bias) : 0.0f;
        }
        float s = d[0] + d[1];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float o = __shfl_up_sync(0xffffffffu, s, off);
          if (lane >= off) s += o;
        }
        const float before = s - d[0] - d[1];
        dts[2 * lane] = d[0];
        dts[2 * lane + 1] = d[1];
        c2[2 * lane] = A2 * (before + d[0]);
        c2[2 * lane + 1] = A2 * s;
      }
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncthreads();
    }
    const float c2end = c2[kQ - 1];

    // ---- output rows of this warp: Y = exp(c_t) C H_in + W X + D x
    const int r0 = 16 * warp;
    float y[8][4];
#pragma unroll
    for (int pj = 0; pj < 8; ++pj) y[pj][0] = y[pj][1] = y[pj][2] = y[pj][3] = 0.0f;
    for (int kk = 0; kk < N / 16; ++kk) {                          // carry: C (rows t) . H (K = N)
      uint32_t a[4];
      frag_a(a, cs_t, PN, r0, 16 * kk, lane);
#pragma unroll
      for (int pj = 0; pj < 8; pj += 2) {
        uint32_t bb[4];
        frag_b_t(bb, hs, kPitchP, 8 * pj, 16 * kk, lane);
        mma(y[pj], a, bb[0], bb[1]);
        mma(y[pj + 1], a, bb[2], bb[3]);
      }
    }
    const float eg = ex2_approx(c2[r0 + g]), eg8 = ex2_approx(c2[r0 + g + 8]);
#pragma unroll
    for (int pj = 0; pj < 8; ++pj) {
      y[pj][0] *= eg; y[pj][1] *= eg; y[pj][2] *= eg8; y[pj][3] *= eg8;
    }
    // G = C B^T for rows t, all s; then W = G exp(c_t - c_s) dt_s (s <= t)
    float gacc[8][4];
#pragma unroll
    for (int sj = 0; sj < 8; ++sj) gacc[sj][0] = gacc[sj][1] = gacc[sj][2] = gacc[sj][3] = 0.0f;
    for (int kk = 0; kk < N / 16; ++kk) {
      uint32_t a[4];
      frag_a(a, cs_t, PN, r0, 16 * kk, lane);
#pragma unroll
      for (int sj = 0; sj < 8; sj += 2) {
        uint32_t bb[4];
        frag_b(bb, bs, PN, 8 * sj, 16 * kk, lane);
        mma(gacc[sj], a, bb[0], bb[1]);
        mma(gacc[sj + 1], a, bb[2], bb[3]);
      }
    }
    uint32_t wa[4][4];
    {
      const int ta = r0 + g, tb = ta + 8;
      const float cta = c2[ta], ctb = c2[tb];
#pragma unroll
      for (int sj = 0; sj < 8; ++sj) {
        const int s0 = 8 * sj + 2 * t4, s1 = s0 + 1;
        const float w0a = s0 <= ta ? ex2_approx(cta - c2[s0]) * dts[s0] : 0.0f;
        const float w1a = s1 <= ta ? ex2_approx(cta - c2[s1]) * dts[s1] : 0.0f;
        const float w0b = s0 <= tb ? ex2_approx(ctb - c2[s0]) * dts[s0] : 0.0f;
        const float w1b = s1 <= tb ? ex2_approx(ctb - c2[s1]) * dts[s1] : 0.0f;
        const uint32_t top = pack2(gacc[sj][0] * w0a, gacc[sj][1] * w1a);
        const uint32_t bot = pack2(gacc[sj][2] * w0b, gacc[sj][3] * w1b);
        // A fragment of k-step sj / 2: regs 0, 1 from n-tile 2kk, regs 2, 3 from 2kk + 1
        wa[sj >> 1][(sj & 1) * 2 + 0] = top;
        wa[sj >> 1][(sj & 1) * 2 + 1] = bot;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {                                // Y += W X (K = s)
#pragma unroll
      for (int pj = 0; pj < 8; pj += 2) {
        uint32_t bb[4];
        frag_b_t(bb, xs, kPitchP, 8 * pj, 16 * kk, lane);
        mma(y[pj], wa[kk], bb[0], bb[1]);
        mma(y[pj + 1], wa[kk], bb[2], bb[3]);
      }
    }
    {
      const int ta = r0 + g, tb = ta + 8;
      const long long rowa = static_cast<long long>(b) * L + t0 + ta, rowb = rowa + 8;
#pragma unroll
      for (int pj = 0; pj < 8; ++pj) {
        const int pp = 8 * pj + 2 * t4;
        if (ta < nt) {
          const float2 xh = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(xs + ta * kPitchP + pp));
          const float2 xo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(xl + ta * kPitchP + pp));
          *reinterpret_cast<__nv_bfloat162*>(p.M + rowa * (H * kP) + hd * kP + pp) =
              __floats2bfloat162_rn(y[pj][0] + Dh * (xh.x + xo.x), y[pj][1] + Dh * (xh.y + xo.y));
        }
        if (tb < nt) {
          const float2 xh = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(xs + tb * kPitchP + pp));
          const float2 xo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(xl + tb * kPitchP + pp));
          *reinterpret_cast<__nv_bfloat162*>(p.M + rowb * (H * kP) + hd * kP + pp) =
              __floats2bfloat162_rn(y[pj][2] + Dh * (xh.x + xo.x), y[pj][3] + Dh * (xh.y + xo.y));
        }
      }
    }
    __syncthreads();   // every warp is done with B (raw) and the state copy

    // ---- B scaled by exp(c_end - c_s) dt_s, in place
    for (int i = tid; i < kQ * (N / 2); i += kThreads) {
      const int r = i / (N / 2), k = 2 * (i % (N / 2));
      const float w = ex2_approx(c2end - c2[r]) * dts[r];
      __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(bs + r * PN + k);
      const float2 v = __bfloat1622float2(*q);
      *q = __floats2bfloat162_rn(v.x * w, v.y * w);
    }
    __syncthreads();
    // ---- state: H = exp(c_end) H + (B scaled)^T X for this warp's rows n
    const float eend = ex2_approx(c2end);
#pragma unroll
    for (int mi = 0; mi < 2; ++mi) {
      if (mi >= ntm) break;
      float sacc[8][4];
#pragma unroll
      for (int pj = 0; pj < 8; ++pj) sacc[pj][0] = sacc[pj][1] = sacc[pj][2] = sacc[pj][3] = 0.0f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        frag_a_t(a, bs, PN, n0 + 16 * mi, 16 * kk, lane);
#pragma unroll
        for (int pj = 0; pj < 8; pj += 2) {
          uint32_t bb[4];
          frag_b_t(bb, xs, kPitchP, 8 * pj, 16 * kk, lane);
          mma(sacc[pj], a, bb[0], bb[1]);
          mma(sacc[pj + 1], a, bb[2], bb[3]);
        }
      }
#pragma unroll
      for (int pj = 0; pj < 8; ++pj)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[mi][pj][e] = fmaf(eend, st[mi][pj][e], sacc[pj][e]);
    }
    store_state_copy();
    __syncthreads();   // state copy complete; x, B, C free for the next chunk
  }
  // final state
#pragma unroll
  for (int mi = 0; mi < 2; ++mi) {
    if (mi >= ntm) break;
#pragma unroll
    for (int pj = 0; pj < 8; ++pj)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int n = n0 + 16 * mi + g + (e >> 1) * 8, pp = 8 * pj + 2 * t4 + (e & 1);
        hglob[pp * N + n] = st[mi][pj][e];
      }
  }
}

// The conv state after a prompt: the last K raw inputs of every channel
// (older ones from the previous state when the prompt is shorter than K).
// Thread: one (sequence, channel).
__global__ void conv_state_update_kernel(const bf16* __restrict__ u, bf16* __restrict__ conv_state, int Bt, int L,
                                         int C, int zero_init) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int K = 4;
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i >= static_cast<long long>(Bt) * C) return;
  const int b = static_cast<int>(i / C), c = static_cast<int>(i % C);
  bf16* cs = conv_state + i * K;
  bf16 nw[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int t = L - K + k;
    if (t >= 0) nw[k] = u[(static_cast<long long>(b) * L + t) * C + c];
    else if (!zero_init) nw[k] = cs[K + t];
    else nw[k] = __float2bfloat16_rn(0.0f);
  }
#pragma unroll
  for (int k = 0; k < K; ++k) cs[k] = nw[k];
}

}  // namespace ssd
}  // namespace sambay
