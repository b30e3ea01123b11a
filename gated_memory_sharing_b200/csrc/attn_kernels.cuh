// Cross-attention decode over the single KV cache (bfloat16 I/O): the
// cross-decoder layers the GMU does not replace ("Decoder-Hybrid-Decoder
// Architecture for Efficient Reasoning with Long Generation", Paper-Notes
// page, 方法详解 > 整体框架: the cross-decoder alternates cross-attention over
// the KV cache the self-decoder wrote once with GMUs; 研究背景与动机: a
// cross-attention layer moves O(d_kv N) memory per decoded token, a GMU layer
// O(d_h)).
//
//   out[b, h] = sum_j softmax_j(scale q[b, h] . K[b, j, h / G]) V[b, j, h / G]
//
// q [B, Hq, dh], K and V [B, N, Hkv, dh] (token-major, heads interleaved),
// G = Hq / Hkv query heads per KV head (grouped-query attention).
//
// Split-KV decoding: CTA (split, KV head, sequence) owns a range of tokens;
// each of its 4 warps streams its own sub-range through a double-buffered
// cp.async ring of 32-token K and V tiles and keeps an online softmax (running
// max m and sum l, in base 2) and the unnormalised output O of the G query
// heads.  S = Q K^T and O += P V are m16n8k16 bf16 MMAs with fp32
// accumulation (the G <= 16 query heads are the MMA's 16 rows); P is rounded
// to bf16 for the second MMA.  The warps combine inside the CTA; with more
// than one split per (sequence, head) a second kernel combines the splits'
// (m, l, O).  Memory-bound: every K and V element is read once.
#pragma once

#include "common.cuh"

namespace sambay {
namespace attn {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kTile = 32;            // tokens per warp tile

struct AttnParams {
  const bf16* q;       // [B, Hq, dh]
  const bf16* K;       // [B, N, Hkv, dh]
  const bf16* V;       // [B, N, Hkv, dh]
  bf16* out;           // [B, Hq, dh]
  float* o_part;       // [B, Hq, splits, dh]   unnormalised partial outputs (splits > 1)
  float* ml_part;      // [B, Hq, splits, 2]    their (m, l), m in base 2
  int B, N, Hq, Hkv, G;
  int splits, chunk;   // tokens per split (a multiple of kTile)
  float scale_log2;    // scale * log2(e)
};

// Shared memory of one warp's tile stage: K rows at a pitch whose 8-byte
// fragment loads are conflict-free, V rows at a pitch whose ldmatrix rows are.
template <int DH>
struct AttnLayout {
  static constexpr int kPitchK = DH + 16;
  static constexpr int kPitchV = DH + 8;
  static constexpr int kStageBytes = kTile * (kPitchK + kPitchV) * 2;
  static constexpr int kWarpBytes = 2 * kStageBytes;
  static constexpr int kBytes = kWarps * kWarpBytes;
  // after the loop the area holds each warp's (m, l) and O of 16 rows
  static constexpr int kCombineBytes = kWarps * 16 * (DH + 2) * 4;
  static_assert(kCombineBytes <= kBytes, "combine area fits the tile stages");
};

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two 8x8 bf16 matrices, transposed: lanes 0-15 give the row addresses (rows
// of matrix 0, then of matrix 1); each thread receives the B fragment (k = 2t,
// 2t+1 of column g) of both.
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t& r0, uint32_t& r1, const void* row_addr) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(row_addr));
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(a));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// grid (splits, Hkv, B)
template <int DH>
__global__ void __launch_bounds__(kThreads) cross_attn_decode_kernel(const AttnParams p) {
  using Ly = AttnLayout<DH>;
  constexpr int KS = DH / 16;          // k-steps of S = Q K^T
  constexpr int ND = DH / 8;           // n-blocks of O
  constexpr int NB = kTile / 8;        // n-blocks of S (tokens)
  extern __shared__ __align__(16) uint8_t smem[];
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int n0 = split * p.chunk, n1 = min(p.N, n0 + p.chunk);
  // this warp's tiles: tile indices tw0, tw0 + kWarps, ... of the split's range
  const int ntiles = (n1 - n0 + kTile - 1) / kTile;
  const long long row_stride = static_cast<long long>(p.Hkv) * DH;   // elements between tokens
  const bf16* kbase = p.K + (static_cast<long long>(b) * p.N * p.Hkv + kvh) * DH;
  const bf16* vbase = p.V + (static_cast<long long>(b) * p.N * p.Hkv + kvh) * DH;
  uint8_t* wsm = smem + warp * Ly::kWarpBytes;

  // Q fragments (rows: the group's query heads g and g + 8, zero past G),
  // columns permuted as logical (2t, 2t+1, 2t+8, 2t+9) -> physical 4t .. 4t+3
  uint32_t qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = g + 8 * half;
      uint2 v = make_uint2(0u, 0u);
      if (r < p.G)
        v = *reinterpret_cast<const uint2*>(p.q + (static_cast<long long>(b) * p.Hq + kvh * p.G + r) * DH +
                                            ks * 16 + 4 * t);
      qa[ks][half] = v.x;
      qa[ks][2 + half] = v.y;
    }

  auto load_tile = [&](int tile, int st) {
    bf16* ks_ = reinterpret_cast<bf16*>(wsm + st * Ly::kStageBytes);
    bf16* vs_ = ks_ + kTile * Ly::kPitchK;
    const int tok0 = n0 + tile * kTile;
    // kTile tokens x DH / 8 chunks of 16 bytes for K and V; tokens past n1 read token n1 - 1
#pragma unroll
    for (int i = lane; i < kTile * DH / 8; i += 32) {
      const int r = i / (DH / 8), c = (i % (DH / 8)) * 8;
      const int tok = min(tok0 + r, n1 - 1);
      cp_async16(ks_ + r * Ly::kPitchK + c, kbase + tok * row_stride + c);
      cp_async16(vs_ + r * Ly::kPitchV + c, vbase + tok * row_stride + c);
    }
  };

  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float o[ND][4];
#pragma unroll
  for (int nd = 0; nd < ND; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.0f;

  int st = 0;
  if (warp < ntiles) load_tile(warp, 0);
  cp_async_commit();
  for (int tile = warp; tile < ntiles; tile += kWarps) {
    if (tile + kWarps < ntiles) load_tile(tile + kWarps, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncwarp();
    const bf16* ks_ = reinterpret_cast<const bf16*>(wsm + st * Ly::kStageBytes);
    const bf16* vs_ = ks_ + kTile * Ly::kPitchK;
    const int tok0 = n0 + tile * kTile;
    // S = Q K^T for the tile's kTile tokens, in base-2 logits
    float s[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.0f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const uint2 kb = *reinterpret_cast<const uint2*>(ks_ + (8 * nb + g) * Ly::kPitchK + ks * 16 + 4 * t);
        mma16816(s[nb], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], kb.x, kb.y);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = tok0 + 8 * nb + 2 * t + (e & 1);
        s[nb][e] = tok < n1 ? s[nb][e] * p.scale_log2 : -INFINITY;
      }
    }
    // online softmax per row (rows g: entries 0, 1; rows g + 8: entries 2, 3)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      mx[0] = fmaxf(mx[0], fmaxf(s[nb][0], s[nb][1]));
      mx[1] = fmaxf(mx[1], fmaxf(s[nb][2], s[nb][3]));
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float corr[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float mn = fmaxf(m[r], mx[r]);          // finite: every tile holds a live token
      corr[r] = ex2_approx(m[r] - mn);              // 0 on the first tile (m = -inf)
      m[r] = mn;
      l[r] *= corr[r];
    }
#pragma unroll
    for (int nd = 0; nd < ND; ++nd) {
      o[nd][0] *= corr[0]; o[nd][1] *= corr[0];
      o[nd][2] *= corr[1]; o[nd][3] *= corr[1];
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      s[nb][0] = ex2_approx(s[nb][0] - m[0]);
      s[nb][1] = ex2_approx(s[nb][1] - m[0]);
      s[nb][2] = ex2_approx(s[nb][2] - m[1]);
      s[nb][3] = ex2_approx(s[nb][3] - m[1]);
      l[0] += s[nb][0] + s[nb][1];
      l[1] += s[nb][2] + s[nb][3];
    }
    // O += P V: P's accumulator layout is the A fragment of k-step kk (tokens
    // 16 kk .. +15): n-blocks 2 kk and 2 kk + 1
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk) {
      const uint32_t a0 = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      const uint32_t a1 = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      const uint32_t a2 = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      const uint32_t a3 = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nd = 0; nd < ND; ++nd) {
        uint32_t b0, b1;
        ldmatrix_x2_trans(b0, b1, vs_ + (16 * kk + (lane & 15)) * Ly::kPitchV + 8 * nd);
        mma16816(o[nd], a0, a1, a2, a3, b0, b1);
      }
    }
    __syncwarp();              // stage st is read; the next iteration's load may refill it
    st ^= 1;
  }
  cp_async_wait<0>();
  // the row sums over the quad's lanes
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
  }
  __syncthreads();             // every warp is done with its tile stages
  // each warp's (m, l) and O rows into shared memory: [warp][row][DH + 2]
  float* cw = reinterpret_cast<float*>(smem) + warp * 16 * (DH + 2);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = g + 8 * r;
#pragma unroll
    for (int nd = 0; nd < ND; ++nd) {
      cw[row * (DH + 2) + 8 * nd + 2 * t] = o[nd][2 * r];
      cw[row * (DH + 2) + 8 * nd + 2 * t + 1] = o[nd][2 * r + 1];
    }
    if (t == 0) {
      cw[row * (DH + 2) + DH] = m[r];
      cw[row * (DH + 2) + DH + 1] = l[r];
    }
  }
  __syncthreads();
  // combine the warps (in warp order): thread -> (row, column)
  const float* cb = reinterpret_cast<const float*>(smem);
  for (int i = threadIdx.x; i < p.G * DH; i += kThreads) {
    const int row = i / DH, c = i % DH;
    float mstar = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mstar = fmaxf(mstar, cb[(w * 16 + row) * (DH + 2) + DH]);
    float num = 0.0f, den = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = cb[(w * 16 + row) * (DH + 2) + DH];
      const float f = mw == -INFINITY ? 0.0f : ex2_approx(mw - mstar);   // a warp without tokens
      num += f * cb[(w * 16 + row) * (DH + 2) + c];
      den += f * cb[(w * 16 + row) * (DH + 2) + DH + 1];
    }
    const long long qh = static_cast<long long>(b) * p.Hq + kvh * p.G + row;
    if (p.splits == 1) {
      p.out[qh * DH + c] = __float2bfloat16_rn(num / den);
    } else {
      p.o_part[(qh * p.splits + split) * DH + c] = num;
      if (c == 0) {
        p.ml_part[(qh * p.splits + split) * 2] = mstar;
        p.ml_part[(qh * p.splits + split) * 2 + 1] = den;
      }
    }
  }
}

// out[b, h, c] from the splits' partials, combined in split order.  Thread:
// one output element.
template <int DH>
__global__ void __launch_bounds__(256) cross_attn_combine_kernel(const AttnParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i >= static_cast<long long>(p.B) * p.Hq * DH) return;
  const long long qh = i / DH;
  const int c = static_cast<int>(i % DH);
  float mstar = -INFINITY;
  for (int sp = 0; sp < p.splits; ++sp) mstar = fmaxf(mstar, p.ml_part[(qh * p.splits + sp) * 2]);
  float num = 0.0f, den = 0.0f;
  for (int sp = 0; sp < p.splits; ++sp) {
    const float f = ex2_approx(p.ml_part[(qh * p.splits + sp) * 2] - mstar);
    num += f * p.o_part[(qh * p.splits + sp) * DH + c];
    den += f * p.ml_part[(qh * p.splits + sp) * 2 + 1];
  }
  p.out[i] = __float2bfloat16_rn(num / den);
}

}  // namespace attn
}  // namespace sambay
