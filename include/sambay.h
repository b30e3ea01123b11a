/*
 * sambay.h - C ABI of the SambaY scan + Gated Memory Unit hot path on B200
 * (sm_100a).  Exported by libsambay.so.
 *
 * The method (sources cited per entry point):
 *   [GMU]   "Decoder-Hybrid-Decoder Architecture for Efficient Reasoning with
 *           Long Generation", Paper-Notes page, 方法详解 > 关键设计 (Gated Memory
 *           Unit): Y = (M ⊙ SiLU(X W1^T)) W2, where M is the token-mixing output
 *           of the self-decoder's last SSM layer, and decoding keeps a
 *           constant-size recurrent state.
 *   [FRAME] same page, 方法详解 > 整体框架: prefill runs only the self-decoder
 *           (linear in length); the cross-decoder's GMU layers reuse M; a GMU
 *           layer moves O(d_h) memory per decoded token.
 *   [ABS]   the paper's abstract (chatpaper.ai page, English abstract): GMUs
 *           share the "memory readout states" of the Samba self-decoder.
 *   [MAMBA] the selective SSM producing M (Gu & Dao 2023, "Mamba", section
 *           3.2 and Algorithm 2; block of section 3.4): causal depthwise
 *           conv + SiLU, x_proj -> (delta, B, C), dt = softplus(delta W_dt^T +
 *           b_dt), h_t = exp(dt A) h_{t-1} + dt B_t u_t, y_t = C_t h_t + D u_t.
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers, caller-owned, row-major and
 *     densely packed in the stated shape; the library allocates no device
 *     memory and keeps no state between calls.  Scratch memory is the
 *     caller's `ws` buffer of at least the queried size (256-byte aligned).
 *   - "io" is the I/O element type of the call (dims->io): SAMBAY_F32 (float)
 *     or SAMBAY_BF16 (bfloat16).  State, dt, B, C and every accumulation are
 *     float32 in both modes.  SAMBAY_F32 runs float32 CUDA-core kernels
 *     (no TF32); SAMBAY_BF16 runs the tcgen05 tensor-core kernels.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronise, except sambay_device_status.
 *     A call's first kernel orders after everything queued before it on the
 *     stream; its later kernels use programmatic dependent launch, starting
 *     while the previous kernel of the same call finishes and waiting for it
 *     before they touch memory.
 *   - Argument errors (NULL pointers, bad or unsupported sizes, misaligned
 *     pointers, short workspace) are detected on the host BEFORE any launch,
 *     and return a status without touching the device.  Launch failures
 *     return SAMBAY_ERR_CUDA.  Faults found by a kernel while running (a
 *     bounded wait that ran out) are recorded in a per-device status word
 *     that sambay_device_status reads and clears.
 *   - Supported sizes: d_state == 16, d_conv == 4, dt_rank a multiple of 4
 *     with dt_rank + 2*d_state <= 256, d_inner a multiple of 32 (scan) or 4
 *     (GMU), d_model a multiple of 4; in SAMBAY_BF16 mode d_inner and d_model
 *     are multiples of 64 and dt_rank a multiple of 8 (16-byte rows for TMA).
 *     batch, seqlen, rows >= 1; gmu_step rows <= 256.  Device pointers must
 *     be 16-byte aligned (ws: 256-byte).  Anything else returns
 *     SAMBAY_ERR_UNSUPPORTED (SAMBAY_ERR_INVALID_ARG for values < 1).
 */
#ifndef SAMBAY_H_
#define SAMBAY_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SAMBAY_API __attribute__((visibility("default")))
#else
#define SAMBAY_API
#endif

typedef struct CUstream_st* sambay_stream_t; /* == cudaStream_t */

typedef enum {
  SAMBAY_OK = 0,
  SAMBAY_ERR_INVALID_ARG = 1, /* NULL pointer, non-positive size, bad enum    */
  SAMBAY_ERR_UNSUPPORTED = 2, /* valid but outside the supported sizes above  */
  SAMBAY_ERR_WORKSPACE = 3,   /* ws NULL/misaligned or ws_bytes too small     */
  SAMBAY_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed            */
  SAMBAY_ERR_TIMEOUT = 5,     /* a kernel's bounded wait ran out (device word) */
  SAMBAY_ERR_DEVICE = 6       /* no sm_100 device current                     */
} sambay_status;

typedef enum { SAMBAY_F32 = 0, SAMBAY_BF16 = 1 } sambay_dtype;

/* Sizes.  B batch, L seqlen, Dm d_model, Di d_inner, N d_state, K d_conv,
 * R dt_rank.  T = B*L tokens. */
typedef struct {
  int32_t batch;
  int32_t seqlen;
  int32_t d_model;
  int32_t d_inner;
  int32_t d_state;
  int32_t d_conv;
  int32_t dt_rank;
  int32_t io; /* sambay_dtype */
} sambay_dims;

/* Weights of the Mamba layer whose readout is M [MAMBA].  Device pointers. */
typedef struct {
  const void* conv_w;    /* [Di, K] io   depthwise causal conv taps; tap K-1
                            multiplies the current token (cross-correlation) */
  const void* conv_b;    /* [Di]    io   conv bias                           */
  const void* x_proj_w;  /* [R+2N, Di] io rows [0,R): delta, [R,R+N): B,
                            [R+N,R+2N): C                                    */
  const void* dt_proj_w; /* [Di, R] io                                       */
  const float* dt_bias;  /* [Di]    f32                                      */
  const float* A;        /* [Di, N] f32  (negative; the decay is exp(dt*A))  */
  const float* D;        /* [Di]    f32  skip weight                         */
} sambay_scan_weights;

/* ---------------------------------------------------------------------- */
/* Workspace queries: bytes of caller-provided scratch each call needs.    */
/* 0 on invalid dims.  Sizes depend only on the arguments.                 */
/* ---------------------------------------------------------------------- */
SAMBAY_API size_t sambay_scan_prefill_workspace(const sambay_dims* dims);
SAMBAY_API size_t sambay_scan_step_workspace(const sambay_dims* dims);
SAMBAY_API size_t gmu_forward_workspace(const sambay_dims* dims, int64_t rows);
SAMBAY_API size_t gmu_step_workspace(const sambay_dims* dims, int64_t rows);

/*
 * sambay_scan_prefill - one Mamba selective scan over a prompt, writing the
 * memory readout M and leaving the constant-size decode state [MAMBA],
 * [GMU] (M^(l') = the token-mixing output; decode state), [FRAME] (prefill
 * = self-decoder only), [ABS] ("memory readout states").
 *
 *   u          [B, L, Di] io  in   scan input (the in_proj x branch)
 *   M          [B, L, Di] io  out  y = C.h + D*uc, before any output gate,
 *                                  norm or out_proj.  Must not alias u.
 *   ssm_state  [B, Di, N] f32 in/out  h; read as h_0 unless zero_init_state,
 *                                  overwritten with h_L.
 *   conv_state [B, Di, K] io  in/out  the last K scan inputs, oldest first;
 *                                  read as left context unless
 *                                  zero_init_state (then zeros), overwritten
 *                                  with the last K inputs seen.
 *   zero_init_state  nonzero: fresh prompt (states treated as zero).
 *   ws, ws_bytes     scratch, >= sambay_scan_prefill_workspace(dims).
 * Steps: uc = SiLU(conv(u)); [delta|B|C] = uc W_x^T; dt = softplus(delta
 * W_dt^T + b_dt); the exp(dt A) recurrence with float32 h; readout.
 */
SAMBAY_API sambay_status sambay_scan_prefill(const sambay_scan_weights* w, const sambay_dims* dims,
                                  const void* u, void* M, float* ssm_state, void* conv_state,
                                  int zero_init_state, void* ws, size_t ws_bytes,
                                  sambay_stream_t stream);

/*
 * Channel-sharded prefill (one shard of d_inner per GPU).  The scan is
 * independent per channel except for x_proj, whose [delta | B | C] sums run
 * over all channels [MAMBA] (selection projections), so sambay_scan_prefill
 * splits there into two calls around the caller's sum over the shards (an
 * all-reduce of xdbl):
 *
 * sambay_scan_prefill_xproj - conv + SiLU and this shard's x_proj partial
 * sums.  dims->d_inner and the weights are the shard's (conv_w, conv_b,
 * x_proj_w [R + 2N, Di_shard], dt_proj_w [Di_shard, R], dt_bias, A, D of its
 * channels); u [B, L, Di_shard] io is its slice of the scan input.
 *   conv_state  [B, Di_shard, K] io  in (read only here; the left context
 *               unless zero_init_state).
 *   xdbl        [B*L, R + 2N] f32 out: sum over the shard's channels of
 *               uc * W_x^T (deterministic order).  Caller-owned, 16-byte
 *               aligned.
 *   ws          >= sambay_scan_prefill_workspace(dims); it carries the conv
 *               output to the second call and must be passed there unchanged.
 * sambay_scan_prefill_finish - given xdbl summed over all shards: delta, B,
 * C, dt_proj + softplus and the scan of the shard's channels; writes M
 * [B, L, Di_shard] and updates ssm_state / conv_state exactly as
 * sambay_scan_prefill does.  u, conv_state, zero_init_state and ws as in the
 * first call.  With one shard the pair computes what sambay_scan_prefill
 * computes.
 */
SAMBAY_API sambay_status sambay_scan_prefill_xproj(const sambay_scan_weights* w, const sambay_dims* dims,
                                        const void* u, const void* conv_state, int zero_init_state,
                                        float* xdbl, void* ws, size_t ws_bytes, sambay_stream_t stream);
SAMBAY_API sambay_status sambay_scan_prefill_finish(const sambay_scan_weights* w, const sambay_dims* dims,
                                         const void* u, const float* xdbl, void* M, float* ssm_state,
                                         void* conv_state, int zero_init_state, void* ws,
                                         size_t ws_bytes, sambay_stream_t stream);

/*
 * sambay_scan_step - one decode token per sequence: the prefill with L = 1
 * on the carried state, updating ssm_state and conv_state IN PLACE [GMU]
 * (constant-size state), [MAMBA].  dims->seqlen is ignored.  In SAMBAY_BF16
 * mode the work is cut into channel slices (about one slice of up to 48
 * channels per SM).  Up to 64 sequences it is ONE cooperative kernel, one CTA
 * per slice, all resident at once: conv + the slice's partial x_proj sums,
 * a grid-wide meeting point, each CTA's share of the sums over slices (a
 * fixed order), a second meeting point, dt_proj + the state update; the
 * slice's state arrives by one tensor copy issued after the conv.  Above 64
 * sequences (or where the slices do not fit the GPU at one CTA per SM) it is
 * three kernels with the same stages, chained.  ws holds the conv output,
 * the partial sums, delta, B | C and the meeting points' words (a
 * generation word and two flags per slice, 128 bytes each; any contents are
 * accepted, and a call leaves them consistent for the next):
 *   B * (4 Di + 4 ceil(Di / chan) (R + 2N) + 4 R16 + 8 N) bytes + 128 *
 *   (1 + 2 ceil(Di / chan)) (R16 = R rounded up to 16), about 7.7 MB for 64
 *   sequences at d_inner 5120.  Calls that share a ws must not overlap on
 *   the GPU (the meeting words are per ws).  After a SAMBAY_ERR_TIMEOUT the
 *   ws's meeting words may be inconsistent: zero the ws before reusing it.
 * SAMBAY_F32 runs a chain of float32 kernels that exchange their
 * intermediates through ws.
 *
 *   u_t [B, Di] io in;  m_t [B, Di] io out (must not alias u_t);
 *   ssm_state [B, Di, N] f32 in/out;  conv_state [B, Di, K] io in/out.
 */
SAMBAY_API sambay_status sambay_scan_step(const sambay_scan_weights* w, const sambay_dims* dims,
                               const void* u_t, void* m_t, float* ssm_state, void* conv_state,
                               void* ws, size_t ws_bytes, sambay_stream_t stream);

/*
 * gmu_forward - Gated Memory Unit over `rows` tokens [GMU]:
 *     Y = (M ⊙ SiLU(X W1^T)) W2   (+ residual when residual != NULL)
 *
 *   X  [rows, Dm] io   W1 [Di, Dm] io (used as W1^T)   M [rows, Di] io
 *   W2 [Di, Dm] io (multiplies on the right: Di -> Dm)
 *   residual [rows, Dm] io or NULL;  Y [rows, Dm] io out (may alias
 *   residual, must not alias X unless X == residual, nor M).
 * Two tensor-core GEMMs: G = X W1^T with SiLU(G) ⊙ M fused into its
 * epilogue (H, io, kept in ws), then H W2 with the residual fused.  In bf16
 * with more than 256 rows, ws also holds the fp32 partial tiles of a GEMM
 * whose last round of tiles is split along K, and flags marking their
 * arrival; the same kernel sums them in a fixed order, so results do not
 * vary from run to run.  ws needs no initialisation, but two calls in flight
 * at once must not share it.
 */
SAMBAY_API sambay_status gmu_forward(const sambay_dims* dims, int64_t rows, const void* X, const void* M,
                          const void* W1, const void* W2, const void* residual, void* Y,
                          void* ws, size_t ws_bytes, sambay_stream_t stream);

/*
 * gmu_forward_partial - the GMU of one d_inner shard [GMU]: H = M ⊙ SiLU(X
 * W1^T) over the shard's channels (W1 [Di_shard, Dm], M [rows, Di_shard]),
 * then Y_part = H W2 (W2 [Di_shard, Dm], the shard's rows) as float32
 * [rows, Dm], with no residual.  The sum of Y_part over the shards (an
 * all-reduce) is Y before the residual; gmu_finish completes it.  ws:
 * >= gmu_forward_workspace(dims, rows) (dims->d_inner = the shard's).
 *
 * gmu_finish - Y = io(Y_sum + residual) (residual [rows, Dm] io or NULL;
 * Y [rows, Dm] io, may alias residual, not Y_sum).
 */
SAMBAY_API sambay_status gmu_forward_partial(const sambay_dims* dims, int64_t rows, const void* X,
                                  const void* M, const void* W1, const void* W2, float* Y_part,
                                  void* ws, size_t ws_bytes, sambay_stream_t stream);
SAMBAY_API sambay_status gmu_finish(const sambay_dims* dims, int64_t rows, const float* Y_sum,
                         const void* residual, void* Y, sambay_stream_t stream);

/*
 * gmu_step - the GMU for one decode token of `rows` sequences (rows <= 256)
 * [GMU], [FRAME] (O(d_h) memory per token: the weights are streamed once).
 * Same arguments and semantics as gmu_forward; a weight-streaming kernel
 * pair (swap-AB tensor-core GEMV with split-K over a cluster of CTAs, the
 * splits summed in a fixed order through distributed shared memory) instead
 * of the tiled GEMMs; ws holds only H.
 */
SAMBAY_API sambay_status gmu_step(const sambay_dims* dims, int64_t rows, const void* X, const void* M,
                       const void* W1, const void* W2, const void* residual, void* Y,
                       void* ws, size_t ws_bytes, sambay_stream_t stream);

/*
 * sambay_in_proj - the scan branch of the Mamba block's input projection
 * [MAMBA] section 3.4: u = X W_in^T, the input of sambay_scan_prefill /
 * sambay_scan_step.  With it the whole Mamba layer whose readout is the
 * memory M runs from its input X [FRAME] (the Samba self-decoder's SSM
 * layers):
 *     u = sambay_in_proj(X, W_in);   M = sambay_scan_prefill(u)  (pre-gate y)
 *     out = gmu_forward(X, M, W_z, W_out, residual = X)
 * since the block's gated output (y ⊙ SiLU(X W_z^T)) W_out is the GMU's
 * computation with W1 = W_z (the z half of in_proj) and W2 = W_out (out_proj's
 * weight, [Di, Dm], multiplying on the right).
 *
 *   X [rows, Dm] io;  W_in [Di, Dm] io (used transposed);  u [rows, Di] io out
 *   (must not alias X).  ws: >= sambay_in_proj_workspace(dims, rows) (the
 *   K-split tail partials of a bf16 GEMM of more than 256 rows and their
 *   arrival flags; else 0), no initialisation needed, not shared by two calls
 *   in flight at once.
 * Up to 256 rows (decode) W_in streams once through the swap-AB decode GEMM.
 */
SAMBAY_API size_t sambay_in_proj_workspace(const sambay_dims* dims, int64_t rows);
SAMBAY_API sambay_status sambay_in_proj(const sambay_dims* dims, int64_t rows, const void* X,
                                        const void* W_in, void* u, void* ws, size_t ws_bytes,
                                        sambay_stream_t stream);

/*
 * sambay_mlp_memory - the memory of SambaY-MLP ([Notes] 实验关键数据 >
 * 消融实验, row SambaY-MLP: the GMUs gate an MLP representation instead of the
 * SSM readout): the hidden activation of a SwiGLU MLP,
 *     M = SiLU(X W_g^T) ⊙ (X W_u^T),
 * which gmu_forward / gmu_step then take in place of the scan readout.
 * dims->d_inner is the MLP width Dff, dims->d_model the input width.
 *
 *   X [rows, Dm] io;  W_g, W_u [Dff, Dm] io (used transposed);
 *   M [rows, Dff] io out (must not alias X);
 *   ws: >= sambay_mlp_memory_workspace(dims, rows) (X W_u^T, then the K-split
 *   tail partials as in sambay_in_proj).
 * Two tensor-core GEMMs: X W_u^T, then X W_g^T with SiLU and the product with
 * X W_u^T fused into its epilogue (the GMU gate GEMM's epilogue).
 */
SAMBAY_API size_t sambay_mlp_memory_workspace(const sambay_dims* dims, int64_t rows);
SAMBAY_API sambay_status sambay_mlp_memory(const sambay_dims* dims, int64_t rows, const void* X,
                                           const void* W_g, const void* W_u, void* M, void* ws,
                                           size_t ws_bytes, sambay_stream_t stream);

/* Weights of one Gated Memory Unit layer (device pointers, [Di, Dm] io each). */
typedef struct {
  const void* W1; /* used as W1^T: X W1^T maps Dm -> Di   */
  const void* W2; /* multiplies on the right: Di -> Dm    */
} sambay_gmu_weights;

/*
 * sambay_decode_step - one decode token of every sequence through the shared
 * memory and the cross-decoder layers that reuse it [GMU], [FRAME]:
 *     m_t = sambay_scan_step(u_t)                    (states updated in place)
 *     for l in 0 .. n_layers-1:  X <- X + GMU_l(X, m_t)   (in place)
 * i.e. sambay_scan_step followed by n_layers gmu_step calls with
 * residual == Y == X, issued as one chain of kernels: each kernel after the
 * first starts while its predecessor finishes (programmatic dependent launch)
 * and loads its weights before waiting for it; layer 0's gate GEMM, whose
 * inputs (X, W1) the scan step does not write, runs its whole main loop before
 * waiting and only its epilogue (which reads m_t) waits.  Results are the
 * same bits as the separate calls.
 *
 *   u_t [B, Di] io in;  m_t [B, Di] io out;  ssm_state, conv_state in/out as in
 *   sambay_scan_step;  layers: HOST array of n_layers weight pairs;
 *   X [B, Dm] io in/out (not used when n_layers == 0; must not alias u_t, m_t);
 *   ws, ws_bytes: >= sambay_decode_step_workspace(dims, n_layers).
 * B <= 256.  dims->seqlen is ignored; dims->d_model is the GMU width.
 */
SAMBAY_API size_t sambay_decode_step_workspace(const sambay_dims* dims, int32_t n_layers);
SAMBAY_API sambay_status sambay_decode_step(const sambay_scan_weights* w, const sambay_dims* dims,
                                            const void* u_t, void* m_t, float* ssm_state,
                                            void* conv_state, int32_t n_layers,
                                            const sambay_gmu_weights* layers, void* X, void* ws,
                                            size_t ws_bytes, sambay_stream_t stream);

/*
 * sambay_gmu_step_stall_test - a test of the fault detector; the paper has no
 * counterpart.  Runs gmu_step (bf16 only) with one change: before its first
 * accumulator, each tensor-core kernel's epilogue waits on a barrier that
 * nothing arrives at, with every bounded wait limited to wait_limit_cycles
 * (1 .. 2^32) clock cycles.  That wait therefore runs out: the kernels record
 * SAMBAY_ERR_TIMEOUT in the device status word, stop their loads and MMAs,
 * drain what is in flight (itself bounded), free their tensor memory and
 * return.  Y is unspecified afterwards; sambay_device_status reports the
 * timeout, and the device stays usable.  Nothing faults, traps or hangs.
 */
SAMBAY_API sambay_status sambay_gmu_step_stall_test(const sambay_dims* dims, int64_t rows, const void* X,
                                                    const void* M, const void* W1, const void* W2,
                                                    const void* residual, void* Y, void* ws,
                                                    size_t ws_bytes, uint64_t wait_limit_cycles,
                                                    sambay_stream_t stream);

/* Sizes of a cross-attention decode.  Tensors are bfloat16. */
typedef struct {
  int32_t batch;      /* B sequences, one query token each                  */
  int32_t kv_len;     /* N cached tokens per sequence                        */
  int32_t q_heads;    /* Hq query heads                                      */
  int32_t kv_heads;   /* Hkv key/value heads; Hq / Hkv <= 16 share one       */
  int32_t head_dim;   /* dh: 64 or 128                                       */
} sambay_attn_dims;

/*
 * sambay_cross_attn_decode - one decoded token per sequence attending over
 * the single KV cache that the self-decoder's full-attention layer wrote once
 * [FRAME] (the cross-decoder's cross-attention layers, the ones the GMU does
 * not replace), i.e. the O(d_kv N) memory-per-token counterpart of gmu_step's
 * O(d_h):
 *     out[b, h] = sum_j softmax_j(scale q[b, h] . K[b, j, h / G]) V[b, j, h / G]
 * with G = Hq / Hkv (consecutive query heads share a KV head).
 *
 *   q [B, Hq, dh], K and V [B, N, Hkv, dh] (token-major), out [B, Hq, dh],
 *   all bf16 (out must not alias the inputs); scale > 0, or 0 for
 *   1 / sqrt(dh).  ws: >= sambay_cross_attn_decode_workspace(dims) (the
 *   partial outputs of a KV range split over several CTAs; 0 when the
 *   sequences and heads alone fill the GPU).
 * Split-KV: each CTA streams a range of one (sequence, KV head)'s tokens
 * once, with an online softmax and fp32 accumulation; ranges are combined in
 * a fixed order.
 */
SAMBAY_API size_t sambay_cross_attn_decode_workspace(const sambay_attn_dims* dims);
SAMBAY_API sambay_status sambay_cross_attn_decode(const sambay_attn_dims* dims, const void* q,
                                                  const void* K, const void* V, void* out, float scale,
                                                  void* ws, size_t ws_bytes, sambay_stream_t stream);

/* ---------------------------------------------------------------------- */
/* SambaY-2: the memory readout of a Mamba-2 (SSD) layer                    */
/* ---------------------------------------------------------------------- */

/* Sizes of the Mamba-2 layer whose readout is M in the SambaY-2 variant
 * ("Decoder-Hybrid-Decoder Architecture ...", Paper-Notes page, 实验关键数据 >
 * 消融实验, row SambaY-2: Mamba replaced by Mamba-2, a scalar forget gate per
 * head).  One group: B and C are shared by all heads. */
typedef struct {
  int32_t batch;     /* Bt sequences                                        */
  int32_t seqlen;    /* L tokens                                            */
  int32_t nheads;    /* H heads; d_inner = H * headdim                       */
  int32_t headdim;   /* P: 64                                               */
  int32_t d_state;   /* N: 64 or 128                                        */
  int32_t d_conv;    /* K: 4                                                */
  int32_t io;        /* sambay_dtype: SAMBAY_BF16                           */
} sambay_ssd_dims;

/* Device pointers.  C = H * P + 2 N conv channels ([x | B | C]). */
typedef struct {
  const void* conv_w;    /* [C, K] io   depthwise causal conv taps (tap K-1 on
                            the current token)                              */
  const void* conv_b;    /* [C]    io                                       */
  const float* dt_bias;  /* [H]    f32  dt = softplus(dt_raw + dt_bias)      */
  const float* A;        /* [H]    f32  negative; decay exp(dt A) per head   */
  const float* D;        /* [H]    f32  skip weight                         */
} sambay_ssd_weights;

/*
 * sambay_ssd_prefill - the SambaY-2 memory M of a prompt: the causal conv +
 * SiLU of the in_proj slice [x | B | C], dt = softplus(dt_raw + dt_bias), and
 * the SSD recurrence of Mamba-2 (Dao & Gu 2024, "Transformers are SSMs"):
 *     H_t = exp(dt_t A_h) H_{t-1} + dt_t x_t B_t^T,   y_t = H_t C_t + D_h x_t
 * per head h (x_t, y_t in R^P, H in R^{P x N}), M = y.  Computed chunk by
 * chunk (64 tokens) on the tensor cores: per chunk and head the products
 * C B^T, (masked, decay-scaled) W X, C H and (B scaled)^T X, with the fp32
 * state carried across chunks; operands bf16, accumulation fp32.
 *
 *   xbc [Bt, L, C] io in;  dt_raw [Bt, L, H] io in;  M [Bt, L, H*P] io out;
 *   ssm_state [Bt, H, P, N] f32 in/out (read unless zero_init);
 *   conv_state [Bt, C, K] io in/out (the left context unless zero_init; the
 *   last K inputs on return).  io must be SAMBAY_BF16, P = 64, N in {64,
 *   128}, K = 4, C a multiple of 32; other sizes return
 *   SAMBAY_ERR_UNSUPPORTED.  M must not alias xbc.
 *   ws: >= sambay_ssd_prefill_workspace(dims): the conv output as a bf16
 *   split pair, Bt * L * C * 4 bytes.
 */
SAMBAY_API size_t sambay_ssd_prefill_workspace(const sambay_ssd_dims* dims);
SAMBAY_API sambay_status sambay_ssd_prefill(const sambay_ssd_weights* w, const sambay_ssd_dims* dims,
                                            const void* xbc, const void* dt_raw, void* M, float* ssm_state,
                                            void* conv_state, int32_t zero_init, void* ws, size_t ws_bytes,
                                            sambay_stream_t stream);

/*
 * sambay_ssd_step - one decode token per sequence of the SambaY-2 memory:
 * the prompt readout with L = 1 on the carried states, both updated IN
 * PLACE (the conv window shifted, the SSD state advanced).  Two kernels: the
 * conv step over [x | B | C] (fp32 output in ws), then the state update per
 * (head, sequence).  dims->seqlen is ignored.
 *
 *   xbc_t [Bt, C] io in;  dt_raw_t [Bt, H] io in;  m_t [Bt, H*P] io out
 *   (must not alias xbc_t);  ssm_state [Bt, H, P, N] f32 in/out;
 *   conv_state [Bt, C, K] io in/out.  Sizes as for sambay_ssd_prefill.
 *   ws: >= sambay_ssd_step_workspace(dims) = Bt * C * 4 bytes (rounded).
 */
SAMBAY_API size_t sambay_ssd_step_workspace(const sambay_ssd_dims* dims);
SAMBAY_API sambay_status sambay_ssd_step(const sambay_ssd_weights* w, const sambay_ssd_dims* dims,
                                         const void* xbc_t, const void* dt_raw_t, void* m_t, float* ssm_state,
                                         void* conv_state, void* ws, size_t ws_bytes, sambay_stream_t stream);

/*
 * sambay_scan_step_noalloc - sambay_scan_step for callers that cannot
 * allocate device memory.  The paper has no counterpart; this is a property
 * of the library, not of the method.
 *
 * Some callers have no way to provide the `ws` buffer: a decode loop inside
 * a serving engine whose memory is planned up front and that forbids
 * allocation on the per-token path, or a plugin host that hands the library
 * only its input and output pointers.  This variant takes the same
 * arguments as sambay_scan_step minus the workspace and computes the same
 * result with the same kernels; its scratch is a fixed array compiled into
 * the library (SAMBAY_NOALLOC_SCRATCH_BYTES per GPU, held by every GPU that
 * loads the library until the process exits).  It allocates nothing.
 *
 *   - The scratch it needs is what sambay_scan_step_workspace(dims) reports
 *     (see sambay_scan_step): about 7.7 MB for 64 bf16 sequences at d_inner
 *     5120, and for SAMBAY_F32 about B * (2 * Di + R + 2N) * 4 bytes.
 *     The bf16 step's meeting words (see sambay_scan_step) live in that
 *     array too; after a SAMBAY_ERR_TIMEOUT from this entry point they may
 *     be inconsistent until the process restarts.
 *     Sizes whose sambay_scan_step_workspace(dims) exceeds
 *     SAMBAY_NOALLOC_SCRATCH_BYTES are rejected with SAMBAY_ERR_UNSUPPORTED
 *     before any launch; check that query against the limit before relying
 *     on this entry point for a size.
 *   - The first call on each device looks up the array's device address on
 *     that device (so that device must be current); make that first call
 *     before any stream capture.  The address is cached per device and not
 *     looked up again, so it is stale after cudaDeviceReset: do not use this
 *     entry point across a reset in one process.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; nothing in it needs to start at zero.  Calls that overlap on
 *     the GPU (different streams, or host threads without ordering) race on
 *     it and give wrong results: order them.
 */
#define SAMBAY_NOALLOC_SCRATCH_BYTES (8u << 20)

SAMBAY_API sambay_status sambay_scan_step_noalloc(const sambay_scan_weights* w,
                                                  const sambay_dims* dims, const void* u_t,
                                                  void* m_t, float* ssm_state, void* conv_state,
                                                  sambay_stream_t stream);

/*
 * sambay_profile_begin / sambay_profile_end - per-kernel timing for
 * measurement; the paper has no counterpart.  Between the two calls, on the
 * calling thread, the i-th kernel the library launches is bracketed by
 * cudaEventRecord(events[2i]) and cudaEventRecord(events[2i+1]) on its stream
 * (events: caller-created cudaEvent_t handles, `capacity` of them; launches
 * beyond capacity/2 are not recorded).  sambay_profile_end closes the session,
 * writes up to max_names static kernel names (launch order) to `names` and
 * returns the number of launches recorded.  Host bookkeeping only: nothing is
 * synchronised or allocated on the device.
 */
SAMBAY_API sambay_status sambay_profile_begin(void* const* events, int32_t capacity);
SAMBAY_API int32_t sambay_profile_end(const char** names, int32_t max_names);

/*
 * sambay_device_status - synchronise `stream`, then read and clear the
 * current device's status word.  *out_code receives the sambay_status a
 * kernel recorded (SAMBAY_OK if none).  Returns SAMBAY_ERR_CUDA if the
 * synchronisation itself failed.
 */
SAMBAY_API sambay_status sambay_device_status(sambay_stream_t stream, int32_t* out_code);

/* Static, human-readable name of a status code. */
SAMBAY_API const char* sambay_status_string(sambay_status status);

/* Library version, "major.minor.patch". */
SAMBAY_API const char* sambay_version(void);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* SAMBAY_H_ */
