/*
 * libsana — C ABI of the SANA-Video 2.0 hybrid linear-softmax attention hot path
 * on NVIDIA B200 (sm_100a).
 *
 * Operations (cited by page title and section / equation):
 *   [SV1]  "SANA-Video: Efficient Video Generation with Block Linear Diffusion
 *          Transformer" (paper notes): sec. 3.2 "Linear Attention with RoPE"
 *          (equation for O_i, linear-attention-with-RoPE pseudocode), sec. 3.4
 *          "Block Linear Attention with Constant-Memory KV Cache" (causal
 *          equation for O_i, cumulative state, Algorithm 1).
 *   [SV2]  "SANA-Video 2.0" (hyper.ai summary), Method: hybrid attention and
 *          block residuals, the AttnRes equation; shared router queries.
 *   [SV2a] "SANA-Video 2.0" abstract: gated linear attention and gated softmax
 *          anchors at a 3:1 ratio.
 *
 * Conventions shared by every entry point:
 *   - Tensors are row-major.  Token tensors are (B, N, C) with C = heads * D,
 *     i.e. (B, N, heads, D) with D contiguous ([SV1] sec. 3.2 pseudocode
 *     layout).  Token n of a latent grid (T, H, W) is n = (t*H + h)*W + w.
 *   - Every pointer argument named "device" is CUDA device memory owned by the
 *     caller; the library allocates no device memory and keeps no state between
 *     calls except a thread-local error string and one device status word.
 *   - Device pointers must be 16-byte aligned; outputs must not alias inputs
 *     (SANA_ERR_INVALID_ARG otherwise).
 *   - bf16 tensors use D = 128 (tcgen05 tensor-core path); fp32 tensors accept
 *     D in {16, 32, 64, 128} (FFMA path).  Other D: SANA_ERR_UNSUPPORTED.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously.  Argument errors are returned before
 *     anything is enqueued; launch errors return SANA_ERR_CUDA.  A kernel that
 *     detects a fault (a bounded wait that ran out) records it in the device
 *     status word, which sana_sync_status() reports as SANA_ERR_TIMEOUT.
 *   - On any non-OK status, sana_last_error_string() describes the cause.
 */
#ifndef SANA_H_
#define SANA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SANA_API __attribute__((visibility("default")))
#else
#define SANA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sana_stream_t; /* == cudaStream_t */

typedef enum {
  SANA_OK = 0,
  SANA_ERR_INVALID_ARG = 1,
  SANA_ERR_UNSUPPORTED = 2,
  SANA_ERR_WORKSPACE = 3,
  SANA_ERR_CUDA = 4,
  SANA_ERR_TIMEOUT = 5
} sana_status;

typedef enum { SANA_F32 = 0, SANA_BF16 = 1 } sana_dtype;

/* Latent token grid of one call.  N = T*H*W tokens per batch entry.
 * t_offset is the absolute index of the first frame (block-causal chunks use
 * absolute frame positions for RoPE); 0 for whole clips. */
typedef struct {
  int B, T, H, W;
  int heads, head_dim;
  int t_offset;
} sana_shape;

/* 3D RoPE tables ([SV1] sec. 3.2, RoPE applied after the ReLU; layout reading:
 * rotary pair j rotates elements (2j, 2j+1) of a head; pairs [0, n_t) follow
 * the absolute frame index, the next n_h the row, the last n_w the column;
 * n_t + n_h + n_w == head_dim / 2).  Device fp32 arrays, row-major:
 * cos_t/sin_t [T_total][n_t], cos_h/sin_h [H][n_h], cos_w/sin_w [W][n_w]. */
typedef struct {
  const float *cos_t, *sin_t, *cos_h, *sin_h, *cos_w, *sin_w;
  int n_t, n_h, n_w;
  int T_total, H, W;
} sana_rope;

/* Number of floats sana_rope_tables_host() writes:
 * 2*(T_total*n_t + H*n_h + W*n_w). */
SANA_API size_t sana_rope_tables_count(int T_total, int H, int W, int n_t, int n_h, int n_w);

/* Fill a HOST buffer with the six tables, in the order cos_t, sin_t, cos_h,
 * sin_h, cos_w, sin_w; angle(pos, local pair k of an axis with n pairs) =
 * pos * theta^(-k/n), evaluated in double and rounded to float.
 * Errors: SANA_ERR_INVALID_ARG on a NULL buffer or negative sizes. */
SANA_API sana_status sana_rope_tables_host(int T_total, int H, int W, int n_t, int n_h, int n_w,
                                  double theta, float* out_tables_host);

/* Point a sana_rope at a DEVICE copy of the buffer sana_rope_tables_host()
 * filled (pointer arithmetic only; nothing is read). */
SANA_API sana_status sana_rope_bind(const float* tables_device, int T_total, int H, int W,
                           int n_t, int n_h, int n_w, sana_rope* out);

/* ---------------------------------------------------------------------------
 * Gated bidirectional ReLU linear attention with RoPE after the ReLU
 * ([SV1] sec. 3.2):
 *   S = sum_j RoPE(phi K_j)^T V_j,  z = sum_j phi K_j,  phi = ReLU,
 *   O_i = RoPE(phi Q_i) S / (phi Q_i . z + eps),  Y_i = sigmoid(G_i) * O_i.
 * q, k, v, gate_logits, out: device (B, N, C) in `dtype`; gate_logits may be
 * NULL (no gate).  eps > 0.  ws: device workspace of at least
 * sana_linattn_workspace_size() bytes (256-byte aligned), caller-owned,
 * contents undefined on return.  The state reduction over N is split across
 * CTAs and combined in a fixed order, so results are bit-reproducible.
 * Gate precision (bf16): sigmoid(G) = 1/2 + tanh(G/2)/2 with the hardware
 * tanh approximation, absolute error about 2.5e-4 -- a relative error below
 * 1.5% for logits >= -4; for logits below -4 the gated output is under 2% of
 * the ungated one and carries an error below 1e-3 of the ungated scale.
 * ------------------------------------------------------------------------- */
SANA_API size_t sana_linattn_workspace_size(const sana_shape* shape, sana_dtype dtype);
SANA_API sana_status sana_linattn_fwd(const sana_shape* shape, sana_dtype dtype, const void* q,
                             const void* k, const void* v, const void* gate_logits,
                             const sana_rope* rope, float eps, void* out, void* ws,
                             size_t ws_bytes, sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * The two halves of sana_linattn_fwd, callable on their own ([SV1] sec. 3.2
 * pseudocode: the key-value contraction, then the query-side product and
 * normalisation).
 * sana_linattn_state: S_out = sum_j RoPE(phi K_j)^T V_j  (device fp32
 *   [B][heads][D][D], S[d][e]) and z_out = sum_j phi K_j (device fp32
 *   [B][heads][D]) over all N tokens.  Workspace:
 *   sana_linattn_state_workspace_size() bytes (split partial sums).
 * sana_linattn_apply: Y_i = sigmoid(G_i) * RoPE(phi Q_i) S / (phi Q_i . z + eps)
 *   for a given state (S, z as above); needs no workspace.  For bf16 it is a
 *   single kernel launch.
 * ------------------------------------------------------------------------- */
SANA_API size_t sana_linattn_state_workspace_size(const sana_shape* shape, sana_dtype dtype);
SANA_API sana_status sana_linattn_state(const sana_shape* shape, sana_dtype dtype, const void* k,
                                        const void* v, const sana_rope* rope, float* S_out,
                                        float* z_out, void* ws, size_t ws_bytes,
                                        sana_stream_t stream);
SANA_API sana_status sana_linattn_apply(const sana_shape* shape, sana_dtype dtype, const void* q,
                                        const void* gate_logits, const sana_rope* rope,
                                        const float* S, const float* z, float eps, void* out,
                                        sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * Backward of sana_linattn_fwd ([SV1] sec. 3.2 forward; the pages train the
 * model from scratch but print no backward: this is the chain rule through the
 * forward as written, with ReLU'(x) = 1 for x > 0 and 0 otherwise).
 * Given dy = dL/dY, writes dq, dk, dv (and d_gate when gate_logits is given;
 * both NULL for the ungated layer), all device (B, N, C) bf16, overwritten.
 * (S, z) are recomputed from k, v.  bf16 only (head_dim 128).  Workspace:
 * sana_linattn_bwd_workspace_size() bytes (split partials and combined S, z,
 * dS, dz; 256-byte aligned).  Gradients must not alias inputs or each other.
 * Deterministic: every reduction runs in a fixed order.
 * ------------------------------------------------------------------------- */
SANA_API size_t sana_linattn_bwd_workspace_size(const sana_shape* shape, sana_dtype dtype);
SANA_API sana_status sana_linattn_bwd(const sana_shape* shape, sana_dtype dtype, const void* q,
                                      const void* k, const void* v, const void* gate_logits,
                                      const sana_rope* rope, float eps, const void* dy, void* dq,
                                      void* dk, void* dv, void* d_gate, void* ws, size_t ws_bytes,
                                      sana_stream_t stream);
/* The same backward for a state the forward already holds: S (device fp32
 * [B][heads][D][D], S[d][e]) and z (device fp32 [B][heads][D]) exactly as
 * sana_linattn_state wrote them for these k, v (the two-phase forward keeps
 * them), so k and v are not read a second time to rebuild them.  Read only;
 * 16-byte aligned; they must not alias a gradient.  Arguments, workspace,
 * errors and determinism as for sana_linattn_bwd; NULL S or z is
 * SANA_ERR_INVALID_ARG. */
SANA_API sana_status sana_linattn_bwd_saved_state(const sana_shape* shape, sana_dtype dtype,
                                                  const void* q, const void* k, const void* v,
                                                  const void* gate_logits, const sana_rope* rope,
                                                  float eps, const float* S, const float* z,
                                                  const void* dy, void* dq, void* dk, void* dv,
                                                  void* d_gate, void* ws, size_t ws_bytes,
                                                  sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * One block of block-causal linear attention with the constant-memory state
 * ([SV1] sec. 3.4 causal O_i and Algorithm 1).  shape describes the chunk
 * (its T frames starting at absolute frame shape->t_offset).  The chunk's own
 * (S_c, z_c) are added to the running state; its output uses
 * (S_prev + S_c, z_prev + z_c): the chunk sees all earlier chunks and all of
 * itself.  state_S: device fp32 [B][heads][D][D] (S[d][e] = sum RoPE(phi k)_d v_e),
 * state_z: device fp32 [B][heads][D]; all-zero means "no past".  commit != 0
 * writes the updated state back in place (Algorithm 1's cache update after the
 * last denoising step); commit == 0 leaves it untouched.  Workspace as for
 * sana_linattn_fwd (sana_linattn_workspace_size of the chunk shape).
 * ------------------------------------------------------------------------- */
SANA_API sana_status sana_linattn_block_causal_step(const sana_shape* chunk, sana_dtype dtype,
                                           const void* q, const void* k, const void* v,
                                           const void* gate_logits, const sana_rope* rope,
                                           float eps, float* state_S, float* state_z,
                                           int commit, void* out, void* ws, size_t ws_bytes,
                                           sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * A whole sequence of blocks at once ([SV1] sec. 3.4 causal O_i and
 * Algorithm 1, for rollouts whose every block is known in advance).  shape
 * describes the sequence: T frames from absolute frame t_offset.  Block c
 * covers frames [c * chunk_frames, (c + 1) * chunk_frames) of it; when T is
 * not a multiple of chunk_frames the last block takes the remaining frames.
 * The output equals running sana_linattn_block_causal_step with commit over
 * the blocks in order from the given state (up to summation order): block c
 * reads state_S + sum_{c' <= c} S_c'.  The blocks' own states are computed
 * in parallel, then summed in block order (fixed order: bit-reproducible).
 * state_S, state_z: device fp32 [B][heads][D][D] / [B][heads][D]; on entry
 * the state before the first block (zeros = no past); commit != 0 writes the
 * state after the last block back in place, commit == 0 leaves it untouched.
 * chunk_frames >= 1.  Workspace: sana_linattn_block_causal_scan_workspace_size()
 * bytes (per-block partial and prefix states, 256-byte aligned).
 * ------------------------------------------------------------------------- */
SANA_API size_t sana_linattn_block_causal_scan_workspace_size(const sana_shape* shape,
                                                              int chunk_frames,
                                                              sana_dtype dtype);
SANA_API sana_status sana_linattn_block_causal_scan(const sana_shape* shape, int chunk_frames,
                                                    sana_dtype dtype, const void* q,
                                                    const void* k, const void* v,
                                                    const void* gate_logits,
                                                    const sana_rope* rope, float eps,
                                                    float* state_S, float* state_z, int commit,
                                                    void* out, void* ws, size_t ws_bytes,
                                                    sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * Gated softmax anchor ([SV2a]; reading: the same 3D RoPE on raw Q, K):
 *   Y = sigmoid(G) * softmax(RoPE(Q) RoPE(K)^T * scale) V, bidirectional over
 *   all N keys of the same batch entry and head.
 * rope may be NULL (no rotation).  scale <= 0 selects 1/sqrt(D).  Workspace:
 * sana_softmax_anchor_workspace_size() bytes (rotated Q and K copies).
 * Accuracy domain (bf16): the rotated operands are rounded to bf16 before
 * QK^T, so each logit carries an error of about 2^-9 of its own size and the
 * output error grows with the spread of the scaled logits q.k * scale.  With
 * Q, K ~ N(0, s^2) style inputs (logit standard deviation s) the max relative
 * error against the float64 oracle measured 4.4e-3 (s = 1), 8.1e-3 (s = 4),
 * 1.9e-2 (s = 8) and 3.1e-2 (s = 16): the 2e-2 parity bar holds for a logit
 * standard deviation up to 8.  (The stack's anchors read RMS-normalised
 * inputs through N(0, 1/C) projections: standard deviation about 1.)
 * ------------------------------------------------------------------------- */
SANA_API size_t sana_softmax_anchor_workspace_size(const sana_shape* shape, sana_dtype dtype);
SANA_API sana_status sana_softmax_anchor_fwd(const sana_shape* shape, sana_dtype dtype, const void* q,
                                    const void* k, const void* v, const void* gate_logits,
                                    const sana_rope* rope, float scale, void* out, void* ws,
                                    size_t ws_bytes, sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * The anchor's two phases, exposed so that each can be timed and reused
 * (sana_softmax_anchor_fwd runs exactly these: sana_rope_apply on Q with
 * mul = scale * log2(e) and on K with mul = 1, then the attention kernel).
 *
 * sana_rope_apply: out = mul * RoPE(x) for a (B, N, heads, head_dim) tensor,
 * the 3D RoPE of the anchor reading ("SANA-Video" paper notes sec. 3.2: 3D
 * RoPE; the pair layout as for the linear attention); rope == NULL applies no
 * rotation (out = mul * x).  bf16 (head_dim 128) or fp32; out must not
 * overlap x.  Shapes as sana_linattn_fwd.
 *
 * sana_softmax_anchor_rotated_fwd: Y = sigmoid(G) * softmax_2(Q' K'^T) V per
 * (batch, head), bidirectional over all N keys ("SANA-Video 2.0" abstract:
 * gated softmax anchors), where softmax_2 normalises 2^(logit) and Q', K' are
 * the rotated operands (Q' = scale * log2(e) * RoPE(Q), K' = RoPE(K), as
 * sana_rope_apply writes them), so the result equals sana_softmax_anchor_fwd.
 * bf16 only, head_dim 128; gate_logits nullable; out must not alias an input.
 * No workspace.  The bf16 rounding of Q' and K' bounds the accuracy: the 2e-2
 * parity bar holds for scaled logits (q.k/sqrt(D)) with a standard deviation
 * up to 8 (see sana_softmax_anchor_fwd).
 * ------------------------------------------------------------------------- */
SANA_API sana_status sana_rope_apply(const sana_shape* shape, sana_dtype dtype, const void* x,
                                     const sana_rope* rope, float mul, void* out,
                                     sana_stream_t stream);
SANA_API sana_status sana_softmax_anchor_rotated_fwd(const sana_shape* shape, const void* q_rot,
                                                     const void* k_rot, const void* v,
                                                     const void* gate_logits, void* out,
                                                     sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * Block-sparse gated softmax anchor ([SV2] Experiments and [SV2a]: the
 * deployment stack applies sparse attention to the softmax anchors; the
 * pattern below is this library's reading, the pages give none).
 * Queries form blocks of 256 tokens and keys tiles of 128 tokens; every query
 * block attends to exactly the keys of the `keep_tiles` key tiles listed for
 * it, with the softmax taken over those keys (same RoPE, scale and gate as
 * sana_softmax_anchor_fwd).
 * tiles: device int32 [B][heads][ceil(ceil(N/128)/2)][keep_tiles].
 *   select_tiles != 0: the library fills it: per block, the keep_tiles key
 *     tiles with the largest pooled logit mean(RoPE(Q)*scale) . mean(RoPE(K))
 *     over the block's and the tile's tokens, ties to the lower index, listed
 *     in ascending order.
 *   select_tiles == 0: the caller's list is used as given; entries must be
 *     distinct and in [0, ceil(N/128)) (other values give undefined results;
 *     loads stay in bounds).
 * 1 <= keep_tiles <= ceil(N/128); keep_tiles = ceil(N/128) is the dense
 * anchor.  bf16 only (head_dim 128); N <= 2^21.  Workspace:
 * sana_softmax_anchor_sparse_workspace_size() bytes (rotated Q, K and the
 * per-tile sums of the selection).
 * ------------------------------------------------------------------------- */
SANA_API size_t sana_softmax_anchor_sparse_workspace_size(const sana_shape* shape,
                                                          sana_dtype dtype);
SANA_API sana_status sana_softmax_anchor_sparse_fwd(const sana_shape* shape, sana_dtype dtype,
                                                    const void* q, const void* k, const void* v,
                                                    const void* gate_logits,
                                                    const sana_rope* rope, float scale,
                                                    int keep_tiles, int* tiles, int select_tiles,
                                                    void* out, void* ws, size_t ws_bytes,
                                                    sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * Block Attention Residuals router ([SV2] AttnRes equation, timestep term 0):
 *   l_i = w . v_i / sqrt(mean_c v_i^2 + rms_eps),  alpha = softmax_i(l),
 *   h = sum_i alpha_i v_i,   per token, over num_sources sources.
 * sources: HOST array of num_sources device pointers, each (B, N, C) in dtype,
 * ordered [embedding, block summaries..., partial sum].  1 <= num_sources <= 16.
 * w: device fp32 (C).  h_out: device (B, N, C) in dtype.  alpha_out: device
 * fp32 (B, N, num_sources) or NULL.  C must be a multiple of 8.
 * ------------------------------------------------------------------------- */
SANA_API sana_status sana_attnres_route(int B, long long N, int C, sana_dtype dtype,
                               const void* const* sources, int num_sources, const float* w,
                               float rms_eps, void* h_out, float* alpha_out,
                               sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * Backward of sana_attnres_route ([SV2] AttnRes equation; the pages print no
 * backward: the chain rule through the route as written).  Given dh = dL/dh
 * (device (B, N, C) bf16) writes d_sources[i] = dL/dv_i (HOST array of
 * num_sources device pointers, each (B, N, C) bf16, overwritten) and
 * dw = dL/dw (device fp32 (C), overwritten; summed over all tokens in a fixed
 * order, bit-reproducible).  bf16 only; 1 <= num_sources <= 4; C a multiple of
 * 256 up to 4096.  Workspace: sana_attnres_route_bwd_workspace_size() bytes
 * (per-CTA partial sums of dw).
 * ------------------------------------------------------------------------- */
SANA_API size_t sana_attnres_route_bwd_workspace_size(int B, long long N, int C);
SANA_API sana_status sana_attnres_route_bwd(int B, long long N, int C, sana_dtype dtype,
                                            const void* const* sources, int num_sources,
                                            const float* w, float rms_eps, const void* dh,
                                            void* const* d_sources, float* dw, void* ws,
                                            size_t ws_bytes, sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * Building blocks of the stack, exported for stage-wise checking.
 * sana_gemm_bf16: out[M][N] = epilogue(A[M][K] . W[N][K]^T) with bf16 A, W, out
 * and fp32 accumulation on tcgen05; epilogue 0 = identity, 1 = SiLU,
 * 2 = out += result (residual add into out).  lda/ldo are row strides in
 * elements (>= K / >= N, multiples of 8).  K must be a multiple of 64.
 * sana_rmsnorm: y = x / sqrt(mean(x^2) + eps) per row (no gain), (rows, C).
 * ------------------------------------------------------------------------- */
typedef enum { SANA_EPI_NONE = 0, SANA_EPI_SILU = 1, SANA_EPI_RESIDUAL = 2 } sana_epilogue;
SANA_API sana_status sana_gemm_bf16(long long M, int N, int K, const void* A, long long lda,
                           const void* W, void* out, long long ldo, int epilogue,
                           sana_stream_t stream);
SANA_API sana_status sana_rmsnorm(long long rows, int C, sana_dtype dtype, const void* x, float eps,
                         void* y, sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * MX block-scaled projection GEMM ("SANA-Video 2.0" hyper.ai summary,
 * Experiments: low-precision inference quantises only the linear GEMM layers,
 * weights to MXFP4 and activations to MXFP8; attention stays bf16).  The
 * formats are the OCP Microscaling v1.0 ones (a reading: the pages name them
 * without defining them): blocks of 32 elements along K share one E8M0 scale
 * 2^s, s = floor(log2 max|x|) - emax (8 for E4M3, 2 for E2M1) clamped to
 * [-127, 127] (-127 for an all-zero block); elements x / 2^s rounded to
 * nearest even and saturated.
 *
 * Layouts (device memory, caller-owned):
 *   E4M3 codes: one byte per element, [rows][K] row-major;
 *   E2M1 codes: two per byte, element 2i in the low nibble, [rows][K/2];
 *   scales: sana_mx_scale_bytes(rows, K) bytes of E8M0 (s + 127) in 512-byte
 *     atoms, one per 128 rows x 128 K-elements, ordered [ceil(rows/128)][K/128];
 *     inside an atom, row r and 32-element block b (0..3) sit at byte
 *     16 (r % 32) + 4 (r / 32) + b.  Padding rows hold scale 0.
 *
 * sana_mx_quantize: x bf16 (rows, K) -> codes q (E4M3 if fp4 == 0, E2M1 if
 *   fp4 == 1) and scales.  K must be a positive multiple of 128.
 * sana_mx_gemm: out[M][N] (bf16, row stride ldo) = epilogue(Q8(x) . Q4(w)^T)
 *   from E4M3 activations (M, K) and E2M1 weights (N, K) with their scales,
 *   fp32 accumulation on tcgen05 (kind::mxf8f6f4 with block scales);
 *   epilogue as sana_gemm_bf16 (0 identity, 1 SiLU, 2 out += result).  N and
 *   K positive multiples of 128; the E2M1 weights 32-byte aligned, the other
 *   pointers 16-byte aligned.
 * sana_mx_linear: the quantised projection of bf16 activations: quantises x
 *   into the workspace (sana_mx_linear_workspace_size bytes, 256-byte
 *   aligned) and runs sana_mx_gemm against pre-quantised weights.
 * Errors: SANA_ERR_UNSUPPORTED for sizes the kernels do not cover,
 * SANA_ERR_INVALID_ARG for NULL, misaligned or aliasing buffers.
 * ------------------------------------------------------------------------- */
SANA_API size_t sana_mx_scale_bytes(long long rows, int K);
SANA_API sana_status sana_mx_quantize(const void* x, long long rows, int K, int fp4, void* q,
                                      void* scales, sana_stream_t stream);
SANA_API sana_status sana_mx_gemm(long long M, int N, int K, const void* xq,
                                  const void* x_scales, const void* wq, const void* w_scales,
                                  void* out, long long ldo, int epilogue, sana_stream_t stream);
SANA_API size_t sana_mx_linear_workspace_size(long long M, int K);
SANA_API sana_status sana_mx_linear(long long M, int N, int K, const void* x, const void* wq,
                                    const void* w_scales, void* out, long long ldo, int epilogue,
                                    void* ws, size_t ws_bytes, sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * Hybrid stack forward ([SV2] method; [SV2a] 3:1 interleave).
 * Layer l (0-based) is a softmax anchor iff l % ratio == ratio - 1, else a
 * gated linear-attention layer.  Each layer has an attention sublayer
 * (RMSNorm -> x.W_qkvg^T split into Q, K, V, G -> gated attention -> .W_o^T)
 * and, when ffn_mult > 0, an FFN sublayer (RMSNorm -> W_down SiLU(W_up x)).
 * use_attnres != 0: each sublayer reads h = route(sources) with the shared
 * attention or FFN query; its output is added to the running partial sum;
 * every block_span layers the partial sum is frozen as a block summary; the
 * result is route(final sources, w_attn).  use_attnres == 0: plain pre-norm
 * residual x += sublayer(RMSNorm(x)); the result is the final x.
 * bf16 only, D = 128, C = heads * 128.
 * ------------------------------------------------------------------------- */
typedef struct {
  int layers;
  int block_span;
  int ratio;
  int use_attnres;
  int ffn_mult;
  float eps;          /* linear-attention denominator eps */
  float rms_eps;      /* RMSNorm eps (routing and pre-norm) */
  float anchor_scale; /* <= 0: 1/sqrt(D) */
  int anchor_keep_tiles; /* 0: dense anchors; k > 0: block-sparse anchors keeping
                            the k highest-scoring 128-key tiles per 256-query
                            block (sana_softmax_anchor_sparse_fwd's selection) */
  int mx_projections;    /* 0: bf16 projections; 1: every projection (QKVG, O, FFN
                            up and down) is the MX projection -- activations
                            quantised to MXFP8 on the fly, MXFP4 weights from the
                            mx_* arrays of sana_stack_weights (the deployment of
                            [SV2] Experiments; attention stays bf16) */
} sana_stack_config;

typedef struct {
  const void* const* w_qkvg; /* HOST array [layers] of device (4C, C) bf16 */
  const void* const* w_o;    /* [layers] of (C, C) */
  const void* const* w_up;   /* [layers] of (ffn_mult*C, C), or NULL if ffn_mult == 0 */
  const void* const* w_down; /* [layers] of (C, ffn_mult*C), or NULL */
  const float* w_attn;       /* device fp32 (C): shared attention router query */
  const float* w_ffn;        /* device fp32 (C): shared FFN router query */
  /* With cfg->mx_projections: per layer, each weight as sana_mx_quantize writes
     it with fp4 = 1 (E2M1 codes, 32-byte aligned, and scale atoms); the bf16
     arrays above are then not read and may be NULL. */
  const void* const* mx_qkvg;
  const void* const* mx_qkvg_scales;
  const void* const* mx_o;
  const void* const* mx_o_scales;
  const void* const* mx_up;
  const void* const* mx_up_scales;
  const void* const* mx_down;
  const void* const* mx_down_scales;
} sana_stack_weights;

SANA_API size_t sana_hybrid_stack_workspace_size(const sana_shape* shape, const sana_stack_config* cfg);

/* Where sana_hybrid_stack_fwd keeps its intermediates inside the workspace,
 * as byte offsets from the workspace base (every tensor bf16, row-major,
 * B*N rows).  Once a call has completed on its stream the workspace holds the
 * state after its last layer L = cfg->layers - 1:
 *   q, k, v, g  layer L's projections x_hat . W_qkvg^T, (B, N, C) each;
 *   attn        layer L's gated attention output, before W_o, (B, N, C);
 *   x_hat       the normalised input of layer L's last sublayer (its FFN
 *               sublayer when ffn_mult > 0), (B, N, C);
 *   ffn         SiLU(x_hat . W_up^T) of layer L, (B, N, ffn_mult*C);
 *               SIZE_MAX when ffn_mult == 0;
 *   blocks[i]   with AttnRes, block summary i for i < floor(layers /
 *               block_span); the next buffer holds the running partial sum
 *               when layers is not a multiple of block_span.  num_blocks
 *               buffers in all (0 without AttnRes; then `out` holds the
 *               residual stream).
 * Running the stack for a prefix of its layers therefore exposes every
 * sublayer's result; the layout depends only on shape and cfg->layers,
 * block_span, ffn_mult and anchor_keep_tiles.  Returns SANA_ERR_INVALID_ARG
 * for a NULL argument or a configuration sana_hybrid_stack_fwd rejects.
 * (A testing and inspection aid: the pages define no such call.) */
typedef struct {
  size_t x_hat, q, k, v, g, attn, ffn;
  int num_blocks;
  size_t blocks[16];
} sana_stack_ws_layout;
SANA_API sana_status sana_hybrid_stack_workspace_layout(const sana_shape* shape,
                                                        const sana_stack_config* cfg,
                                                        sana_stack_ws_layout* layout);
SANA_API sana_status sana_hybrid_stack_fwd(const sana_shape* shape, const sana_stack_config* cfg,
                                  const sana_stack_weights* weights, const sana_rope* rope,
                                  const void* x_embed, void* out, void* ws, size_t ws_bytes,
                                  sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * Allocation-free linear attention (the pages have no counterpart; this is a
 * deployment convenience).  For callers that cannot allocate device memory:
 * same arguments and result as sana_linattn_fwd minus the workspace, which is
 * taken from a fixed array inside the library of
 * sana_linattn_noalloc_scratch_bytes() bytes (16 MiB) held on every GPU that
 * loads the library until the process exits.  Shapes needing more scratch
 * than that (sana_linattn_workspace_size() larger) return
 * SANA_ERR_UNSUPPORTED; for bf16 at head_dim 128 that is B * heads >= 128.
 * All calls share the array: calls that overlap on the GPU (different streams
 * or host threads) race.  The first call on a device (and the first after a
 * device reset) looks up the array's device address; make it before any
 * stream capture.  Under lazy module loading (the CUDA 12 default) the
 * library's device code, and the array with it, is loaded onto a device by
 * the first library call made there, which may synchronise the device: make
 * one call (or call sana_linattn_noalloc_scratch_bytes() after any other
 * library call on that device) at initialisation time.
 * ------------------------------------------------------------------------- */
SANA_API size_t sana_linattn_noalloc_scratch_bytes(void);
SANA_API sana_status sana_linattn_fwd_noalloc(const sana_shape* shape, sana_dtype dtype,
                                              const void* q, const void* k, const void* v,
                                              const void* gate_logits, const sana_rope* rope,
                                              float eps, void* out, sana_stream_t stream);

/* ---------------------------------------------------------------------------
 * Status helpers.
 * sana_sync_status: synchronizes `stream`, then reports (and clears) the
 * device status word: SANA_ERR_TIMEOUT if a kernel gave up a bounded wait,
 * SANA_ERR_CUDA on an asynchronous CUDA error, else SANA_OK.
 * sana_last_error_string: thread-local message of the last non-OK status.
 * ------------------------------------------------------------------------- */
SANA_API sana_status sana_sync_status(sana_stream_t stream);

/* Failure-detection self-test: enqueues one small kernel that waits on a
 * barrier nothing ever signals, through the same bounded wait every pipeline
 * uses; after limit_ms (1..2000) it records a timeout in the device status word
 * and returns normally, so the next sana_sync_status() reports SANA_ERR_TIMEOUT
 * and the CUDA context stays usable.  No fault, trap or hang is involved. */
SANA_API sana_status sana_selftest_bounded_wait(unsigned int limit_ms, sana_stream_t stream);
SANA_API const char* sana_last_error_string(void);
SANA_API const char* sana_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SANA_H_ */
