// Hybrid linear-softmax stack forward: the host-side schedule over the
// kernels, all launches stream-ordered with no host synchronisation.
//
//   "SANA-Video 2.0" abstract: three gated linear-attention layers to one
//   gated softmax anchor (3:1).  hyper.ai summary, Method: Block Attention
//   Residuals -- sublayer outputs accumulate into a running partial sum, a
//   completed block of `block_span` layers freezes it as a block summary, and
//   every sublayer reads h = sum_i softmax_i(w . RMSNorm(v_i)) v_i over
//   [embedding, block summaries, partial sum] with one shared query for the
//   attention sublayers and one for the FFN sublayers.
//
// Per layer (AttnRes on):
//   route(w_attn) + RMSNorm  -> x_hat            (one fused kernel)
//   x_hat . W_qkvg^T         -> Q, K, V, G       (one GEMM, output split in 4)
//   linear attention | softmax anchor -> a
//   a . W_o^T                -> partial (+)=     (GEMM, residual epilogue)
//   route(w_ffn) + RMSNorm   -> x_hat
//   SiLU(x_hat . W_up^T)     -> u                (GEMM, SiLU epilogue)
//   u . W_down^T             -> partial +=       (GEMM, residual epilogue)
//   every block_span layers: partial becomes a summary (pointer hand-over).
#include <cmath>
#include <cstdint>
#include <vector>

#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {

sana_status gemm_run_parts(long long M, int N, int K, const void* A, long long lda, const void* W,
                           void* const* outs, int nparts, long long ldo, int epilogue,
                           cudaStream_t st);

namespace {

struct StackWs {
  __nv_bfloat16 *xhat, *q, *k, *v, *g, *attn, *ffn;
  std::vector<__nv_bfloat16*> blocks;  // summaries + the running partial sum
  void* attn_ws;
  size_t attn_ws_bytes;
  int* tiles;  // kept key tiles of the sparse anchors
  uint8_t *mxq, *mxs;  // quantised activations of the MX projections (codes, scales)
  size_t bytes;
};

StackWs carve_stack(const sana_shape& s, const sana_stack_config& c, void* ws) {
  const size_t tok = (size_t)s.B * s.T * s.H * s.W;
  const size_t C = (size_t)s.heads * s.head_dim;
  Carver cv(ws, ~size_t(0));
  StackWs w{};
  w.xhat = cv.take<__nv_bfloat16>(tok * C);
  w.q = cv.take<__nv_bfloat16>(tok * C);
  w.k = cv.take<__nv_bfloat16>(tok * C);
  w.v = cv.take<__nv_bfloat16>(tok * C);
  w.g = cv.take<__nv_bfloat16>(tok * C);
  w.attn = cv.take<__nv_bfloat16>(tok * C);
  w.ffn = c.ffn_mult > 0 ? cv.take<__nv_bfloat16>(tok * C * c.ffn_mult) : nullptr;
  if (c.use_attnres) {
    const int nblocks = (c.layers + c.block_span - 1) / c.block_span;
    for (int i = 0; i < nblocks; ++i) w.blocks.push_back(cv.take<__nv_bfloat16>(tok * C));
  }
  const size_t lin = linattn_ws_bytes(s, SANA_BF16);
  const size_t anc = c.anchor_keep_tiles > 0 ? anchor_sparse_ws_bytes(s) : anchor_ws_bytes(s, SANA_BF16);
  w.attn_ws_bytes = lin > anc ? lin : anc;
  w.attn_ws = cv.take<char>(w.attn_ws_bytes);
  if (c.anchor_keep_tiles > 0) {
    const size_t ntiles = (tok / s.B + 127) / 128;
    w.tiles = cv.take<int>((size_t)s.B * s.heads * ((ntiles + 1) / 2) * c.anchor_keep_tiles);
  }
  if (c.mx_projections) {
    const size_t kmax = c.ffn_mult > 1 ? C * c.ffn_mult : C;  // widest contraction
    w.mxq = cv.take<uint8_t>(tok * kmax);
    w.mxs = cv.take<uint8_t>(mx_scale_bytes((long long)tok, (int)kmax));
  }
  w.bytes = align_up(cv.used, 256);
  return w;
}

sana_status check_cfg(const sana_shape* s, const sana_stack_config* c) {
  if (!s || !c) return fail(SANA_ERR_INVALID_ARG, "stack: NULL shape or config");
  if (s->head_dim != 128) return fail(SANA_ERR_UNSUPPORTED, "stack: bf16 path needs head_dim 128");
  if (s->B < 1 || s->T < 1 || s->H < 1 || s->W < 1 || s->heads < 1)
    return fail(SANA_ERR_INVALID_ARG, "stack: bad shape");
  if (s->heads * 128 % 256 != 0)
    return fail(SANA_ERR_UNSUPPORTED, "stack: hidden size must be a multiple of 256");
  if (c->layers < 1 || c->ratio < 1 || c->ffn_mult < 0 || c->ffn_mult > 8 ||
      (c->use_attnres && c->block_span < 1))
    return fail(SANA_ERR_INVALID_ARG, "stack: bad config");
  if (c->mx_projections != 0 && c->mx_projections != 1)
    return fail(SANA_ERR_INVALID_ARG, "stack: mx_projections must be 0 or 1");
  if (c->use_attnres && 1 + (c->layers + c->block_span - 1) / c->block_span > 16)
    return fail(SANA_ERR_UNSUPPORTED, "stack: more than 16 AttnRes sources");
  if (!(c->eps >= 0.f) || !(c->rms_eps >= 0.f)) return fail(SANA_ERR_INVALID_ARG, "stack: bad eps");
  const long long ntiles = ((long long)s->T * s->H * s->W + 127) / 128;
  if (c->anchor_keep_tiles < 0 || c->anchor_keep_tiles > ntiles ||
      (c->anchor_keep_tiles > 0 && ntiles > kAnchorMaxTiles))
    return fail(SANA_ERR_INVALID_ARG, "stack: anchor_keep_tiles=%d outside [0, %lld]",
                c->anchor_keep_tiles, ntiles);
  return SANA_OK;
}

}  // namespace
}  // namespace sana

using namespace sana;

extern "C" size_t sana_hybrid_stack_workspace_size(const sana_shape* s, const sana_stack_config* c) {
  if (check_cfg(s, c) != SANA_OK) return 0;
  return carve_stack(*s, *c, nullptr).bytes;
}

extern "C" sana_status sana_hybrid_stack_workspace_layout(const sana_shape* s,
                                                          const sana_stack_config* c,
                                                          sana_stack_ws_layout* out) {
  if (!out) return fail(SANA_ERR_INVALID_ARG, "stack layout: NULL output");
  if (sana_status e = check_cfg(s, c)) return e;
  // carve from a fake non-null base so that the offsets come out directly
  char* const base = reinterpret_cast<char*>(256);
  const StackWs w = carve_stack(*s, *c, base);
  auto off = [&](const void* p) { return static_cast<size_t>(static_cast<const char*>(p) - base); };
  sana_stack_ws_layout L{};
  L.x_hat = off(w.xhat);
  L.q = off(w.q);
  L.k = off(w.k);
  L.v = off(w.v);
  L.g = off(w.g);
  L.attn = off(w.attn);
  L.ffn = w.ffn ? off(w.ffn) : SIZE_MAX;
  L.num_blocks = static_cast<int>(w.blocks.size());
  for (int i = 0; i < L.num_blocks; ++i) L.blocks[i] = off(w.blocks[i]);
  *out = L;
  return SANA_OK;
}

extern "C" sana_status sana_hybrid_stack_fwd(const sana_shape* s, const sana_stack_config* c,
                                             const sana_stack_weights* w, const sana_rope* rope,
                                             const void* x_embed, void* out, void* ws,
                                             size_t ws_bytes, sana_stream_t st) {
  if (sana_status e = check_cfg(s, c)) return e;
  const bool mx = c->mx_projections != 0;
  if (!w || !rope || !x_embed || !out)
    return fail(SANA_ERR_INVALID_ARG, "stack: NULL argument");
  if (!mx && (!w->w_qkvg || !w->w_o || (c->ffn_mult > 0 && (!w->w_up || !w->w_down))))
    return fail(SANA_ERR_INVALID_ARG, "stack: bf16 weights are NULL");
  if (mx && (!w->mx_qkvg || !w->mx_qkvg_scales || !w->mx_o || !w->mx_o_scales ||
             (c->ffn_mult > 0 && (!w->mx_up || !w->mx_up_scales || !w->mx_down ||
                                  !w->mx_down_scales))))
    return fail(SANA_ERR_INVALID_ARG, "stack: MX weights are NULL");
  if (c->use_attnres && (!w->w_attn || (c->ffn_mult > 0 && !w->w_ffn)))
    return fail(SANA_ERR_INVALID_ARG, "stack: router queries are NULL");
  if (rope->n_t + rope->n_h + rope->n_w != 64 || rope->H != s->H || rope->W != s->W ||
      rope->T_total < s->t_offset + s->T)
    return fail(SANA_ERR_INVALID_ARG, "stack: rope tables do not match the grid");
  const size_t need = carve_stack(*s, *c, nullptr).bytes;
  if (!ws || ws_bytes < need)
    return fail(SANA_ERR_WORKSPACE, "stack: workspace %zu < %zu bytes", ws ? ws_bytes : 0, need);
  const StackWs P = carve_stack(*s, *c, ws);
  const int C = s->heads * 128, F = c->ffn_mult * C;
  const long long M = (long long)s->B * s->T * s->H * s->W;
  const long long Nseq = (long long)s->T * s->H * s->W;
  const RopeDev rd{rope->cos_t, rope->sin_t, rope->cos_h, rope->sin_h, rope->cos_w, rope->sin_w,
                   rope->n_t, rope->n_h, rope->n_w};
  const float scale = c->anchor_scale > 0.f ? c->anchor_scale : 1.f / sqrtf(128.f);
  // one projection x (M, K) . W^T into `outs`: a bf16 GEMM, or the MX
  // projection (x quantised to MXFP8 into the workspace, MXFP4 weights)
  auto project = [&](const void* x, int K, int Nout, const void* wbf, const void* wq,
                     const void* wsc, void* const* outs, int nparts, int epi) -> sana_status {
    if (!mx) return gemm_run_parts(M, Nout, K, x, K, wbf, outs, nparts, Nout / nparts, epi, st);
    if (sana_status e = mx_quantize_run(x, M, K, false, P.mxq, P.mxs, st)) return e;
    return mx_gemm_run_parts(M, Nout, K, P.mxq, P.mxs, wq, wsc, outs, nparts, Nout / nparts, epi,
                             st);
  };
  auto wsel = [&](const void* const* arr, int l) -> const void* { return arr ? arr[l] : nullptr; };
  auto attention = [&](int l) -> sana_status {
    void* parts[4] = {P.q, P.k, P.v, P.g};
    if (sana_status e = project(P.xhat, C, 4 * C, wsel(w->w_qkvg, l), wsel(w->mx_qkvg, l),
                                wsel(w->mx_qkvg_scales, l), parts, 4, 0))
      return e;
    if (l % c->ratio == c->ratio - 1) {
      if (c->anchor_keep_tiles > 0)
        return anchor_sparse_run(*s, P.q, P.k, P.v, P.g, &rd, scale, c->anchor_keep_tiles, P.tiles,
                                 true, P.attn, P.attn_ws, P.attn_ws_bytes, st);
      return anchor_run(*s, SANA_BF16, P.q, P.k, P.v, P.g, &rd, scale, P.attn, P.attn_ws,
                        P.attn_ws_bytes, st);
    }
    return linattn_run(*s, SANA_BF16, P.q, P.k, P.v, P.g, rd, c->eps, nullptr, nullptr, false,
                       false, P.attn, P.attn_ws, P.attn_ws_bytes, st);
  };

  if (!c->use_attnres) {
    // plain pre-norm residual stream in `out`
    if (cudaMemcpyAsync(out, x_embed, (size_t)M * C * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return fail(SANA_ERR_CUDA, "stack: copy of the embedding failed");
    void* o_out[1] = {out};
    void* f_out[1] = {P.ffn};
    for (int l = 0; l < c->layers; ++l) {
      if (sana_status e = rmsnorm_run(M, C, SANA_BF16, out, c->rms_eps, P.xhat, st)) return e;
      if (sana_status e = attention(l)) return e;
      if (sana_status e = project(P.attn, C, C, wsel(w->w_o, l), wsel(w->mx_o, l),
                                  wsel(w->mx_o_scales, l), o_out, 1, 2))
        return e;
      if (c->ffn_mult > 0) {
        if (sana_status e = rmsnorm_run(M, C, SANA_BF16, out, c->rms_eps, P.xhat, st)) return e;
        if (sana_status e = project(P.xhat, C, F, wsel(w->w_up, l), wsel(w->mx_up, l),
                                    wsel(w->mx_up_scales, l), f_out, 1, 1))
          return e;
        if (sana_status e = project(P.ffn, F, C, wsel(w->w_down, l), wsel(w->mx_down, l),
                                    wsel(w->mx_down_scales, l), o_out, 1, 2))
          return e;
      }
    }
    return SANA_OK;
  }

  // AttnRes: sources = [embedding, summaries..., partial (when non-empty)]
  std::vector<const void*> src;
  int nsum = 0;
  bool partial_live = false;
  auto sources = [&]() {
    src.clear();
    src.push_back(x_embed);
    for (int i = 0; i < nsum; ++i) src.push_back(P.blocks[i]);
    if (partial_live) src.push_back(P.blocks[nsum]);
  };
  for (int l = 0; l < c->layers; ++l) {
    __nv_bfloat16* partial = P.blocks[nsum];
    sources();
    if (sana_status e = attnres_run(s->B, Nseq, C, SANA_BF16, src.data(), (int)src.size(),
                                    w->w_attn, c->rms_eps, nullptr, nullptr, true, P.xhat, st))
      return e;
    if (sana_status e = attention(l)) return e;
    void* p_out[1] = {partial};
    void* f_out[1] = {P.ffn};
    if (sana_status e = project(P.attn, C, C, wsel(w->w_o, l), wsel(w->mx_o, l),
                                wsel(w->mx_o_scales, l), p_out, 1, partial_live ? 2 : 0))
      return e;
    partial_live = true;
    if (c->ffn_mult > 0) {
      sources();
      if (sana_status e = attnres_run(s->B, Nseq, C, SANA_BF16, src.data(), (int)src.size(),
                                      w->w_ffn, c->rms_eps, nullptr, nullptr, true, P.xhat, st))
        return e;
      if (sana_status e = project(P.xhat, C, F, wsel(w->w_up, l), wsel(w->mx_up, l),
                                  wsel(w->mx_up_scales, l), f_out, 1, 1))
        return e;
      if (sana_status e = project(P.ffn, F, C, wsel(w->w_down, l), wsel(w->mx_down, l),
                                  wsel(w->mx_down_scales, l), p_out, 1, 2))
        return e;
    }
    if ((l + 1) % c->block_span == 0) {  // freeze the block summary
      ++nsum;
      partial_live = false;
    }
  }
  sources();
  return attnres_run(s->B, Nseq, C, SANA_BF16, src.data(), (int)src.size(), w->w_attn,
                     c->rms_eps, out, nullptr, false, nullptr, st);
}
