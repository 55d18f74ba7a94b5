// Block-causal linear attention over a whole known sequence.
//
// "SANA-Video" paper notes, sec. 3.4: the causal state after a block is the
// running sum of every earlier block's S = sum RoPE(phi K)^T V and z = sum phi K,
// and Algorithm 1 adds a block to the cache once the block is done, so block c
// is read against S_0 + sum_{c' <= c} S_c' (itself included).  When every block
// is known up front (teacher-forced or self-forcing rollouts, sec. 4 training
// paragraphs) the blocks' own states do not depend on one another:
//
//   1. one split-reduction launch computes every block's S_c, z_c (blocks are
//      batch entries of a strided view; the rotary frame of entry c starts at
//      t_offset + c * block_frames),
//   2. a fixed-order prefix over blocks forms P_c = S_0 + sum_{c' <= c} S_c'
//      (and the final state when committing),
//   3. one output launch applies each block's P_c to its own queries.
//
// A last block shorter than the others (the frame count not divisible by the
// block length) is a second, one-entry view through the same kernels.
#include <cuda_runtime.h>

#include "sana_internal.h"

namespace sana {
namespace {

// P[c][h][e] = S0[h][e] + sum_{c' <= c} sum_split partial[c'][h][split][e], in
// that order, for e over the D*D entries of S followed by the D entries of z.
// One thread per (head, entry); each walks the blocks in order.
__global__ void __launch_bounds__(256)
    linattn_prefix_kernel(const float* __restrict__ pS_main, const float* __restrict__ pz_main,
                          int n_main, int splits_main, const float* __restrict__ pS_tail,
                          const float* __restrict__ pz_tail, int splits_tail, int heads, int D,
                          const float* S0, const float* z0, float* __restrict__ P_S,
                          float* __restrict__ P_z, float* S_fin, float* z_fin) {
  const int DD = D * D;
  const int e = blockIdx.y * blockDim.x + threadIdx.x;
  if (e >= DD + D) return;
  const int h = blockIdx.x;
  const bool is_z = e >= DD;
  const int i = is_z ? e - DD : e;
  const size_t L = is_z ? (size_t)D : (size_t)DD;
  const float* pm = is_z ? pz_main : pS_main;
  const float* pt = is_z ? pz_tail : pS_tail;
  const float* init = is_z ? z0 : S0;
  float* P = is_z ? P_z : P_S;
  float* fin = is_z ? z_fin : S_fin;
  float run = init ? init[h * L + i] : 0.f;
  for (int c = 0; c < n_main; ++c) {
    const float* part = pm + ((size_t)c * heads + h) * splits_main * L + i;
    float acc = 0.f;
    for (int sp = 0; sp < splits_main; ++sp) acc += part[sp * L];
    run += acc;
    P[((size_t)c * heads + h) * L + i] = run;
  }
  if (pt) {
    const float* part = pt + (size_t)h * splits_tail * L + i;
    float acc = 0.f;
    for (int sp = 0; sp < splits_tail; ++sp) acc += part[sp * L];
    run += acc;
    P[((size_t)n_main * heads + h) * L + i] = run;
  }
  if (fin) fin[h * L + i] = run;
}

// The two views of one sequence: n_full blocks of `frames` frames as batch
// entries, and the last `tail` frames (if any) as one more entry.
struct ScanParts {
  int n_full, tail;
  sana_shape full_view, tail_view;
  LinAttnPlan plan_full, plan_tail;
};

ScanParts scan_parts(const sana_shape& s, int frames, sana_dtype dt) {
  ScanParts p{};
  p.n_full = s.T / frames;
  p.tail = s.T % frames;
  p.full_view = s;
  p.full_view.B = p.n_full > 0 ? p.n_full : 1;
  p.full_view.T = frames;
  p.tail_view = s;
  p.tail_view.B = 1;
  p.tail_view.T = p.tail;
  p.tail_view.t_offset = s.t_offset + p.n_full * frames;
  p.plan_full = linattn_plan(p.full_view, dt);
  p.plan_tail = linattn_plan(p.tail_view, dt);
  return p;
}

struct ScanWs {
  float *pS_full, *pz_full, *pS_tail, *pz_tail;  // split partials of every block
  float *P_S, *P_z;                              // inclusive prefix per block
  size_t bytes;
};

ScanWs carve_scan(const sana_shape& s, const ScanParts& p, void* ws) {
  const size_t D = s.head_dim, H = s.heads, nf = p.n_full, nt = p.tail ? 1 : 0;
  Carver cv(ws, ~size_t(0));
  ScanWs w{};
  w.pS_full = cv.take<float>(nf * H * p.plan_full.splits_a * D * D);
  w.pz_full = cv.take<float>(nf * H * p.plan_full.splits_a * D);
  w.pS_tail = cv.take<float>(nt * H * p.plan_tail.splits_a * D * D);
  w.pz_tail = cv.take<float>(nt * H * p.plan_tail.splits_a * D);
  w.P_S = cv.take<float>((nf + nt) * H * D * D);
  w.P_z = cv.take<float>((nf + nt) * H * D);
  w.bytes = align_up(cv.used, 256);
  return w;
}

GridDev view_grid(const sana_shape& v, int t_stride) {
  GridDev g{v.T, v.H, v.W, v.t_offset, v.T * v.H * v.W, v.heads};
  g.t_stride = t_stride;
  return g;
}

sana_status partials(const sana_shape& v, const LinAttnPlan& plan, sana_dtype dt, const void* k,
                     const void* vv, const RopeDev& rope, const GridDev& g, float* pS, float* pz,
                     cudaStream_t st) {
  if (dt == SANA_BF16) return linattn_bf16_partials(v, plan, k, vv, rope, g, pS, pz, st);
  return linattn_f32_partials(v, static_cast<const float*>(k), static_cast<const float*>(vv), rope,
                              g, plan.splits_a, pS, pz, st);
}

sana_status apply(const sana_shape& v, const LinAttnPlan& plan, sana_dtype dt, const void* q,
                  const void* gt, const RopeDev& rope, const GridDev& g, const float* S,
                  const float* z, float eps, void* out, cudaStream_t st) {
  if (dt == SANA_BF16) return linattn_bf16_apply(v, plan, q, gt, rope, g, S, z, eps, out, st);
  return linattn_f32_apply(v, static_cast<const float*>(q), static_cast<const float*>(gt), rope, g,
                           S, z, eps, static_cast<float*>(out), st);
}

}  // namespace

size_t linattn_scan_ws_bytes(const sana_shape& s, int chunk_frames, sana_dtype dt) {
  return carve_scan(s, scan_parts(s, chunk_frames, dt), nullptr).bytes;
}

sana_status linattn_scan_run(const sana_shape& s, int chunk_frames, sana_dtype dt, const void* q,
                             const void* k, const void* v, const void* g, const RopeDev& rope,
                             float eps, float* state_S, float* state_z, bool commit, void* out,
                             void* ws, size_t ws_bytes, cudaStream_t st) {
  if (s.T == 0) return SANA_OK;
  const ScanParts p = scan_parts(s, chunk_frames, dt);
  const ScanWs w = carve_scan(s, p, ws);
  if (ws_bytes < w.bytes)
    return fail(SANA_ERR_WORKSPACE, "block-causal scan: workspace %zu < %zu bytes", ws_bytes,
                w.bytes);
  const GridDev g_full = view_grid(p.full_view, chunk_frames);
  const GridDev g_tail = view_grid(p.tail_view, 0);
  if (dt == SANA_BF16) {
    const GridDev& widest = p.n_full ? g_full : g_tail;
    if (rope_smem_bytes(widest, rope) > kRopeSmemMax)
      return fail(SANA_ERR_UNSUPPORTED,
                  "block-causal scan: blocks of %d frames of %dx%d need too many RoPE table bytes",
                  widest.T, s.H, s.W);
  }
  const size_t es = dt == SANA_BF16 ? 2 : 4;
  const size_t D = s.head_dim, H = s.heads, DD = D * D;
  const size_t hw = (size_t)s.H * s.W, N = (size_t)s.T * hw, C = H * D;
  const size_t tail_tok = (size_t)p.n_full * chunk_frames * hw;
  const dim3 prefix_grid(s.heads, (unsigned)((DD + D + 255) / 256));
  for (int b = 0; b < s.B; ++b) {
    // token `tok` of sequence b
    auto in = [&](const void* base, size_t tok) -> const void* {
      return base ? static_cast<const char*>(base) + ((size_t)b * N + tok) * C * es : nullptr;
    };
    void* out_b = static_cast<char*>(out) + (size_t)b * N * C * es;
    float* Sb = state_S + (size_t)b * H * DD;
    float* zb = state_z + (size_t)b * H * D;
    if (p.n_full)
      if (sana_status e = partials(p.full_view, p.plan_full, dt, in(k, 0), in(v, 0), rope, g_full,
                                   w.pS_full, w.pz_full, st))
        return e;
    if (p.tail)
      if (sana_status e = partials(p.tail_view, p.plan_tail, dt, in(k, tail_tok), in(v, tail_tok),
                                   rope, g_tail, w.pS_tail, w.pz_tail, st))
        return e;
    linattn_prefix_kernel<<<prefix_grid, 256, 0, st>>>(
        w.pS_full, w.pz_full, p.n_full, p.plan_full.splits_a, p.tail ? w.pS_tail : nullptr,
        p.tail ? w.pz_tail : nullptr, p.plan_tail.splits_a, s.heads, (int)D, Sb, zb, w.P_S, w.P_z,
        commit ? Sb : nullptr, commit ? zb : nullptr);
    if (sana_status e = check_launch("linattn_prefix_kernel")) return e;
    if (p.n_full)
      if (sana_status e = apply(p.full_view, p.plan_full, dt, in(q, 0), in(g, 0), rope, g_full,
                                w.P_S, w.P_z, eps, out_b, st))
        return e;
    if (p.tail)
      if (sana_status e = apply(p.tail_view, p.plan_tail, dt, in(q, tail_tok), in(g, tail_tok),
                                rope, g_tail, w.P_S + (size_t)p.n_full * H * DD,
                                w.P_z + (size_t)p.n_full * H * D, eps,
                                static_cast<char*>(out_b) + tail_tok * C * es, st))
        return e;
  }
  return SANA_OK;
}

}  // namespace sana
