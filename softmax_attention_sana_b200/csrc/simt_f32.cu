// fp32 FFMA kernels: linear attention (state, output) and the softmax anchor
// for head dims 16 / 32 / 64 / 128.  These serve fp32 tensors, where the
// 1e-4 error bar rules out tensor-core (TF32/bf16) inputs.
//
//   "SANA-Video" paper notes, sec. 3.2 (O_i with RoPE after the ReLU and a
//   RoPE-free denominator), sec. 3.4 (cumulative state);
//   "SANA-Video 2.0" abstract: gated linear attention, gated softmax anchors.
#include "rope_dev.cuh"
#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {

void launch_linattn_combine(int BH, const float* ws_S, const float* ws_z, int splits, int D,
                            const float* S_prev, const float* z_prev, float* S_state,
                            float* z_state, float* S_f32, float* z_out, cudaStream_t st);

namespace {

constexpr int kTok = 32;  // tokens staged per step

__device__ __forceinline__ float sigmoid_precise(float x) { return 1.f / (1.f + expf(-x)); }

// Partial S[d][e] = sum_tok RoPE(phi K)[tok][d] V[tok][e] and z = sum phi K over
// this CTA's token range.
template <int D>
__global__ void __launch_bounds__(256)
    linattn_state_f32_kernel(const float* __restrict__ k, const float* __restrict__ v,
                             RopeDev rope, GridDev g, int splits, float* __restrict__ ws_S,
                             float* __restrict__ ws_z) {
  constexpr int ENT = D * D / 256 > 0 ? D * D / 256 : 1;
  __shared__ float kp[kTok][D], kphi[kTok][D], vs[kTok][D];
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int C = g.heads * D;
  const int chunks = (g.N + kTok - 1) / kTok;
  const int c0 = (int)((long long)split * chunks / splits);
  const int c1 = (int)((long long)(split + 1) * chunks / splits);
  float acc[ENT];
#pragma unroll
  for (int i = 0; i < ENT; ++i) acc[i] = 0.f;
  float zacc = 0.f;
  for (int ch = c0; ch < c1; ++ch) {
    const int n0 = ch * kTok;
    for (int p = tid; p < kTok * D / 2; p += 256) {
      const int tok = p / (D / 2), j = p - tok * (D / 2), n = n0 + tok;
      float x = 0.f, y = 0.f, vx = 0.f, vy = 0.f;
      if (n < g.N) {
        const size_t base = ((size_t)b * g.N + n) * C + (size_t)h * D + 2 * j;
        x = fmaxf(k[base], 0.f);
        y = fmaxf(k[base + 1], 0.f);
        vx = v[base];
        vy = v[base + 1];
      }
      kphi[tok][2 * j] = x;
      kphi[tok][2 * j + 1] = y;
      const float2 r = n < g.N ? rotate(x, y, rope_cs_global(rope, g, b, n, j)) : make_float2(0.f, 0.f);
      kp[tok][2 * j] = r.x;
      kp[tok][2 * j + 1] = r.y;
      vs[tok][2 * j] = vx;
      vs[tok][2 * j + 1] = vy;
    }
    __syncthreads();
    for (int tok = 0; tok < kTok; ++tok) {
#pragma unroll
      for (int i = 0; i < ENT; ++i) {
        const int idx = tid + 256 * i;
        if (idx < D * D) acc[i] = fmaf(kp[tok][idx / D], vs[tok][idx % D], acc[i]);
      }
      if (tid < D) zacc += kphi[tok][tid];
    }
    __syncthreads();
  }
  const size_t part = (size_t)(b * g.heads + h) * splits + split;
#pragma unroll
  for (int i = 0; i < ENT; ++i) {
    const int idx = tid + 256 * i;
    if (idx < D * D) ws_S[part * D * D + idx] = acc[i];
  }
  if (tid < D) ws_z[part * D + tid] = zacc;
}

// Y[n][e] = sigmoid(G) * (RoPE(phi Q_n) . S[:, e]) / (phi Q_n . z + eps)
template <int D>
__global__ void __launch_bounds__(256)
    linattn_out_f32_kernel(const float* __restrict__ q, const float* __restrict__ gt,
                           const float* __restrict__ S_all, const float* __restrict__ z_all,
                           RopeDev rope, GridDev g, float eps, float* __restrict__ y) {
  extern __shared__ float sm[];
  float* S = sm;                 // D*D
  float* z = S + D * D;          // D
  float* qp = z + D;             // kTok*D
  float* den = qp + kTok * D;    // kTok
  float* qphi = den + kTok;      // kTok*D
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int bh = b * g.heads + h, C = g.heads * D;
  const int n0 = blockIdx.x * kTok;
  for (int i = tid; i < D * D; i += 256) S[i] = S_all[(size_t)bh * D * D + i];
  for (int i = tid; i < D; i += 256) z[i] = z_all[(size_t)bh * D + i];
  for (int p = tid; p < kTok * D / 2; p += 256) {
    const int tok = p / (D / 2), j = p - tok * (D / 2), n = n0 + tok;
    float x = 0.f, yv = 0.f;
    if (n < g.N) {
      const size_t base = ((size_t)b * g.N + n) * C + (size_t)h * D + 2 * j;
      x = fmaxf(q[base], 0.f);
      yv = fmaxf(q[base + 1], 0.f);
    }
    qphi[tok * D + 2 * j] = x;
    qphi[tok * D + 2 * j + 1] = yv;
    const float2 r = n < g.N ? rotate(x, yv, rope_cs_global(rope, g, b, n, j)) : make_float2(0.f, 0.f);
    qp[tok * D + 2 * j] = r.x;
    qp[tok * D + 2 * j + 1] = r.y;
  }
  __syncthreads();
  if (tid < kTok) {
    float d = 0.f;
    for (int i = 0; i < D; ++i) d = fmaf(qphi[tid * D + i], z[i], d);
    den[tid] = d;
  }
  __syncthreads();
  for (int idx = tid; idx < kTok * D; idx += 256) {
    const int tok = idx / D, e = idx - tok * D, n = n0 + tok;
    if (n >= g.N) continue;
    float o = 0.f;
    for (int d = 0; d < D; ++d) o = fmaf(qp[tok * D + d], S[d * D + e], o);
    o = o / (den[tok] + eps);
    const size_t off = ((size_t)b * g.N + n) * C + (size_t)h * D + e;
    if (gt) o *= sigmoid_precise(gt[off]);
    y[off] = o;
  }
}

// RoPE of raw Q and K for the anchor (no ReLU); fp32 or bf16 outputs.
template <typename T>
__global__ void rope_rotate_kernel(const T* __restrict__ x, RopeDev rope, GridDev g, int D,
                                   float mul, T* __restrict__ out) {
  const long long pairs = (long long)g.N * g.heads * (D / 2);  // per batch entry
  const int b = blockIdx.y;
  for (long long p = blockIdx.x * (long long)blockDim.x + threadIdx.x; p < pairs;
       p += (long long)gridDim.x * blockDim.x) {
    const int j = (int)(p % (D / 2));
    const long long rest = p / (D / 2);
    const int h = (int)(rest % g.heads);
    const int n = (int)(rest / g.heads);
    const size_t off = ((size_t)b * g.N + n) * g.heads * D + (size_t)h * D + 2 * j;
    float a, c;
    if constexpr (sizeof(T) == 4) {
      a = x[off];
      c = x[off + 1];
    } else {
      a = __bfloat162float(x[off]);
      c = __bfloat162float(x[off + 1]);
    }
    float2 r = rope.cos_t ? rotate(a, c, rope_cs_global(rope, g, b, n, j)) : make_float2(a, c);
    r.x *= mul;
    r.y *= mul;
    if constexpr (sizeof(T) == 4) {
      out[off] = r.x;
      out[off + 1] = r.y;
    } else {
      out[off] = __float2bfloat16_rn(r.x);
      out[off + 1] = __float2bfloat16_rn(r.y);
    }
  }
}

// bf16 form: a thread owns one 16-byte chunk position within a head (four
// rotary pairs) of one token and walks that position through every head of
// the token, so the token's (cos, sin) for its four pairs are read once and
// used heads times; 16 threads cover one token's chunk positions (D = 128)
// and a warp two tokens, each a contiguous 256-byte run per head.  Loads of
// eight heads are in flight before the first rotation.
constexpr int kRopeHeadsInFlight = 8;
__global__ void __launch_bounds__(256)
    rope_rotate_bf16x8_kernel(const uint4* __restrict__ x, RopeDev rope, GridDev g, int D,
                              float mul, uint4* __restrict__ out) {
  const int b = blockIdx.y;
  const int cpd = D / 8;                       // chunk positions per head
  const int tpb = blockDim.x / cpd;            // tokens per block and pass
  const int cl = threadIdx.x % cpd, tl = threadIdx.x / cpd;
  const int chunks = g.heads * cpd;            // per token
  const int hw = g.H * g.W;
  const int j0 = cl * 4;                       // first rotary pair of the chunk
  int ax[4], col[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int j = j0 + k;
    ax[k] = j < rope.n_t ? 0 : (j < rope.n_t + rope.n_h ? 1 : 2);
    col[k] = ax[k] == 0 ? j : (ax[k] == 1 ? j - rope.n_t : j - rope.n_t - rope.n_h);
  }
  for (int n = blockIdx.x * tpb + tl; n < g.N; n += gridDim.x * tpb) {
    float2 cs[4];
    if (rope.cos_t) {
      const int t = n / hw, rem = n - t * hw, hh = rem / g.W, ww = rem - hh * g.W;
      const int tt = g.t_offset + b * g.t_stride + t;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int pos = ax[k] == 0 ? tt : (ax[k] == 1 ? hh : ww);
        const int np = ax[k] == 0 ? rope.n_t : (ax[k] == 1 ? rope.n_h : rope.n_w);
        const float* ct = ax[k] == 0 ? rope.cos_t : (ax[k] == 1 ? rope.cos_h : rope.cos_w);
        const float* st = ax[k] == 0 ? rope.sin_t : (ax[k] == 1 ? rope.sin_h : rope.sin_w);
        cs[k] = make_float2(__ldg(ct + pos * np + col[k]), __ldg(st + pos * np + col[k]));
      }
    }
    const size_t row = ((size_t)b * g.N + n) * chunks + cl;
    for (int h0 = 0; h0 < g.heads; h0 += kRopeHeadsInFlight) {
      uint4 raw[kRopeHeadsInFlight];
#pragma unroll
      for (int u = 0; u < kRopeHeadsInFlight; ++u)
        raw[u] = h0 + u < g.heads ? x[row + (size_t)(h0 + u) * cpd] : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < kRopeHeadsInFlight; ++u) {
        if (h0 + u >= g.heads) break;
        uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float2 v = bf2_to_f2(w[k]);
          if (rope.cos_t) v = rotate(v.x, v.y, cs[k]);
          w[k] = f2_to_bf2(v.x * mul, v.y * mul);
        }
        out[row + (size_t)(h0 + u) * cpd] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

// One thread per (query, head, batch): online softmax over all keys in fp32.
template <int D>
__global__ void __launch_bounds__(128)
    anchor_f32_kernel(const float* __restrict__ qr, const float* __restrict__ kr,
                      const float* __restrict__ v, const float* __restrict__ gt, GridDev g,
                      float scale, float* __restrict__ y) {
  __shared__ float ks[32][D], vsm[32][D];
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int i = blockIdx.x * blockDim.x + tid;
  const int C = g.heads * D;
  float qv[D], acc[D];
  const bool active = i < g.N;
#pragma unroll
  for (int d = 0; d < D; ++d) {
    qv[d] = active ? qr[((size_t)b * g.N + i) * C + (size_t)h * D + d] * scale : 0.f;
    acc[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j0 = 0; j0 < g.N; j0 += 32) {
    for (int p = tid; p < 32 * D; p += blockDim.x) {
      const int jj = p / D, d = p - jj * D, j = j0 + jj;
      const size_t off = ((size_t)b * g.N + j) * C + (size_t)h * D + d;
      ks[jj][d] = j < g.N ? kr[off] : 0.f;
      vsm[jj][d] = j < g.N ? v[off] : 0.f;
    }
    __syncthreads();
    const int jn = min(32, g.N - j0);
    for (int jj = 0; jj < jn; ++jj) {
      float s = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) s = fmaf(qv[d], ks[jj][d], s);
      const float mn = fmaxf(m, s);
      const float corr = expf(m - mn);
      const float p = expf(s - mn);
      l = l * corr + p;
#pragma unroll
      for (int d = 0; d < D; ++d) acc[d] = fmaf(p, vsm[jj][d], acc[d] * corr);
      m = mn;
    }
    __syncthreads();
  }
  if (!active) return;
  const float inv = 1.f / l;
#pragma unroll
  for (int d = 0; d < D; ++d) {
    const size_t off = ((size_t)b * g.N + i) * C + (size_t)h * D + d;
    float o = acc[d] * inv;
    if (gt) o *= sigmoid_precise(gt[off]);
    y[off] = o;
  }
}

template <int D>
void run_partials(const sana_shape& s, const float* k, const float* v, const RopeDev& rope,
                  const GridDev& g, int splits, float* ws_S, float* ws_z, cudaStream_t st) {
  linattn_state_f32_kernel<D><<<dim3(splits, s.heads, s.B), 256, 0, st>>>(k, v, rope, g, splits,
                                                                          ws_S, ws_z);
}

template <int D>
void run_state(const sana_shape& s, const float* k, const float* v, const RopeDev& rope,
               const GridDev& g, int splits, const float* S_prev, const float* z_prev,
               float* S_state, float* z_state, float* ws_S, float* ws_z, float* S_f32,
               float* z_comb, cudaStream_t st) {
  run_partials<D>(s, k, v, rope, g, splits, ws_S, ws_z, st);
  launch_linattn_combine(s.B * s.heads, ws_S, ws_z, splits, D, S_prev, z_prev, S_state, z_state,
                         S_f32, z_comb, st);
}

template <int D>
void run_apply(const sana_shape& s, const float* q, const float* gt, const RopeDev& rope,
               const GridDev& g, const float* S_f32, const float* z, float eps, float* out,
               cudaStream_t st) {
  const size_t smem = sizeof(float) * ((size_t)D * D + D + 2 * kTok * D + kTok);
  cudaFuncSetAttribute(linattn_out_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  linattn_out_f32_kernel<D><<<dim3((g.N + kTok - 1) / kTok, s.heads, s.B), 256, smem, st>>>(
      q, gt, S_f32, z, rope, g, eps, out);
}

template <int D>
void run_anchor(const sana_shape& s, const float* qr, const float* kr, const float* v,
                const float* gt, const GridDev& g, float scale, float* out, cudaStream_t st) {
  anchor_f32_kernel<D><<<dim3((g.N + 127) / 128, s.heads, s.B), 128, 0, st>>>(qr, kr, v, gt, g,
                                                                            scale, out);
}

}  // namespace

int linattn_f32_splits(const sana_shape& s, int N) {
  const int chunks = (N + kTok - 1) / kTok;
  int sp = kNumSMs / (s.B * s.heads);
  if (sp < 1) sp = 1;
  if (sp > chunks) sp = chunks;
  return sp;
}

sana_status linattn_f32_state(const sana_shape& s, const float* k, const float* v,
                              const RopeDev& rope, const GridDev& g, int splits,
                              const float* S_prev, const float* z_prev, float* S_state,
                              float* z_state, float* ws_S, float* ws_z, float* S_f32,
                              float* z_comb, cudaStream_t st) {
  switch (s.head_dim) {
    case 16: run_state<16>(s, k, v, rope, g, splits, S_prev, z_prev, S_state, z_state, ws_S, ws_z, S_f32, z_comb, st); break;
    case 32: run_state<32>(s, k, v, rope, g, splits, S_prev, z_prev, S_state, z_state, ws_S, ws_z, S_f32, z_comb, st); break;
    case 64: run_state<64>(s, k, v, rope, g, splits, S_prev, z_prev, S_state, z_state, ws_S, ws_z, S_f32, z_comb, st); break;
    case 128: run_state<128>(s, k, v, rope, g, splits, S_prev, z_prev, S_state, z_state, ws_S, ws_z, S_f32, z_comb, st); break;
    default: return fail(SANA_ERR_UNSUPPORTED, "fp32 linear attention: head_dim %d", s.head_dim);
  }
  return check_launch("linattn fp32 state kernels");
}

sana_status linattn_f32_partials(const sana_shape& s, const float* k, const float* v,
                                 const RopeDev& rope, const GridDev& g, int splits, float* ws_S,
                                 float* ws_z, cudaStream_t st) {
  switch (s.head_dim) {
    case 16: run_partials<16>(s, k, v, rope, g, splits, ws_S, ws_z, st); break;
    case 32: run_partials<32>(s, k, v, rope, g, splits, ws_S, ws_z, st); break;
    case 64: run_partials<64>(s, k, v, rope, g, splits, ws_S, ws_z, st); break;
    case 128: run_partials<128>(s, k, v, rope, g, splits, ws_S, ws_z, st); break;
    default: return fail(SANA_ERR_UNSUPPORTED, "fp32 linear attention: head_dim %d", s.head_dim);
  }
  return check_launch("linattn_state_f32_kernel");
}

sana_status linattn_f32_apply(const sana_shape& s, const float* q, const float* gt,
                              const RopeDev& rope, const GridDev& g, const float* S_f32,
                              const float* z, float eps, float* out, cudaStream_t st) {
  switch (s.head_dim) {
    case 16: run_apply<16>(s, q, gt, rope, g, S_f32, z, eps, out, st); break;
    case 32: run_apply<32>(s, q, gt, rope, g, S_f32, z, eps, out, st); break;
    case 64: run_apply<64>(s, q, gt, rope, g, S_f32, z, eps, out, st); break;
    case 128: run_apply<128>(s, q, gt, rope, g, S_f32, z, eps, out, st); break;
    default: return fail(SANA_ERR_UNSUPPORTED, "fp32 linear attention: head_dim %d", s.head_dim);
  }
  return check_launch("linattn_out_f32_kernel");
}

// Rotate (and scale) Q or K for the anchor; bf16 or fp32.
sana_status rope_rotate_run(const void* x, bool bf16, const RopeDev* rope, const GridDev& g,
                            int B, int D, float mul, void* out, cudaStream_t st) {
  RopeDev r{};
  if (rope) r = *rope;
  const long long pairs = (long long)g.N * g.heads * (D / 2);
  int blocks = (int)((pairs + 255) / 256);
  if (blocks > 4 * kNumSMs * 8) blocks = 4 * kNumSMs * 8;
  if (blocks < 1) blocks = 1;
  if (bf16 && D % 8 == 0 && D <= 256) {
    const int cpd = D / 8;
    const int threads = 256 / cpd * cpd;       // whole tokens per block
    const int tpb = threads / cpd;
    long long nb = ((long long)g.N + tpb - 1) / tpb;
    const long long cap = (long long)kNumSMs * 8 / (B > 0 ? B : 1);
    if (nb > cap) nb = cap > 0 ? cap : 1;
    rope_rotate_bf16x8_kernel<<<dim3((unsigned)nb, B), threads, 0, st>>>(
        static_cast<const uint4*>(x), r, g, D, mul, static_cast<uint4*>(out));
  } else if (bf16)
    rope_rotate_kernel<__nv_bfloat16><<<dim3(blocks, B), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), r, g, D, mul, static_cast<__nv_bfloat16*>(out));
  else
    rope_rotate_kernel<float><<<dim3(blocks, B), 256, 0, st>>>(static_cast<const float*>(x), r, g,
                                                               D, mul, static_cast<float*>(out));
  return check_launch("rope_rotate_kernel");
}

sana_status anchor_f32_run(const sana_shape& s, const float* qr, const float* kr, const float* v,
                           const float* gt, const GridDev& g, float scale, float* out,
                           cudaStream_t st) {
  switch (s.head_dim) {
    case 16: run_anchor<16>(s, qr, kr, v, gt, g, scale, out, st); break;
    case 32: run_anchor<32>(s, qr, kr, v, gt, g, scale, out, st); break;
    case 64: run_anchor<64>(s, qr, kr, v, gt, g, scale, out, st); break;
    case 128: run_anchor<128>(s, qr, kr, v, gt, g, scale, out, st); break;
    default: return fail(SANA_ERR_UNSUPPORTED, "fp32 anchor: head_dim %d", s.head_dim);
  }
  return check_launch("anchor_f32_kernel");
}

}  // namespace sana
