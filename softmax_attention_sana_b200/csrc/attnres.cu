// Block Attention Residuals router and RMSNorm.
//
//   "SANA-Video 2.0" (hyper.ai summary), Method, AttnRes equation:
//     h_l = sum_i alpha_{i->l} v_i,  alpha = softmax_i((w + phi_tau(t))^T RMSNorm(v_i)),
//   with the timestep term phi_tau(t) = 0 (Experiments: timestep-free router)
//   and one router query per sublayer kind shared across depth.
//
// One CTA per token (grid-stride): thread i owns elements [8i, 8i + 8) of every
// source, so each source is read from HBM exactly once; the per-source sums
// (sum v^2, w.v) are reduced with warp shuffles and one shared-memory pass.
#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {
namespace {

constexpr int kMaxSources = 16;

template <typename T>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = *reinterpret_cast<const uint4*>(p); }
  __device__ __forceinline__ void to_float(float (&f)[8]) const {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = bf2_to_f2(w[i]);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float (&f)[8]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(f2_to_bf2(f[0], f[1]), f2_to_bf2(f[2], f[3]),
                                              f2_to_bf2(f[4], f[5]), f2_to_bf2(f[6], f[7]));
  }
};
template <>
struct Vec8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = *reinterpret_cast<const float4*>(p);
    b = *reinterpret_cast<const float4*>(p + 4);
  }
  __device__ __forceinline__ void to_float(float (&f)[8]) const {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
  __device__ __forceinline__ static void store(float* p, const float (&f)[8]) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
  }
};

struct SourcePtrs {
  const void* p[kMaxSources];
};

// Block-wide sum of `n` per-thread values (n <= 2 * kMaxSources), fixed order.
template <int NV>
__device__ __forceinline__ void block_sum(float (&v)[NV], int n, float* red, int nwarps) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    if (i >= n) break;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
  }
  __syncthreads();  // red[] may still be read from the previous token
  if (lane == 0)
    for (int i = 0; i < n; ++i) red[i * 32 + warp] = v[i];
  __syncthreads();
  for (int i = 0; i < n; ++i) {
    float acc = 0.f;
    for (int w = 0; w < nwarps; ++w) acc += red[i * 32 + w];
    v[i] = acc;
  }
}

// Up to 4 sources: any C <= 8192 (1024 threads); up to 16 sources: C <= 4096.
template <typename T, int MAXS>
__global__ void __launch_bounds__(MAXS <= 4 ? 1024 : 512)
    attnres_kernel(SourcePtrs src, int S, long long tokens, int C, const float* __restrict__ w,
                   float eps, T* __restrict__ h_out, float* __restrict__ alpha_out,
                   T* __restrict__ hn_out) {
  __shared__ float red[2 * MAXS * 32 + 32];
  const int tid = threadIdx.x, nwarps = blockDim.x >> 5;
  const int c0 = tid * 8;
  const bool act = c0 < C;
  float wv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) wv[i] = act ? w[c0 + i] : 0.f;
  const float invC = 1.f / (float)C;
  for (long long tok = blockIdx.x; tok < tokens; tok += gridDim.x) {
    const size_t off = (size_t)tok * C + c0;
    Vec8<T> x[MAXS];
    float sums[2 * MAXS];
#pragma unroll
    for (int s = 0; s < MAXS; ++s) {
      if (s >= S) break;
      if (act) x[s].load(static_cast<const T*>(src.p[s]) + off);
    }
#pragma unroll
    for (int s = 0; s < MAXS; ++s) {
      sums[2 * s] = 0.f;
      sums[2 * s + 1] = 0.f;
      if (s >= S || !act) continue;
      float f[8];
      x[s].to_float(f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        sums[2 * s] = fmaf(f[i], f[i], sums[2 * s]);
        sums[2 * s + 1] = fmaf(wv[i], f[i], sums[2 * s + 1]);
      }
    }
    block_sum<2 * MAXS>(sums, 2 * S, red, nwarps);
    // logits, softmax over sources
    float m = -INFINITY;
    float logit[MAXS];
#pragma unroll
    for (int s = 0; s < MAXS; ++s) {
      if (s >= S) break;
      logit[s] = sums[2 * s + 1] * rsqrtf(sums[2 * s] * invC + eps);
      m = fmaxf(m, logit[s]);
    }
    float den = 0.f;
#pragma unroll
    for (int s = 0; s < MAXS; ++s) {
      if (s >= S) break;
      logit[s] = expf(logit[s] - m);
      den += logit[s];
    }
    const float inv = 1.f / den;
    float hv[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int s = 0; s < MAXS; ++s) {
      if (s >= S) break;
      const float a = logit[s] * inv;
      if (alpha_out && tid == 0) alpha_out[(size_t)tok * S + s] = a;
      if (!act) continue;
      float f[8];
      x[s].to_float(f);
#pragma unroll
      for (int i = 0; i < 8; ++i) hv[i] = fmaf(a, f[i], hv[i]);
    }
    if (act && h_out) Vec8<T>::store(h_out + off, hv);
    if (hn_out) {  // fused pre-norm of the routed representation
      float ss[1] = {0.f};
      if (act)
#pragma unroll
        for (int i = 0; i < 8; ++i) ss[0] = fmaf(hv[i], hv[i], ss[0]);
      block_sum<1>(ss, 1, red, nwarps);
      const float r = rsqrtf(ss[0] * invC + eps);
#pragma unroll
      for (int i = 0; i < 8; ++i) hv[i] *= r;
      if (act) Vec8<T>::store(hn_out + off, hv);
    }
  }
}

// Warp per token, the token's row of every source held in registers (bf16,
// NS <= 4 sources, C <= 256 * CH): one HBM read of each source, warp-shuffle
// reductions only, several tokens in flight per SM.
template <int NS, int CH>
__global__ void __launch_bounds__(256)
    attnres_warp_kernel(SourcePtrs src, long long tokens, int C, const float* __restrict__ w,
                        float eps, __nv_bfloat16* __restrict__ h_out, float* __restrict__ alpha_out,
                        __nv_bfloat16* __restrict__ hn_out) {
  const int lane = threadIdx.x & 31;
  const long long warp0 = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  const float invC = 1.f / (float)C;
  for (long long tok = warp0; tok < tokens; tok += nwarps) {
    const size_t row = (size_t)tok * C;
    uint4 x[NS][CH];
#pragma unroll
    for (int s = 0; s < NS; ++s)
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int col = (c * 32 + lane) * 8;
        x[s][c] = col < C ? *reinterpret_cast<const uint4*>(
                                static_cast<const __nv_bfloat16*>(src.p[s]) + row + col)
                          : make_uint4(0, 0, 0, 0);
      }
    float ss[NS], sw[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) ss[s] = sw[s] = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (c * 32 + lane) * 8;
      if (col >= C) continue;
      const float4 w0 = *reinterpret_cast<const float4*>(w + col);
      const float4 w1 = *reinterpret_cast<const float4*>(w + col + 4);
      const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        const uint32_t u[4] = {x[s][c].x, x[s][c].y, x[s][c].z, x[s][c].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = bf2_to_f2(u[i]);
          ss[s] = fmaf(f.x, f.x, fmaf(f.y, f.y, ss[s]));
          sw[s] = fmaf(wv[2 * i], f.x, fmaf(wv[2 * i + 1], f.y, sw[s]));
        }
      }
    }
    float a[NS], m = -INFINITY;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ss[s] += __shfl_xor_sync(0xffffffffu, ss[s], o);
        sw[s] += __shfl_xor_sync(0xffffffffu, sw[s], o);
      }
      a[s] = sw[s] * rsqrtf(ss[s] * invC + eps);
      m = fmaxf(m, a[s]);
    }
    float den = 0.f;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      a[s] = expf(a[s] - m);
      den += a[s];
    }
    const float inv = 1.f / den;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      a[s] *= inv;
      if (alpha_out && lane == s) alpha_out[(size_t)tok * NS + s] = a[s];
    }
    // h = sum_s a_s v_s, chunk by chunk from the registers
    float hss = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (c * 32 + lane) * 8;
      float hv[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        const uint32_t u[4] = {x[s][c].x, x[s][c].y, x[s][c].z, x[s][c].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = bf2_to_f2(u[i]);
          hv[2 * i] = fmaf(a[s], f.x, hv[2 * i]);
          hv[2 * i + 1] = fmaf(a[s], f.y, hv[2 * i + 1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) hss = fmaf(hv[i], hv[i], hss);
      if (h_out && col < C) Vec8<__nv_bfloat16>::store(h_out + row + col, hv);
    }
    if (hn_out) {  // fused pre-norm of the routed representation (h recomputed)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) hss += __shfl_xor_sync(0xffffffffu, hss, o);
      const float rn = rsqrtf(hss * invC + eps);
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int col = (c * 32 + lane) * 8;
        if (col >= C) continue;
        float hv[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
        for (int s = 0; s < NS; ++s) {
          const uint32_t u[4] = {x[s][c].x, x[s][c].y, x[s][c].z, x[s][c].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = bf2_to_f2(u[i]);
            hv[2 * i] = fmaf(a[s], f.x, hv[2 * i]);
            hv[2 * i + 1] = fmaf(a[s], f.y, hv[2 * i + 1]);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) hv[i] *= rn;
        Vec8<__nv_bfloat16>::store(hn_out + row + col, hv);
      }
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(1024)
    rmsnorm_kernel(const T* __restrict__ x, long long rows, int C, float eps, T* __restrict__ y) {
  __shared__ float red[64];
  const int tid = threadIdx.x, nwarps = blockDim.x >> 5;
  const int c0 = tid * 8;
  const bool act = c0 < C;
  for (long long row = blockIdx.x; row < rows; row += gridDim.x) {
    const size_t off = (size_t)row * C + c0;
    Vec8<T> v;
    float f[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (act) {
      v.load(x + off);
      v.to_float(f);
    }
    float ss[1] = {0.f};
#pragma unroll
    for (int i = 0; i < 8; ++i) ss[0] = fmaf(f[i], f[i], ss[0]);
    block_sum<1>(ss, 1, red, nwarps);
    const float r = rsqrtf(ss[0] / (float)C + eps);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] *= r;
    if (act) Vec8<T>::store(y + off, f);
  }
}

// ---------------------------------------------------------------- backward
// Chain rule through the route as written (the pages print no backward):
//   r_s = sqrt(mean v_s^2 + eps),  l_s = w . v_s / r_s,  alpha = softmax(l),
//   d alpha_s = dh . v_s,  d l_s = alpha_s (d alpha_s - sum_t alpha_t d alpha_t),
//   d v_s = alpha_s dh + (d l_s / r_s) w - (d l_s l_s / (C r_s^2)) v_s,
//   d w = sum over tokens of sum_s (d l_s / r_s) v_s.
// Two warps per token (a warp pair of the CTA), each holding one half of the
// token's columns of every source in registers between the reductions and
// the gradient pass; the pair adds its partial sums (sum v^2, w.v, dh.v per
// source) through shared memory behind a named barrier of the pair, half 0's
// first (fixed order).  Halving the registers per thread puts two CTAs, 16
// warps, on an SM: twice the loads in flight of one warp per token.  Each
// warp adds its share of d w to its own shared-memory row; the CTA writes the
// fixed-order sum of its rows and attnres_dw_reduce_kernel adds the CTA rows
// in order, so d w is bit-reproducible.
constexpr int kBwdWarps = 8;   // 4 pairs
constexpr int kBwdPairs = 4;

template <int NS, int CH>
__global__ void __launch_bounds__(256, 2)
    attnres_bwd_kernel(SourcePtrs src, const __nv_bfloat16* __restrict__ dh, long long tokens,
                       int C, const float* __restrict__ w, float eps, SourcePtrs dsrc,
                       float* __restrict__ dw_part) {
  extern __shared__ float dw_rows[];  // [kBwdWarps][C]
  __shared__ float xch[2][kBwdPairs][2][3 * NS];
  constexpr int CHH = (CH + 1) / 2;   // chunks of 256 columns per half
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int pair = wib & (kBwdPairs - 1), half = wib / kBwdPairs;
  float* myrow = dw_rows + (size_t)wib * C;
  for (int i = lane; i < C; i += 32) myrow[i] = 0.f;
  __syncwarp();
  const long long npairs = (long long)gridDim.x * kBwdPairs;
  const float invC = 1.f / (float)C;
  int par = 0;
  for (long long tok = (long long)blockIdx.x * kBwdPairs + pair; tok < tokens;
       tok += npairs, par ^= 1) {
    const size_t row = (size_t)tok * C;
    uint4 x[NS][CHH];
#pragma unroll
    for (int s = 0; s < NS; ++s)
#pragma unroll
      for (int c = 0; c < CHH; ++c) {
        const int col = ((half * CHH + c) * 32 + lane) * 8;
        x[s][c] = col < C ? *reinterpret_cast<const uint4*>(
                                static_cast<const __nv_bfloat16*>(src.p[s]) + row + col)
                          : make_uint4(0, 0, 0, 0);
      }
    float ss[NS], sw[NS], sd[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) ss[s] = sw[s] = sd[s] = 0.f;
#pragma unroll
    for (int c = 0; c < CHH; ++c) {
      const int col = ((half * CHH + c) * 32 + lane) * 8;
      if (col >= C) continue;
      const float4 w0 = *reinterpret_cast<const float4*>(w + col);
      const float4 w1 = *reinterpret_cast<const float4*>(w + col + 4);
      const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      float dv[8];
      Vec8<__nv_bfloat16> dhc;
      dhc.load(dh + row + col);
      dhc.to_float(dv);
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        const uint32_t u[4] = {x[s][c].x, x[s][c].y, x[s][c].z, x[s][c].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = bf2_to_f2(u[i]);
          ss[s] = fmaf(f.x, f.x, fmaf(f.y, f.y, ss[s]));
          sw[s] = fmaf(wv[2 * i], f.x, fmaf(wv[2 * i + 1], f.y, sw[s]));
          sd[s] = fmaf(dv[2 * i], f.x, fmaf(dv[2 * i + 1], f.y, sd[s]));
        }
      }
    }
#pragma unroll
    for (int s = 0; s < NS; ++s) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ss[s] += __shfl_xor_sync(0xffffffffu, ss[s], o);
        sw[s] += __shfl_xor_sync(0xffffffffu, sw[s], o);
        sd[s] += __shfl_xor_sync(0xffffffffu, sd[s], o);
      }
    }
    // the pair's halves meet: half 0's partials plus half 1's, in that order
    if (lane == 0) {
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        xch[par][pair][half][3 * s] = ss[s];
        xch[par][pair][half][3 * s + 1] = sw[s];
        xch[par][pair][half][3 * s + 2] = sd[s];
      }
    }
    named_bar_sync(1 + pair, 64);
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      ss[s] = xch[par][pair][0][3 * s] + xch[par][pair][1][3 * s];
      sw[s] = xch[par][pair][0][3 * s + 1] + xch[par][pair][1][3 * s + 1];
      sd[s] = xch[par][pair][0][3 * s + 2] + xch[par][pair][1][3 * s + 2];
    }
    float a[NS], l[NS], r[NS], m = -INFINITY;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      r[s] = sqrtf(ss[s] * invC + eps);
      l[s] = sw[s] / r[s];
      m = fmaxf(m, l[s]);
    }
    float den = 0.f;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      a[s] = expf(l[s] - m);
      den += a[s];
    }
    float adot = 0.f;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      a[s] /= den;
      adot = fmaf(a[s], sd[s], adot);
    }
    float cw[NS], cv[NS];  // d v_s = a_s dh + cw_s w + cv_s v_s
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const float dl = a[s] * (sd[s] - adot);
      cw[s] = dl / r[s];
      cv[s] = -dl * l[s] * invC / (r[s] * r[s]);
    }
#pragma unroll
    for (int c = 0; c < CHH; ++c) {
      const int col = ((half * CHH + c) * 32 + lane) * 8;
      if (col >= C) continue;
      const float4 w0 = *reinterpret_cast<const float4*>(w + col);
      const float4 w1 = *reinterpret_cast<const float4*>(w + col + 4);
      const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      float dv[8];
      Vec8<__nv_bfloat16> dhc;
      dhc.load(dh + row + col);
      dhc.to_float(dv);
      float dwv[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        const uint32_t u[4] = {x[s][c].x, x[s][c].y, x[s][c].z, x[s][c].w};
        float g[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = bf2_to_f2(u[i]);
          g[2 * i] = fmaf(cv[s], f.x, fmaf(cw[s], wv[2 * i], a[s] * dv[2 * i]));
          g[2 * i + 1] = fmaf(cv[s], f.y, fmaf(cw[s], wv[2 * i + 1], a[s] * dv[2 * i + 1]));
          dwv[2 * i] = fmaf(cw[s], f.x, dwv[2 * i]);
          dwv[2 * i + 1] = fmaf(cw[s], f.y, dwv[2 * i + 1]);
        }
        Vec8<__nv_bfloat16>::store(static_cast<__nv_bfloat16*>(const_cast<void*>(dsrc.p[s])) + row + col, g);
      }
      float4* acc = reinterpret_cast<float4*>(myrow + col);
      const float4 a0 = acc[0], a1 = acc[1];
      acc[0] = make_float4(a0.x + dwv[0], a0.y + dwv[1], a0.z + dwv[2], a0.w + dwv[3]);
      acc[1] = make_float4(a1.x + dwv[4], a1.y + dwv[5], a1.z + dwv[6], a1.w + dwv[7]);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < kBwdWarps; ++k) acc += dw_rows[k * C + c];
    dw_part[(size_t)blockIdx.x * C + c] = acc;
  }
}

__global__ void __launch_bounds__(256)
    attnres_dw_reduce_kernel(const float* __restrict__ dw_part, int nblocks, int C,
                             float* __restrict__ dw) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  float acc = 0.f;
  for (int b = 0; b < nblocks; ++b) acc += dw_part[(size_t)b * C + c];
  dw[c] = acc;
}

int attnres_bwd_blocks(long long tokens) {
  const long long want = (tokens + kBwdPairs - 1) / kBwdPairs;
  const long long cap = 2LL * kNumSMs;  // two CTAs of 8 warps (4 token pairs) per SM
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

template <int NS, int CH>
void bwd_launch(const SourcePtrs& sp, const void* dh, long long tokens, int C, const float* w,
                float eps, const SourcePtrs& dsp, float* dw_part, cudaStream_t st) {
  const int blocks = attnres_bwd_blocks(tokens);
  const int smem = kBwdWarps * C * (int)sizeof(float);
  cudaFuncSetAttribute(attnres_bwd_kernel<NS, CH>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  attnres_bwd_kernel<NS, CH><<<blocks, 256, smem, st>>>(
      sp, static_cast<const __nv_bfloat16*>(dh), tokens, C, w, eps, dsp, dw_part);
}

template <int CH>
void bwd_launch_s(const SourcePtrs& sp, int S, const void* dh, long long tokens, int C,
                  const float* w, float eps, const SourcePtrs& dsp, float* dw_part, cudaStream_t st) {
  switch (S) {
    case 1: bwd_launch<1, CH>(sp, dh, tokens, C, w, eps, dsp, dw_part, st); break;
    case 2: bwd_launch<2, CH>(sp, dh, tokens, C, w, eps, dsp, dw_part, st); break;
    case 3: bwd_launch<3, CH>(sp, dh, tokens, C, w, eps, dsp, dw_part, st); break;
    default: bwd_launch<4, CH>(sp, dh, tokens, C, w, eps, dsp, dw_part, st); break;
  }
}

int threads_for(int C) {
  int t = ((C / 8) + 31) / 32 * 32;
  return t < 32 ? 32 : t;
}

template <int NS, int CH>
void warp_launch(const SourcePtrs& sp, long long tokens, int C, const float* w, float eps, void* h,
                 float* alpha, void* hn, cudaStream_t st) {
  const long long warps = tokens < (long long)kNumSMs * 64 ? tokens : (long long)kNumSMs * 64;
  attnres_warp_kernel<NS, CH><<<(int)((warps + 7) / 8), 256, 0, st>>>(
      sp, tokens, C, w, eps, static_cast<__nv_bfloat16*>(h), alpha,
      static_cast<__nv_bfloat16*>(hn));
}

template <int CH>
bool warp_launch_s(const SourcePtrs& sp, int S, long long tokens, int C, const float* w, float eps,
                   void* h, float* alpha, void* hn, cudaStream_t st) {
  switch (S) {
    case 1: warp_launch<1, CH>(sp, tokens, C, w, eps, h, alpha, hn, st); return true;
    case 2: warp_launch<2, CH>(sp, tokens, C, w, eps, h, alpha, hn, st); return true;
    case 3: warp_launch<3, CH>(sp, tokens, C, w, eps, h, alpha, hn, st); return true;
    case 4: warp_launch<4, CH>(sp, tokens, C, w, eps, h, alpha, hn, st); return true;
  }
  return false;
}

// bf16, <= 4 sources, C a multiple of 256 up to 4096: warp per token.
bool launch_attnres_warp(const SourcePtrs& sp, int S, long long tokens, int C, const float* w,
                         float eps, void* h, float* alpha, void* hn, cudaStream_t st) {
  const int ch = C / 256;
  if (ch <= 4) return warp_launch_s<4>(sp, S, tokens, C, w, eps, h, alpha, hn, st);
  if (ch <= 8) return warp_launch_s<8>(sp, S, tokens, C, w, eps, h, alpha, hn, st);
  if (ch <= 12) return warp_launch_s<12>(sp, S, tokens, C, w, eps, h, alpha, hn, st);
  return warp_launch_s<16>(sp, S, tokens, C, w, eps, h, alpha, hn, st);
}

template <typename T>
void launch_attnres(const SourcePtrs& sp, int S, long long tokens, int C, const float* w, float eps,
                    void* h, float* alpha, void* hn, cudaStream_t st) {
  if constexpr (sizeof(T) == 2) {
    if (S <= 4 && C <= 4096 && C % 256 == 0 && launch_attnres_warp(sp, S, tokens, C, w, eps, h,
                                                                    alpha, hn, st))
      return;
  }
  const int threads = threads_for(C);
  long long blocks = tokens < (long long)kNumSMs * 16 ? tokens : (long long)kNumSMs * 16;
  if (blocks < 1) blocks = 1;
  T* ho = static_cast<T*>(h);
  T* hno = static_cast<T*>(hn);
  if (S <= 4)
    attnres_kernel<T, 4><<<(int)blocks, threads, 0, st>>>(sp, S, tokens, C, w, eps, ho, alpha, hno);
  else
    attnres_kernel<T, kMaxSources><<<(int)blocks, threads, 0, st>>>(sp, S, tokens, C, w, eps, ho,
                                                                   alpha, hno);
}

}  // namespace

sana_status attnres_run(int B, long long N, int C, sana_dtype dt, const void* const* sources,
                        int S, const float* w, float eps, void* h, float* alpha, bool normed_out,
                        void* h_norm, cudaStream_t st) {
  if (S < 1 || S > kMaxSources) return fail(SANA_ERR_UNSUPPORTED, "attnres: %d sources (1..16)", S);
  if (C % 8 != 0 || C > (S <= 4 ? 8192 : 4096))
    return fail(SANA_ERR_UNSUPPORTED, "attnres: C=%d with %d sources (C %% 8 == 0; C <= 8192 for <= 4 sources, <= 4096 above)", C, S);
  SourcePtrs sp{};
  for (int i = 0; i < S; ++i) sp.p[i] = sources[i];
  const long long tokens = (long long)B * N;
  if (tokens == 0) return SANA_OK;
  void* hn = normed_out ? h_norm : nullptr;
  if (dt == SANA_BF16) launch_attnres<__nv_bfloat16>(sp, S, tokens, C, w, eps, h, alpha, hn, st);
  else launch_attnres<float>(sp, S, tokens, C, w, eps, h, alpha, hn, st);
  return check_launch("attnres_kernel");
}

size_t attnres_bwd_ws_bytes(long long tokens, int C) {
  return align_up((size_t)attnres_bwd_blocks(tokens) * C * sizeof(float), 256);
}

sana_status attnres_bwd_run(long long tokens, int C, const void* const* sources, int S,
                            const float* w, float eps, const void* dh, void* const* d_sources,
                            float* dw, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (S < 1 || S > 4 || C % 256 != 0 || C > 4096)
    return fail(SANA_ERR_UNSUPPORTED, "attnres backward: %d sources, C=%d (1..4 sources, C a multiple of 256 up to 4096)", S, C);
  if (tokens == 0) {
    cudaMemsetAsync(dw, 0, (size_t)C * sizeof(float), st);
    return check_launch("attnres backward (no tokens)");
  }
  if (ws_bytes < attnres_bwd_ws_bytes(tokens, C))
    return fail(SANA_ERR_WORKSPACE, "attnres backward: workspace %zu < %zu bytes", ws_bytes,
                attnres_bwd_ws_bytes(tokens, C));
  SourcePtrs sp{}, dsp{};
  for (int i = 0; i < S; ++i) {
    sp.p[i] = sources[i];
    dsp.p[i] = d_sources[i];
  }
  float* dw_part = static_cast<float*>(ws);
  const int ch = C / 256;
  if (ch <= 4) bwd_launch_s<4>(sp, S, dh, tokens, C, w, eps, dsp, dw_part, st);
  else if (ch <= 8) bwd_launch_s<8>(sp, S, dh, tokens, C, w, eps, dsp, dw_part, st);
  else if (ch <= 12) bwd_launch_s<12>(sp, S, dh, tokens, C, w, eps, dsp, dw_part, st);
  else bwd_launch_s<16>(sp, S, dh, tokens, C, w, eps, dsp, dw_part, st);
  if (sana_status e = check_launch("attnres_bwd_kernel")) return e;
  attnres_dw_reduce_kernel<<<(C + 255) / 256, 256, 0, st>>>(dw_part, attnres_bwd_blocks(tokens), C, dw);
  return check_launch("attnres_dw_reduce_kernel");
}

sana_status rmsnorm_run(long long rows, int C, sana_dtype dt, const void* x, float eps, void* y,
                        cudaStream_t st) {
  if (C % 8 != 0 || C > 8192) return fail(SANA_ERR_UNSUPPORTED, "rmsnorm: C=%d", C);
  if (rows == 0) return SANA_OK;
  const int threads = threads_for(C);
  long long blocks = rows < (long long)kNumSMs * 16 ? rows : (long long)kNumSMs * 16;
  if (dt == SANA_BF16)
    rmsnorm_kernel<__nv_bfloat16><<<(int)blocks, threads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), rows, C, eps, static_cast<__nv_bfloat16*>(y));
  else
    rmsnorm_kernel<float><<<(int)blocks, threads, 0, st>>>(static_cast<const float*>(x), rows, C,
                                                           eps, static_cast<float*>(y));
  return check_launch("rmsnorm_kernel");
}

}  // namespace sana
