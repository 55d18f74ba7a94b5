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
