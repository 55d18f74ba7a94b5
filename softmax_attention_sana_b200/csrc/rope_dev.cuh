// Device-side 3D RoPE lookup ("SANA-Video" paper notes, sec. 3.2: RoPE applied
// after the ReLU feature map; Fig. 2(c): 3D RoPE over the latent grid).
// Rotary pair j of a head rotates elements (2j, 2j+1); pairs [0, n_t) follow the
// absolute frame index, the next n_h the row, the last n_w the column.
#pragma once

#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {

// Tables of one grid staged in shared memory as float2(cos, sin).  Row strides
// are rounded up to odd counts so that neighbouring grid positions read by
// neighbouring lanes fall in different banks.
struct RopeSmem {
  const float2* t;
  const float2* h;
  const float2* w;
  int st, sh, sw;
  int n_t, n_th;
};

__device__ __forceinline__ int odd_up_d(int n) { return n | 1; }

// Cooperative staging by `nthreads` threads for batch entry b; caller
// synchronises afterwards.
__device__ inline RopeSmem rope_stage(float2* base, const RopeDev& r, const GridDev& g, int b,
                                      int tid, int nthreads) {
  RopeSmem rs;
  rs.st = odd_up_d(r.n_t);
  rs.sh = odd_up_d(r.n_h);
  rs.sw = odd_up_d(r.n_w);
  float2* pt = base;
  float2* ph = pt + g.T * rs.st;
  float2* pw = ph + g.H * rs.sh;
  for (int i = tid; i < g.T * r.n_t; i += nthreads) {
    const int row = i / r.n_t, j = i - row * r.n_t;
    const int src = (g.t_offset + b * g.t_stride + row) * r.n_t + j;
    pt[row * rs.st + j] = make_float2(r.cos_t[src], r.sin_t[src]);
  }
  for (int i = tid; i < g.H * r.n_h; i += nthreads) {
    const int row = i / r.n_h, j = i - row * r.n_h;
    ph[row * rs.sh + j] = make_float2(r.cos_h[i], r.sin_h[i]);
  }
  for (int i = tid; i < g.W * r.n_w; i += nthreads) {
    const int row = i / r.n_w, j = i - row * r.n_w;
    pw[row * rs.sw + j] = make_float2(r.cos_w[i], r.sin_w[i]);
  }
  rs.t = pt;
  rs.h = ph;
  rs.w = pw;
  rs.n_t = r.n_t;
  rs.n_th = r.n_t + r.n_h;
  return rs;
}

// Per-token view: (cos, sin) of pair j of token n (local index within the grid).
struct RowRope {
  const float2* pt;
  const float2* ph;
  const float2* pw;
  int n_t, n_th;
  __device__ __forceinline__ float2 cs(int j) const {
    return j < n_t ? pt[j] : (j < n_th ? ph[j - n_t] : pw[j - n_th]);
  }
};

__device__ __forceinline__ RowRope row_rope(const RopeSmem& rs, const GridDev& g, int n) {
  const int hw = g.H * g.W;
  const int t = n / hw;
  const int rem = n - t * hw;
  const int h = rem / g.W;
  const int w = rem - h * g.W;
  RowRope rr;
  rr.pt = rs.t + t * rs.st;
  rr.ph = rs.h + h * rs.sh;
  rr.pw = rs.w + w * rs.sw;
  rr.n_t = rs.n_t;
  rr.n_th = rs.n_th;
  return rr;
}

// Same lookup straight from the global tables (fp32 paths), batch entry b.
__device__ __forceinline__ float2 rope_cs_global(const RopeDev& r, const GridDev& g, int b, int n,
                                                 int j) {
  const int hw = g.H * g.W;
  const int t = n / hw;
  const int rem = n - t * hw;
  const int h = rem / g.W;
  const int w = rem - h * g.W;
  if (j < r.n_t) {
    const int i = (g.t_offset + b * g.t_stride + t) * r.n_t + j;
    return make_float2(r.cos_t[i], r.sin_t[i]);
  }
  if (j < r.n_t + r.n_h) {
    const int i = h * r.n_h + (j - r.n_t);
    return make_float2(r.cos_h[i], r.sin_h[i]);
  }
  const int i = w * r.n_w + (j - r.n_t - r.n_h);
  return make_float2(r.cos_w[i], r.sin_w[i]);
}

// Rotate one pair: (x, y) -> (x cos - y sin, x sin + y cos).
__device__ __forceinline__ float2 rotate(float x, float y, float2 cs) {
  return make_float2(x * cs.x - y * cs.y, x * cs.y + y * cs.x);
}

}  // namespace sana
