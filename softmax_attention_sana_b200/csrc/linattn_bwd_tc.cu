// Backward of the gated ReLU linear attention with RoPE after the ReLU, bf16 on
// tcgen05.  Forward ("SANA-Video" paper notes, sec. 3.2; gate per the
// "SANA-Video 2.0" abstract), per (batch, head):
//   q'_i = R_i phi(q_i),  S = sum_j k'_j^T v_j,  z = sum_j phi(k_j),
//   num_i = q'_i S,  den_i = phi(q_i) . z + eps,  o_i = num_i / den_i,
//   y_i = sigmoid(g_i) o_i.
// Given dy, the chain rule gives (sigma = sigmoid(g)):
//   dg = dy o sigma (1 - sigma),   do = dy sigma,   dnum = do / den,
//   dden = -(do . o) / den,        dq' = dnum S^T,
//   dq = (R^T dq' + dden z) [q > 0],
//   dS = sum_i q'_i^T dnum_i,      dz = sum_i dden_i phi(q_i),
//   dk' = v dS^T,  dv = k' dS,     dk = (R^T dk' + dz) [k > 0].
//
// Launches: the forward state kernel (S, z), the query-side kernel below
// (dq, dg and split partials of dS, dz), the fixed-order combine, and the
// key-side kernel (dk, dv).  Both new kernels keep the forward's layout:
// 16 worker warps, thread = (token row, 32-column quarter), one TMA producer
// warp (which also stores the results) and one MMA-issuing thread.  S and dS
// sit once in shared memory as a bf16 [d][e] tile with the 128-byte swizzle:
// read K-major it is the B operand of (.) S^T, read MN-major that of (.) S.
#include <cuda.h>

#include <cstddef>

#include "rope_dev.cuh"
#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {
namespace {

constexpr int kD = 128;
constexpr int kRows = 128;
constexpr int kHalf = kRows * 64 * 2;  // 16 KB
constexpr int kTileB = 2 * kHalf;      // 32 KB
constexpr int kWorkers = 512;
constexpr int kThreads = kWorkers + 64;  // + producer warp + MMA warp
constexpr int kWarpProd = 16, kWarpMma = 17;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

template <int NT, int NH>
__device__ __forceinline__ float2 pair_cs(const RowRope& rr, int j) {
  if (NT >= 0) return j < NT ? rr.pt[j] : (j < NT + NH ? rr.ph[j - NT] : rr.pw[j - NT - NH]);
  return rr.cs(j);
}

// Rotary (cos, sin) of one token read straight from the global tables (the
// key-side kernel leaves its shared memory to the K/V ring; the tables are
// small enough to stay in L1).
struct GlobalRowRope {
  const float *ct, *st, *ch, *sh, *cw, *sw;
  int n_t, n_th;
  __device__ __forceinline__ float2 cs(int j) const {
    return j < n_t ? make_float2(ct[j], st[j])
                   : (j < n_th ? make_float2(ch[j - n_t], sh[j - n_t])
                               : make_float2(cw[j - n_th], sw[j - n_th]));
  }
};

__device__ __forceinline__ GlobalRowRope global_row_rope(const RopeDev& r, const GridDev& g,
                                                         int b, int n) {
  const int hw = g.H * g.W;
  const int t = n / hw, rem = n - t * hw, hh = rem / g.W, ww = rem - hh * g.W;
  const int tt = g.t_offset + b * g.t_stride + t;
  GlobalRowRope rr;
  rr.ct = r.cos_t + tt * r.n_t;
  rr.st = r.sin_t + tt * r.n_t;
  rr.ch = r.cos_h + hh * r.n_h;
  rr.sh = r.sin_h + hh * r.n_h;
  rr.cw = r.cos_w + ww * r.n_w;
  rr.sw = r.sin_w + ww * r.n_w;
  rr.n_t = r.n_t;
  rr.n_th = r.n_t + r.n_h;
  return rr;
}

template <int NT, int NH>
__device__ __forceinline__ float2 pair_cs(const GlobalRowRope& rr, int j) {
  if (NT >= 0)
    return j < NT ? make_float2(rr.ct[j], rr.st[j])
                  : (j < NT + NH ? make_float2(rr.ch[j - NT], rr.sh[j - NT])
                                 : make_float2(rr.cw[j - NT - NH], rr.sw[j - NT - NH]));
  return rr.cs(j);
}

// ---- packed fp32 (f32x2): one instruction for two values
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void up2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t bf2_to_pk2(uint32_t u) {
  return pk2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t pk2_to_bf2(uint64_t v) {
  float a, b;
  up2(v, a, b);
  return f2_to_bf2(a, b);
}
// max(x, 0) of both bf16 halves
__device__ __forceinline__ uint32_t relu_bf2(uint32_t w) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(0u));
  return r;
}
// sigmoid of two values, the steps of sigmoid_fast on f32x2 (the same
// exponential and the same two Newton steps for 1 / (1 + t))
__device__ __forceinline__ uint64_t sigmoid_pk2(float x0, float x1) {
  float t0, t1;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(t0) : "f"(-1.4426950408889634f * fabsf(x0)));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(t1) : "f"(-1.4426950408889634f * fabsf(x1)));
  const uint64_t t = pk2(t0, t1);
  const uint64_t d = add2(t, pk2(1.f, 1.f));
  const uint64_t nd = mul2(d, pk2(-1.f, -1.f));
  uint64_t r = fma2(pk2(-0.47058823529411764f, -0.47058823529411764f), d,
                    pk2(1.4117647058823530f, 1.4117647058823530f));
  r = mul2(r, fma2(nd, r, pk2(2.f, 2.f)));
  r = mul2(r, fma2(nd, r, pk2(2.f, 2.f)));
  const uint64_t tr = mul2(t, r);
  float r0, r1, q0, q1;
  up2(r, r0, r1);
  up2(tr, q0, q1);
  return pk2(x0 >= 0.f ? r0 : q0, x1 >= 0.f ? r1 : q1);
}

// Rotation by the opposite angle (the transpose of the RoPE rotation).
__device__ __forceinline__ float2 rotate_t(float x, float y, float2 cs) {
  return make_float2(x * cs.x + y * cs.y, y * cs.x - x * cs.y);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// A 128 x 128 fp32 matrix M[d][e] as a bf16 tile in shared memory: rows d, two
// 64-column halves of e, 128-byte swizzle (the layout TMA gives a token tile).
__device__ void stage_matrix(uint8_t* dst, const float* __restrict__ M, int tid, int nthreads) {
  for (int i = tid; i < kD * 16; i += nthreads) {
    const int d = i >> 4, ch = i & 15;  // 16-byte chunk = 8 consecutive e
    const float4 a = *reinterpret_cast<const float4*>(M + d * kD + ch * 8);
    const float4 c = *reinterpret_cast<const float4*>(M + d * kD + ch * 8 + 4);
    *reinterpret_cast<uint4*>(dst + (ch >> 3) * kHalf + sw128_off(d, ch & 7)) =
        make_uint4(f2_to_bf2(a.x, a.y), f2_to_bf2(a.z, a.w), f2_to_bf2(c.x, c.y),
                   f2_to_bf2(c.z, c.w));
  }
}

// ReLU + RoPE of this thread's 32 columns (quarter C4) of token row r, in
// place; returns the partial phi(x) . z over those columns and the (x > 0) bits.
template <int NT, int NH, int C4, class RR>
__device__ __forceinline__ float quarter_forward(uint8_t* tile, int r, const RR& rr,
                                                 const float* z, uint32_t& mask) {
  uint8_t* half = tile + (C4 >> 1) * kHalf;
  uint64_t den2 = pk2(0.f, 0.f);  // even and odd columns, summed at the end
  mask = 0;
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint4* p = reinterpret_cast<uint4*>(half + sw128_off(r, (C4 & 1) * 4 + ch));
    const uint4 raw = *p;
    uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    float zc[8];
    if (z) {
      const float4 z0 = *reinterpret_cast<const float4*>(z + C4 * 32 + ch * 8);
      const float4 z1 = *reinterpret_cast<const float4*>(z + C4 * 32 + ch * 8 + 4);
      zc[0] = z0.x; zc[1] = z0.y; zc[2] = z0.z; zc[3] = z0.w;
      zc[4] = z1.x; zc[5] = z1.y; zc[6] = z1.z; zc[7] = z1.w;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t xr = relu_bf2(w[i]);  // exact: ReLU commutes with widening
      const float2 x = bf2_to_f2(xr);
      mask |= (x.x > 0.f ? 1u : 0u) << (ch * 8 + 2 * i);
      mask |= (x.y > 0.f ? 1u : 0u) << (ch * 8 + 2 * i + 1);
      const int col = C4 * 32 + ch * 8 + 2 * i;
      if (z) den2 = fma2(pk2(x.x, x.y), pk2(zc[2 * i], zc[2 * i + 1]), den2);
      const float2 rt = rotate(x.x, x.y, pair_cs<NT, NH>(rr, col >> 1));
      w[i] = f2_to_bf2(rt.x, rt.y);
    }
    *p = make_uint4(w[0], w[1], w[2], w[3]);
  }
  float d0, d1;
  up2(den2, d0, d1);
  return d0 + d1;
}

template <int NT, int NH, class RR>
__device__ __forceinline__ float quarter_forward_any(int c4, uint8_t* tile, int r,
                                                     const RR& rr, const float* z,
                                                     uint32_t& mask) {
  switch (c4) {  // warp-uniform
    case 0: return quarter_forward<NT, NH, 0>(tile, r, rr, z, mask);
    case 1: return quarter_forward<NT, NH, 1>(tile, r, rr, z, mask);
    case 2: return quarter_forward<NT, NH, 2>(tile, r, rr, z, mask);
    default: return quarter_forward<NT, NH, 3>(tile, r, rr, z, mask);
  }
}

// (R^T grad + add * zz) masked by (x > 0), for this thread's 32 columns of row
// r (quarter C4): grad comes from TMEM in two 16-column parts at tmem_col; the
// result replaces the tile's row segment.  With zacc, the tile's contents
// (R phi) are first rotated back and accumulated as add * phi.
template <int NT, int NH, int C4, class RR>
__device__ __forceinline__ void quarter_backward(uint8_t* tile, int r, const RR& rr,
                                                 uint32_t tmem_row, float add, const float* zz,
                                                 uint32_t mask, float* zacc,
                                                 uint64_t* freed) {
  uint8_t* half = tile + (C4 >> 1) * kHalf;
#pragma unroll
  for (int part = 0; part < 2; ++part) {
    uint32_t gv[16];
    tmem_ld16(tmem_row + C4 * 32 + part * 16, gv);
    tmem_ld_wait();
    if (part == 1 && freed) {  // this thread has read its gradient columns
      tc_fence_before();
      mbar_arrive(freed);
    }
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      uint4* p = reinterpret_cast<uint4*>(half + sw128_off(r, (C4 & 1) * 4 + part * 2 + cc));
      const uint4 raw = *p;
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      const int cb = C4 * 32 + part * 16 + cc * 8;  // first of these 8 columns
      const float4 z0 = *reinterpret_cast<const float4*>(zz + cb);
      const float4 z1 = *reinterpret_cast<const float4*>(zz + cb + 4);
      const float zc[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
      const uint64_t add2v = pk2(add, add);
      uint32_t out[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = part * 16 + cc * 8 + 2 * i;  // column within the quarter
        const int col = C4 * 32 + j;
        const float2 cs = pair_cs<NT, NH>(rr, col >> 1);
        if (zacc) {
          const float2 xr = bf2_to_f2(w[i]);
          const float2 ph = rotate_t(xr.x, xr.y, cs);
          float a0, a1;
          up2(fma2(add2v, pk2(ph.x, ph.y), pk2(zacc[j], zacc[j + 1])), a0, a1);
          zacc[j] = a0;
          zacc[j + 1] = a1;
        }
        const float2 gr =
            rotate_t(__uint_as_float(gv[cc * 8 + 2 * i]), __uint_as_float(gv[cc * 8 + 2 * i + 1]), cs);
        float g0, g1;
        up2(fma2(add2v, pk2(zc[2 * i], zc[2 * i + 1]), pk2(gr.x, gr.y)), g0, g1);
        g0 = ((mask >> j) & 1u) ? g0 : 0.f;
        g1 = ((mask >> (j + 1)) & 1u) ? g1 : 0.f;
        out[i] = f2_to_bf2(g0, g1);
      }
      *p = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

template <int NT, int NH, class RR>
__device__ __forceinline__ void quarter_backward_any(int c4, uint8_t* tile, int r,
                                                     const RR& rr, uint32_t tmem_row,
                                                     float add, const float* zz, uint32_t mask,
                                                     float* zacc, uint64_t* freed) {
  switch (c4) {  // warp-uniform
    case 0: quarter_backward<NT, NH, 0>(tile, r, rr, tmem_row, add, zz, mask, zacc, freed); break;
    case 1: quarter_backward<NT, NH, 1>(tile, r, rr, tmem_row, add, zz, mask, zacc, freed); break;
    case 2: quarter_backward<NT, NH, 2>(tile, r, rr, tmem_row, add, zz, mask, zacc, freed); break;
    default: quarter_backward<NT, NH, 3>(tile, r, rr, tmem_row, add, zz, mask, zacc, freed); break;
  }
}

// ------------------------------------------------------------------------
// query side: dq, dg, partial dS and dz
// ------------------------------------------------------------------------
struct BwdQCtl {
  uint64_t fullQ[2], fullD[2], emptyD[2], qready[2], out_ready[2];
  uint64_t fullG;
  uint64_t num_done, dnum_ready, bc_done, dq_free, dS_done;
  uint32_t tmem;
  int abort_flag;
  alignas(16) float den[2][4][kRows];   // [q stage][column quarter][row]
  alignas(16) float dden[2][4][kRows];  // [tile parity][column quarter][row]
  alignas(16) float z[kD];
};
// After the last tile the denominators are dead; their slots hold the dz
// partials [column quarter][row quarter][column] of the final reduction.
static_assert(sizeof(BwdQCtl::den) >= 4 * 4 * 32 * sizeof(float), "dz partials fit in den");

// TMEM columns: num [0, 128), dq' [128, 256), dS accumulator [256, 384).
template <bool kGate, int NT, int NH>
__global__ void __launch_bounds__(kThreads, 1)
    linattn_bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_dy,
                         const __grid_constant__ CUtensorMap tm_g,
                         const __grid_constant__ CUtensorMap tm_dq,
                         const __grid_constant__ CUtensorMap tm_dg,
                         const float* __restrict__ S_all, const float* __restrict__ z_all,
                         RopeDev rope, GridDev g, int tiles_total, int splits, float eps,
                         float* __restrict__ ws_dS, float* __restrict__ ws_dz, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ BwdQCtl ctl;
  uint8_t* smem = align1024(smem_raw);
  uint8_t* s_op = smem;                      // S as bf16 [d][e], 32 KB
  uint8_t* q_st = s_op + kTileB;             // 2 stages: q -> q' -> dq
  uint8_t* d_st = q_st + 2 * kTileB;         // 2 stages: dy -> dnum
  uint8_t* g_st = d_st + 2 * kTileB;         // 1 stage: g -> dg
  float2* rope_base = reinterpret_cast<float2*>(g_st + kTileB);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tile0 = (int)((long long)split * tiles_total / splits);
  const int ntiles = (int)((long long)(split + 1) * tiles_total / splits) - tile0;
  const int bh = b * g.heads + h;
  const WaitCtx wc{&ctl.abort_flag, status};

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl.fullQ[s], 1);
      mbar_init(&ctl.fullD[s], 1);
      mbar_init(&ctl.emptyD[s], 1);
      mbar_init(&ctl.qready[s], kWorkers);
      mbar_init(&ctl.out_ready[s], kWorkers);
    }
    mbar_init(&ctl.fullG, 1);
    mbar_init(&ctl.num_done, 1);
    mbar_init(&ctl.dnum_ready, kWorkers);
    mbar_init(&ctl.bc_done, 1);
    mbar_init(&ctl.dq_free, kWorkers);
    mbar_init(&ctl.dS_done, 1);
    ctl.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl.tmem, 512);
    tmem_relinquish();
  }
  if (tid < kD) ctl.z[tid] = z_all[(size_t)bh * kD + tid];
  if (tid < kWorkers) {
    stage_matrix(s_op, S_all + (size_t)bh * kD * kD, tid, kWorkers);
    fence_proxy_async_smem();
  }
  const RopeSmem rs = rope_stage(rope_base, rope, g, b, tid, kThreads);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;

  if (warp == kWarpProd) {
    // ---------------- TMA producer; also stores dg and dq and recycles stages
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_dy);
      if (kGate) prefetch_tmap(&tm_g);
      int issued_qd = 0, issued_g = 0;
      auto load_qd = [&](int it) {
        const int s = it & 1, n0 = (tile0 + it) * kRows;
        mbar_arrive_expect_tx(&ctl.fullQ[s], kTileB);
        tma_load_3d(q_st + s * kTileB, &tm_q, &ctl.fullQ[s], h * kD, n0, b);
        tma_load_3d(q_st + s * kTileB + kHalf, &tm_q, &ctl.fullQ[s], h * kD + 64, n0, b);
        mbar_arrive_expect_tx(&ctl.fullD[s], kTileB);
        tma_load_3d(d_st + s * kTileB, &tm_dy, &ctl.fullD[s], h * kD, n0, b);
        tma_load_3d(d_st + s * kTileB + kHalf, &tm_dy, &ctl.fullD[s], h * kD + 64, n0, b);
        ++issued_qd;
      };
      auto load_g = [&](int it) {
        const int n0 = (tile0 + it) * kRows;
        mbar_arrive_expect_tx(&ctl.fullG, kTileB);
        tma_load_3d(g_st, &tm_g, &ctl.fullG, h * kD, n0, b);
        tma_load_3d(g_st + kHalf, &tm_g, &ctl.fullG, h * kD + 64, n0, b);
        ++issued_g;
      };
      if (ntiles > 0) {
        load_qd(0);
        if (kGate) load_g(0);
      }
      if (ntiles > 1) load_qd(1);
      bool ok = true;
      for (int it = 0; ok && it < ntiles; ++it) {
        const int s = it & 1, n0 = (tile0 + it) * kRows;
        if (kGate) {
          // dg of tile it sits in the g stage once every worker is past phase B
          if (!mbar_wait(&ctl.dnum_ready, it & 1, wc, 0x51)) {
            ok = false;
            break;
          }
          tma_store_3d(&tm_dg, g_st, h * kD, n0, b);
          tma_store_3d(&tm_dg, g_st + kHalf, h * kD + 64, n0, b);
          bulk_commit();
          bulk_wait_read0();
          if (it + 1 < ntiles) load_g(it + 1);
        }
        // dq of tile it sits in q stage s once every worker is past phase C
        if (!mbar_wait(&ctl.out_ready[s], (it >> 1) & 1, wc, 0x52)) {
          ok = false;
          break;
        }
        tma_store_3d(&tm_dq, q_st + s * kTileB, h * kD, n0, b);
        tma_store_3d(&tm_dq, q_st + s * kTileB + kHalf, h * kD + 64, n0, b);
        bulk_commit();
        bulk_wait_read0();
        if (it + 2 < ntiles) {
          // dy stage s is free once the MMAs of tile it have read dnum from it
          if (!mbar_wait(&ctl.emptyD[s], (it >> 1) & 1, wc, 0x53)) {
            ok = false;
            break;
          }
          load_qd(it + 2);
        }
      }
      bulk_wait0();
      if (!ok) {  // loads in flight land before the CTA exits
        for (int it = issued_qd > 2 ? issued_qd - 2 : 0; it < issued_qd; ++it) {
          mbar_drain(&ctl.fullQ[it & 1], (it >> 1) & 1);
          mbar_drain(&ctl.fullD[it & 1], (it >> 1) & 1);
        }
        if (issued_g > 0) mbar_drain(&ctl.fullG, (issued_g - 1) & 1);
      }
    }
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer
    if (lane == 0) {
      // num = q' S      : A = q' K-major [tok][d], B = S MN-major (N = e, K = d)
      // dq' = dnum S^T  : A = dnum K-major [tok][e], B = S K-major (N = d, K = e)
      // dS += q'^T dnum : A = q' MN-major (M = d), B = dnum MN-major (N = e)
      const uint32_t id_num = idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t id_dq = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_dS = idesc_bf16_f32(128, 128, 1, 1);
      const uint64_t q_k = smem_desc_sw128(smem_u32(q_st), 16, 1024);
      const uint64_t q_m = smem_desc_sw128(smem_u32(q_st), kHalf, 1024);
      const uint64_t d_k = smem_desc_sw128(smem_u32(d_st), 16, 1024);
      const uint64_t d_m = smem_desc_sw128(smem_u32(d_st), kHalf, 1024);
      const uint64_t s_k = smem_desc_sw128(smem_u32(s_op), 16, 1024);
      const uint64_t s_m = smem_desc_sw128(smem_u32(s_op), kHalf, 1024);
      for (int it = 0; it < ntiles; ++it) {
        const int s = it & 1;
        if (!mbar_wait(&ctl.qready[s], (it >> 1) & 1, wc, 0x54)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t offk = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_ss(tmem, desc_advance(q_k, s * kTileB + offk), desc_advance(s_m, kk * 2048), id_num,
                  kk != 0);
        }
        umma_commit(&ctl.num_done);
        if (!mbar_wait(&ctl.dnum_ready, it & 1, wc, 0x55)) break;
        if (it >= 1 && !mbar_wait(&ctl.dq_free, (it - 1) & 1, wc, 0x56)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t offk = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_ss(tmem + 128, desc_advance(d_k, s * kTileB + offk), desc_advance(s_k, offk), id_dq,
                  kk != 0);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss(tmem + 256, desc_advance(q_m, s * kTileB + kk * 2048),
                  desc_advance(d_m, s * kTileB + kk * 2048), id_dS, (it | kk) != 0);
        umma_commit(&ctl.emptyD[s]);
        umma_commit(&ctl.bc_done);
      }
      umma_commit(&ctl.dS_done);
    }
  } else if (warp < 16) {
    // ---------------- workers: thread = (token row r, column quarter c4)
    const int q4 = warp & 3, c4 = warp >> 2, r = q4 * 32 + lane;
    const int hf = c4 >> 1;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    float zacc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) zacc[i] = 0.f;
    uint32_t mask0 = 0, mask1 = 0;  // (q > 0) bits of the tile in q stage 0 / 1
    bool ok = true;
    // A: q -> q' in place, partial denominators, (q > 0) bits
    auto phase_a = [&](int it) {
      const int s = it & 1;
      if (!mbar_wait(&ctl.fullQ[s], (it >> 1) & 1, wc, 0x57)) {
        ok = false;
        return;
      }
      const int n = (tile0 + it) * kRows + r;
      float den = 0.f;
      uint32_t m = 0;
      if (n < g.N) {  // rows past N were zero-filled by TMA
        const RowRope rr = row_rope(rs, g, n);
        den = quarter_forward_any<NT, NH>(c4, q_st + s * kTileB, r, rr, ctl.z, m);
      }
      if (s) mask1 = m;
      else mask0 = m;
      ctl.den[s][c4][r] = den;
      fence_proxy_async_smem();
      mbar_arrive(&ctl.qready[s]);
    };
    // B: o = num / den; dg into the g stage, dnum over dy, partial dden
    auto phase_b = [&](int it) {
      const int s = it & 1;
      bool okw = mbar_wait(&ctl.num_done, it & 1, wc, 0x58);
      okw = mbar_wait(&ctl.fullD[s], (it >> 1) & 1, wc, 0x59) && okw;
      if (kGate) okw = mbar_wait(&ctl.fullG, it & 1, wc, 0x5a) && okw;
      if (!__all_sync(0xffffffffu, okw)) {  // tcgen05.ld is warp-collective
        ok = false;
        return;
      }
      tc_fence_after();
      const float inv =
          1.f / (ctl.den[s][0][r] + ctl.den[s][1][r] + ctl.den[s][2][r] + ctl.den[s][3][r] + eps);
      uint8_t* dhalf = d_st + s * kTileB + hf * kHalf;
      uint8_t* ghalf = g_st + hf * kHalf;
      const uint64_t inv2 = pk2(inv, inv);
      uint64_t ddot2 = pk2(0.f, 0.f);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        uint32_t nv[16];
        tmem_ld16(tmem + lane_base + c4 * 32 + part * 16, nv);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int ch = (c4 & 1) * 4 + part * 2 + cc;
          uint4* pd = reinterpret_cast<uint4*>(dhalf + sw128_off(r, ch));
          uint4* pg = reinterpret_cast<uint4*>(ghalf + sw128_off(r, ch));
          const uint4 draw = *pd;
          const uint32_t dw[4] = {draw.x, draw.y, draw.z, draw.w};
          uint32_t gw[4] = {0, 0, 0, 0};
          if (kGate) {
            const uint4 graw = *pg;
            gw[0] = graw.x; gw[1] = graw.y; gw[2] = graw.z; gw[3] = graw.w;
          }
          uint32_t od[4], og[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint64_t o2 =
                mul2(pk2(__uint_as_float(nv[cc * 8 + 2 * i]), __uint_as_float(nv[cc * 8 + 2 * i + 1])),
                     inv2);
            uint64_t do2 = bf2_to_pk2(dw[i]);
            if (kGate) {
              const float2 gv = bf2_to_f2(gw[i]);
              const uint64_t s2 = sigmoid_pk2(gv.x, gv.y);
              const uint64_t oms = fma2(s2, pk2(-1.f, -1.f), pk2(1.f, 1.f));  // 1 - sigma
              og[i] = pk2_to_bf2(mul2(mul2(do2, o2), mul2(s2, oms)));
              do2 = mul2(do2, s2);
            }
            ddot2 = fma2(do2, o2, ddot2);
            od[i] = pk2_to_bf2(mul2(do2, inv2));
          }
          *pd = make_uint4(od[0], od[1], od[2], od[3]);
          if (kGate) *pg = make_uint4(og[0], og[1], og[2], og[3]);
        }
      }
      float dd0, dd1;
      up2(ddot2, dd0, dd1);
      ctl.dden[it & 1][c4][r] = -(dd0 + dd1) * inv;
      fence_proxy_async_smem();
      mbar_arrive(&ctl.dnum_ready);
    };
    // C: dq = (R^T dq' + dden z) [q > 0] over q' in place; dz += dden phi(q)
    auto phase_c = [&](int it) {
      const int s = it & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl.bc_done, it & 1, wc, 0x5b))) {
        ok = false;
        return;
      }
      tc_fence_after();
      const float dden = ctl.dden[it & 1][0][r] + ctl.dden[it & 1][1][r] +
                         ctl.dden[it & 1][2][r] + ctl.dden[it & 1][3][r];
      const int n = (tile0 + it) * kRows + r;
      const RowRope rr = row_rope(rs, g, n < g.N ? n : 0);
      quarter_backward_any<NT, NH>(c4, q_st + s * kTileB, r, rr, tmem + lane_base + 128, dden,
                                   ctl.z, s ? mask1 : mask0, zacc, &ctl.dq_free);
      fence_proxy_async_smem();
      mbar_arrive(&ctl.out_ready[s]);
    };
    if (ntiles > 0) phase_a(0);
    for (int it = 0; ok && it < ntiles; ++it) {
      phase_b(it);
      if (!ok) break;
      if (it + 1 < ntiles) {
        phase_a(it + 1);
        if (!ok) break;
      }
      phase_c(it);
    }
    // partial dS (rows d = r, columns of this quarter) and dz of this split
    const size_t part = (size_t)bh * splits + split;
    const bool okd = __all_sync(0xffffffffu, mbar_wait(&ctl.dS_done, 0, wc, 0x5c)) && ok;
    if (okd) {
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(tmem + lane_base + 256 + c4 * 32, v);
      tmem_ld_wait();
      if (ntiles == 0)  // no token of this split: the accumulator was never written
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0u;
      float4* dst = reinterpret_cast<float4*>(ws_dS + part * kD * kD + (size_t)r * kD + c4 * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                             __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
    }
    // dz: fixed-order sums over the 32 rows of the warp, then the 4 row quarters
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float a = zacc[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      zacc[i] = a;
    }
    // every worker is past its last phase B (dS_done follows the last dnum
    // arrivals), so nobody reads the denominators any more
    float* zred = &ctl.den[0][0][0];
    if (lane == 0)
#pragma unroll
      for (int i = 0; i < 32; ++i) zred[(c4 * 4 + q4) * 32 + i] = zacc[i];
    named_bar_sync(1, kWorkers);
    if (tid < kD) {
      const int cc = tid >> 5, i = tid & 31;
      ws_dz[part * kD + cc * 32 + i] = zred[(cc * 4 + 0) * 32 + i] + zred[(cc * 4 + 1) * 32 + i] +
                                       zred[(cc * 4 + 2) * 32 + i] + zred[(cc * 4 + 3) * 32 + i];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    if (*wc.abort_flag) mbar_drain(&ctl.dS_done, 0);  // MMAs in flight finish before TMEM is freed
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------
// key side: dk, dv
// ------------------------------------------------------------------------
constexpr int kStagesK = 3;  // k and v rings (they double as dk / dv staging)

struct BwdKCtl {
  uint64_t fullK[kStagesK], fullV[kStagesK], kready[kStagesK], out_ready[kStagesK];
  uint64_t mma_done[2], tmem_free[2];
  uint32_t tmem;
  int abort_flag;
  alignas(16) float dz[kD];
};

// TMEM columns, per tile parity tb: dk' [256 tb, +128), dv [256 tb + 128, +128).
// The rotary tables are read from global memory, leaving shared memory to a
// three-stage K/V ring.
template <int NT, int NH>
__global__ void __launch_bounds__(kThreads, 1)
    linattn_bwd_k_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_dk,
                         const __grid_constant__ CUtensorMap tm_dv,
                         const float* __restrict__ dS_all, const float* __restrict__ dz_all,
                         RopeDev rope, GridDev g, int tiles_total, int splits, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ BwdKCtl ctl;
  uint8_t* smem = align1024(smem_raw);
  uint8_t* ds_op = smem;                     // dS as bf16 [d][e], 32 KB
  uint8_t* k_st = ds_op + kTileB;            // k -> k' -> dk
  uint8_t* v_st = k_st + kStagesK * kTileB;  // v -> dv

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tile0 = (int)((long long)split * tiles_total / splits);
  const int ntiles = (int)((long long)(split + 1) * tiles_total / splits) - tile0;
  const int bh = b * g.heads + h;
  const WaitCtx wc{&ctl.abort_flag, status};

  if (tid == 0) {
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(&ctl.fullK[s], 1);
      mbar_init(&ctl.fullV[s], 1);
      mbar_init(&ctl.kready[s], kWorkers);
      mbar_init(&ctl.out_ready[s], kWorkers);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl.mma_done[t], 1);
      mbar_init(&ctl.tmem_free[t], kWorkers);
    }
    ctl.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl.tmem, 512);
    tmem_relinquish();
  }
  if (tid < kD) ctl.dz[tid] = dz_all[(size_t)bh * kD + tid];
  if (tid < kWorkers) {
    stage_matrix(ds_op, dS_all + (size_t)bh * kD * kD, tid, kWorkers);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;

  if (warp == kWarpProd) {
    // ---------------- TMA producer; also stores dk and dv and recycles stages
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int issued = 0;
      auto load = [&](int it) {
        const int s = it % kStagesK, n0 = (tile0 + it) * kRows;
        mbar_arrive_expect_tx(&ctl.fullK[s], kTileB);
        tma_load_3d(k_st + s * kTileB, &tm_k, &ctl.fullK[s], h * kD, n0, b);
        tma_load_3d(k_st + s * kTileB + kHalf, &tm_k, &ctl.fullK[s], h * kD + 64, n0, b);
        mbar_arrive_expect_tx(&ctl.fullV[s], kTileB);
        tma_load_3d(v_st + s * kTileB, &tm_v, &ctl.fullV[s], h * kD, n0, b);
        tma_load_3d(v_st + s * kTileB + kHalf, &tm_v, &ctl.fullV[s], h * kD + 64, n0, b);
        ++issued;
      };
      for (int it = 0; it < kStagesK && it < ntiles; ++it) load(it);
      bool ok = true;
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % kStagesK, n0 = (tile0 + it) * kRows;
        if (!mbar_wait(&ctl.out_ready[s], (it / kStagesK) & 1, wc, 0x61)) {
          ok = false;
          break;
        }
        tma_store_3d(&tm_dk, k_st + s * kTileB, h * kD, n0, b);
        tma_store_3d(&tm_dk, k_st + s * kTileB + kHalf, h * kD + 64, n0, b);
        tma_store_3d(&tm_dv, v_st + s * kTileB, h * kD, n0, b);
        tma_store_3d(&tm_dv, v_st + s * kTileB + kHalf, h * kD + 64, n0, b);
        bulk_commit();
        bulk_wait_read0();
        if (it + kStagesK < ntiles) load(it + kStagesK);
      }
      bulk_wait0();
      if (!ok)
        for (int it = issued > kStagesK ? issued - kStagesK : 0; it < issued; ++it) {
          mbar_drain(&ctl.fullK[it % kStagesK], (it / kStagesK) & 1);
          mbar_drain(&ctl.fullV[it % kStagesK], (it / kStagesK) & 1);
        }
    }
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer
    if (lane == 0) {
      // dk' = v dS^T : A = v K-major [tok][e], B = dS K-major (N = d, K = e)
      // dv  = k' dS  : A = k' K-major [tok][d], B = dS MN-major (N = e, K = d)
      const uint32_t id_dk = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_dv = idesc_bf16_f32(128, 128, 0, 1);
      const uint64_t k_k = smem_desc_sw128(smem_u32(k_st), 16, 1024);
      const uint64_t v_k = smem_desc_sw128(smem_u32(v_st), 16, 1024);
      const uint64_t ds_k = smem_desc_sw128(smem_u32(ds_op), 16, 1024);
      const uint64_t ds_m = smem_desc_sw128(smem_u32(ds_op), kHalf, 1024);
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % kStagesK, tb = it & 1;
        if (!mbar_wait(&ctl.fullV[s], (it / kStagesK) & 1, wc, 0x62)) break;
        if (it >= 2 && !mbar_wait(&ctl.tmem_free[tb], ((it >> 1) - 1) & 1, wc, 0x63)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t offk = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_ss(tmem + tb * 256, desc_advance(v_k, s * kTileB + offk), desc_advance(ds_k, offk),
                  id_dk, kk != 0);
        }
        if (!mbar_wait(&ctl.kready[s], (it / kStagesK) & 1, wc, 0x64)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t offk = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_ss(tmem + tb * 256 + 128, desc_advance(k_k, s * kTileB + offk),
                  desc_advance(ds_m, kk * 2048), id_dv, kk != 0);
        }
        umma_commit(&ctl.mma_done[tb]);
      }
    }
  } else if (warp < 16) {
    // ---------------- workers: thread = (token row r, column quarter c4)
    const int q4 = warp & 3, c4 = warp >> 2, r = q4 * 32 + lane;
    const int hf = c4 >> 1;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    uint32_t mask[kStagesK] = {0, 0, 0};  // (k > 0) bits of the tile in each k stage
    bool ok = true;
    auto phase_a = [&](int it) {  // k -> k' in place, (k > 0) bits
      const int s = it % kStagesK;
      if (!mbar_wait(&ctl.fullK[s], (it / kStagesK) & 1, wc, 0x65)) {
        ok = false;
        return;
      }
      const int n = (tile0 + it) * kRows + r;
      uint32_t m = 0;
      if (n < g.N) {
        const GlobalRowRope rr = global_row_rope(rope, g, b, n);
        quarter_forward_any<NT, NH>(c4, k_st + s * kTileB, r, rr, nullptr, m);
      }
#pragma unroll
      for (int i = 0; i < kStagesK; ++i)  // static register indexing
        if (i == s) mask[i] = m;
      fence_proxy_async_smem();
      mbar_arrive(&ctl.kready[s]);
    };
    auto phase_b = [&](int it) {  // dk over k', dv over v
      const int s = it % kStagesK, tb = it & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl.mma_done[tb], (it >> 1) & 1, wc, 0x66))) {
        ok = false;
        return;
      }
      tc_fence_after();
      const int n = (tile0 + it) * kRows + r;
      const GlobalRowRope rr = global_row_rope(rope, g, b, n < g.N ? n : 0);
      uint32_t m = 0;
#pragma unroll
      for (int i = 0; i < kStagesK; ++i)
        if (i == s) m = mask[i];
      quarter_backward_any<NT, NH>(c4, k_st + s * kTileB, r, rr, tmem + lane_base + tb * 256, 1.f,
                                   ctl.dz, m, nullptr, nullptr);
      uint8_t* vhalf = v_st + s * kTileB + hf * kHalf;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        uint32_t dvv[16];
        tmem_ld16(tmem + lane_base + tb * 256 + 128 + c4 * 32 + part * 16, dvv);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            w[i] = f2_to_bf2(__uint_as_float(dvv[cc * 8 + 2 * i]),
                             __uint_as_float(dvv[cc * 8 + 2 * i + 1]));
          *reinterpret_cast<uint4*>(vhalf + sw128_off(r, (c4 & 1) * 4 + part * 2 + cc)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl.tmem_free[tb]);
      fence_proxy_async_smem();
      mbar_arrive(&ctl.out_ready[s]);
    };
    if (ntiles > 0) phase_a(0);
    for (int it = 0; ok && it < ntiles; ++it) {
      if (it + 1 < ntiles) {
        phase_a(it + 1);
        if (!ok) break;
      }
      phase_b(it);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    if (*wc.abort_flag)  // MMAs in flight finish before TMEM is freed
      for (int t = ntiles > 2 ? ntiles - 2 : 0; t < ntiles; ++t)
        mbar_drain(&ctl.mma_done[t & 1], (t >> 1) & 1);
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

constexpr size_t kBwdQSmem = 1024 + 6 * (size_t)kTileB;  // S, q x2, dy x2, g
constexpr size_t kBwdKSmem = 1024 + (1 + 2 * kStagesK) * (size_t)kTileB;  // dS, k and v rings
constexpr size_t kSmemPerBlock = 232448;                  // sm_100 opt-in maximum
constexpr int kStdNT = 22, kStdNH = 21;

bool std_split(const RopeDev& r) { return r.n_t == kStdNT && r.n_h == kStdNH && r.n_w == 21; }

void set_bwd_attrs() {
  once_per_context(kAttrLinattnBwd, [] {
    const int q = (int)(kSmemPerBlock - sizeof(BwdQCtl)), k = (int)kBwdKSmem;
    cudaFuncSetAttribute(linattn_bwd_q_kernel<true, kStdNT, kStdNH>, cudaFuncAttributeMaxDynamicSharedMemorySize, q);
    cudaFuncSetAttribute(linattn_bwd_q_kernel<false, kStdNT, kStdNH>, cudaFuncAttributeMaxDynamicSharedMemorySize, q);
    cudaFuncSetAttribute(linattn_bwd_q_kernel<true, -1, -1>, cudaFuncAttributeMaxDynamicSharedMemorySize, q);
    cudaFuncSetAttribute(linattn_bwd_q_kernel<false, -1, -1>, cudaFuncAttributeMaxDynamicSharedMemorySize, q);
    cudaFuncSetAttribute(linattn_bwd_k_kernel<kStdNT, kStdNH>, cudaFuncAttributeMaxDynamicSharedMemorySize, k);
    cudaFuncSetAttribute(linattn_bwd_k_kernel<-1, -1>, cudaFuncAttributeMaxDynamicSharedMemorySize, k);
  });
}

}  // namespace

// Query side, fixed-order combine of dS / dz, key side (S, z come from the
// forward state phase).
sana_status linattn_bf16_backward(const sana_shape& s, const LinAttnPlan& plan, const void* q,
                                  const void* k, const void* v, const void* gt, const void* dy,
                                  const RopeDev& rope, const GridDev& g, float eps,
                                  const float* S, const float* z, float* ws_dS, float* ws_dz,
                                  float* dS, float* dz, void* dq, void* dk, void* dv, void* dg,
                                  cudaStream_t st) {
  const uint64_t C = (uint64_t)s.heads * kD, N = (uint64_t)g.N;
  CUtensorMap tq, tdy, tg, tdq, tdg, tk, tv, tdk, tdv;
  bool okm = make_tmap_bf16_3d(&tq, q, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&tdy, dy, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&tdq, dq, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&tk, k, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&tv, v, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&tdk, dk, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&tdv, dv, C, N, s.B, C, N * C, kRows);
  if (gt)
    okm = okm && make_tmap_bf16_3d(&tg, gt, C, N, s.B, C, N * C, kRows) &&
          make_tmap_bf16_3d(&tdg, dg, C, N, s.B, C, N * C, kRows);
  else
    tg = tdg = tq;
  if (!okm) return fail(SANA_ERR_CUDA, "linattn backward: cuTensorMapEncodeTiled failed");
  if (kBwdQSmem + rope_smem_bytes(g, rope) + sizeof(BwdQCtl) > kSmemPerBlock)
    return fail(SANA_ERR_UNSUPPORTED, "linattn backward: grid %dx%dx%d needs too many RoPE table bytes",
                g.T, g.H, g.W);
  set_bwd_attrs();
  const dim3 grid(plan.splits_a, s.heads, s.B);
  const size_t smq = kBwdQSmem + rope_smem_bytes(g, rope), smk = kBwdKSmem;
  const bool sd = std_split(rope);
  int* sw = status_word();
  if (gt && sd)
    linattn_bwd_q_kernel<true, kStdNT, kStdNH><<<grid, kThreads, smq, st>>>(
        tq, tdy, tg, tdq, tdg, S, z, rope, g, plan.tiles, plan.splits_a, eps, ws_dS, ws_dz, sw);
  else if (gt)
    linattn_bwd_q_kernel<true, -1, -1><<<grid, kThreads, smq, st>>>(
        tq, tdy, tg, tdq, tdg, S, z, rope, g, plan.tiles, plan.splits_a, eps, ws_dS, ws_dz, sw);
  else if (sd)
    linattn_bwd_q_kernel<false, kStdNT, kStdNH><<<grid, kThreads, smq, st>>>(
        tq, tdy, tg, tdq, tdg, S, z, rope, g, plan.tiles, plan.splits_a, eps, ws_dS, ws_dz, sw);
  else
    linattn_bwd_q_kernel<false, -1, -1><<<grid, kThreads, smq, st>>>(
        tq, tdy, tg, tdq, tdg, S, z, rope, g, plan.tiles, plan.splits_a, eps, ws_dS, ws_dz, sw);
  if (sana_status e = check_launch("linattn_bwd_q_kernel")) return e;
  launch_linattn_combine(s.B * s.heads, ws_dS, ws_dz, plan.splits_a, kD, nullptr, nullptr, nullptr,
                         nullptr, dS, dz, st);
  if (sana_status e = check_launch("linattn_combine_kernel")) return e;
  if (sd)
    linattn_bwd_k_kernel<kStdNT, kStdNH><<<grid, kThreads, smk, st>>>(
        tk, tv, tdk, tdv, dS, dz, rope, g, plan.tiles, plan.splits_a, sw);
  else
    linattn_bwd_k_kernel<-1, -1><<<grid, kThreads, smk, st>>>(
        tk, tv, tdk, tdv, dS, dz, rope, g, plan.tiles, plan.splits_a, sw);
  return check_launch("linattn_bwd_k_kernel");
}

}  // namespace sana
