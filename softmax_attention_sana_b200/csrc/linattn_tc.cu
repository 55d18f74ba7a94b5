// Gated ReLU linear attention with RoPE after the ReLU, bf16 on tcgen05.
//
//   "SANA-Video" paper notes, sec. 3.2 (equation for O_i, pseudocode):
//     S = sum_j RoPE(phi K_j)^T V_j,  z = sum_j phi K_j,
//     O_i = RoPE(phi Q_i) S / (phi Q_i . z + eps)
//   sec. 3.4 (causal form, cumulative state S, z), Algorithm 1 (state update).
//   "SANA-Video 2.0" abstract: gated linear attention; gate = sigmoid(G).
//
// Three kernels per call:
//   state   per (batch, head, split): TMA K, V tiles (128 tokens x 128) ->
//           ReLU + RoPE of K in shared memory (z accumulated on the way) ->
//           tcgen05 D[d][e] += K'^T V with fp32 accumulation in TMEM ->
//           partial S and z to the workspace.
//   combine per (batch, head, slice of S): fixed-order sum of the split
//           partials (plus the carried state in block-causal mode).
//   output  per (batch, head, split): S (fp32) -> bf16 S^T operand in shared
//           memory once per CTA; TMA Q, G tiles -> ReLU + RoPE of Q and the
//           RoPE-free denominator phi(Q).z in registers -> tcgen05 D = Q' S ->
//           epilogue divides, gates with sigmoid(G), stores bf16 through
//           shared memory with TMA.
//
// Workers are 16 warps: warp w owns TMEM lane quarter w % 4 (token rows
// 32(w%4) .. +31) and column quarter w / 4 (32 of the 128 head dims), so each
// thread transforms one 64-byte run of one token row per tile.  The rotary
// split 22/21/21 of the 128-dim heads is compiled in (pair-to-axis selection
// folds away); other splits take the general path.
#include <cuda.h>

#include <cstddef>

#include "pdl.cuh"
#include "rope_dev.cuh"
#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {
namespace {

constexpr int kD = 128;
constexpr int kRows = 128;                // tokens per tile
constexpr int kHalf = kRows * 64 * 2;     // one 64-column half of a tile: 16 KB
constexpr int kTileB = 2 * kHalf;         // 32 KB
constexpr int kWorkers = 512;             // 16 warps: (row quarter, column quarter)
constexpr int kThreadsA = kWorkers + 64;  // + producer warp + MMA warp
constexpr int kStagesA = 3;
constexpr int kStagesQ = 3;
constexpr int kStagesG = 2;
constexpr int kThreadsB = kWorkers + 96;  // + Q producer, MMA, G producer
constexpr int kWarpProdA = 16, kWarpMmaA = 17;
constexpr int kWarpProdQ = 16, kWarpMmaB = 17, kWarpProdG = 18;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// (cos, sin) of rotary pair j.  NT >= 0: the split is a compile-time constant
// and, with j unrolled, the axis selection is resolved by the compiler.
template <int NT, int NH>
__device__ __forceinline__ float2 pair_cs(const RowRope& rr, int j) {
  if (NT >= 0) return j < NT ? rr.pt[j] : (j < NT + NH ? rr.ph[j - NT] : rr.pw[j - NT - NH]);
  return rr.cs(j);
}

// ---- packed arithmetic: one instruction for two columns
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void up2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
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
// max(x, 0) of both bf16 halves
__device__ __forceinline__ uint32_t relu_bf2(uint32_t w) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(0u));
  return r;
}
// sigmoid of both bf16 halves of w (gate logits) as f32x2, by the tanh
// identity sigmoid(x) = 1/2 + tanh(x/2)/2 (one MUFU op per value).  Its
// absolute error is about 2.5e-4 (tanh.approx), i.e. a relative error below
// 1.5% while sigmoid(x) >= sigmoid(-4); below that the gated output is under
// 2% of the ungated one and its relative error grows.  An exact form (one
// exponential and the reciprocal by Newton steps, as sigmoid_fast), even taken
// only for chunks holding logits below -4, made this pass about 10% slower
// (measured side by side), so the epilogue keeps the tanh identity.
__device__ __forceinline__ uint64_t sigmoid2(uint32_t w) {
  const float2 g = bf2_to_f2(w);
  float t0, t1;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t0) : "f"(0.5f * g.x));
  asm("tanh.approx.f32 %0, %1;" : "=f"(t1) : "f"(0.5f * g.y));
  return fma2(pk2(t0, t1), pk2(0.5f, 0.5f), pk2(0.5f, 0.5f));
}

// ReLU + RoPE of one 16-byte chunk (4 rotary pairs starting at pair0) of a
// swizzled tile row, rewritten in place; the ReLU values are returned.
template <int NT, int NH>
__device__ __forceinline__ void relu_rope_chunk(uint8_t* p, const RowRope& rr, int pair0,
                                                float (&phi_out)[8]) {
  uint4 raw = *reinterpret_cast<uint4*>(p);
  uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = bf2_to_f2(relu_bf2(w[i]));  // exact: ReLU commutes with widening
    phi_out[2 * i] = x.x;
    phi_out[2 * i + 1] = x.y;
    const float2 r = rotate(x.x, x.y, pair_cs<NT, NH>(rr, pair0 + i));
    w[i] = f2_to_bf2(r.x, r.y);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Column quarter C4 of token row r: chunks 4*(C4&1) .. +3 of half C4>>1.
template <int NT, int NH, int C4>
__device__ __forceinline__ void quarter_state(uint8_t* tile, int r, const RowRope& rr,
                                              float (&zacc)[32]) {
  uint8_t* half = tile + (C4 >> 1) * kHalf;
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    float ph[8];
    relu_rope_chunk<NT, NH>(half + sw128_off(r, (C4 & 1) * 4 + ch), rr, C4 * 16 + ch * 4, ph);
#pragma unroll
    for (int i = 0; i < 8; ++i) zacc[ch * 8 + i] += ph[i];
  }
}

template <int NT, int NH, int C4>
__device__ __forceinline__ float quarter_query(uint8_t* tile, int r, const RowRope& rr,
                                               const float* z) {
  uint8_t* half = tile + (C4 >> 1) * kHalf;
  uint64_t den2 = pk2(0.f, 0.f);  // even and odd columns, summed at the end
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    float ph[8];
    relu_rope_chunk<NT, NH>(half + sw128_off(r, (C4 & 1) * 4 + ch), rr, C4 * 16 + ch * 4, ph);
    const float4 z0 = *reinterpret_cast<const float4*>(z + C4 * 32 + ch * 8);
    const float4 z1 = *reinterpret_cast<const float4*>(z + C4 * 32 + ch * 8 + 4);
    den2 = fma2(pk2(ph[0], ph[1]), pk2(z0.x, z0.y), den2);
    den2 = fma2(pk2(ph[2], ph[3]), pk2(z0.z, z0.w), den2);
    den2 = fma2(pk2(ph[4], ph[5]), pk2(z1.x, z1.y), den2);
    den2 = fma2(pk2(ph[6], ph[7]), pk2(z1.z, z1.w), den2);
  }
  float d0, d1;
  up2(den2, d0, d1);
  return d0 + d1;
}

// ------------------------------------------------------------------------
// state kernel
// ------------------------------------------------------------------------
struct StateSmemCtl {
  uint64_t full[kStagesA];
  uint64_t kready[kStagesA];
  uint64_t empty[kStagesA];
  uint64_t done;
  uint32_t tmem;
  int abort_flag;
};

template <int NT, int NH>
__global__ void __launch_bounds__(kThreadsA, 1)
    linattn_state_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, RopeDev rope, GridDev g,
                         int tiles_total, int splits, float* __restrict__ ws_S,
                         float* __restrict__ ws_z, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ StateSmemCtl ctl;
  uint8_t* smem = align1024(smem_raw);
  uint8_t* stages = smem;
  float2* rope_base = reinterpret_cast<float2*>(smem + kStagesA * 2 * kTileB);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tile0 = (int)((long long)split * tiles_total / splits);
  const int ntiles = (int)((long long)(split + 1) * tiles_total / splits) - tile0;
  const WaitCtx wc{&ctl.abort_flag, status};
  volatile int* abort_flag = &ctl.abort_flag;
  griddep_launch_next();

  if (tid == 0) {
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.kready[s], kWorkers);
      mbar_init(&ctl.empty[s], 1);
    }
    mbar_init(&ctl.done, 1);
    ctl.abort_flag = 0;
    mbar_fence_init();
    // K and V are inputs of an ordinarily launched kernel, complete when it
    // starts: the first stages load while the RoPE tables are staged
    fence_proxy_async_smem();
    for (int it = 0; it < kStagesA && it < ntiles; ++it) {
      const int n0 = (tile0 + it) * kRows;
      uint8_t* st = stages + it * 2 * kTileB;
      mbar_arrive_expect_tx(&ctl.full[it], 2 * kTileB);
      tma_load_3d(st, &tm_k, &ctl.full[it], h * kD, n0, b);
      tma_load_3d(st + kHalf, &tm_k, &ctl.full[it], h * kD + 64, n0, b);
      tma_load_3d(st + kTileB, &tm_v, &ctl.full[it], h * kD, n0, b);
      tma_load_3d(st + kTileB + kHalf, &tm_v, &ctl.full[it], h * kD + 64, n0, b);
    }
  }
  if (warp == kWarpMmaA) {
    tmem_alloc(&ctl.tmem, 128);
    tmem_relinquish();
  }
  const RopeSmem rs = rope_stage(rope_base, rope, g, b, tid, kThreadsA);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;

  if (warp == kWarpProdA) {
    // ---------------- TMA producer
    if (lane == 0) {
      int issued = ntiles < kStagesA ? ntiles : kStagesA;  // loaded at the start
      for (int it = kStagesA; it < ntiles; ++it) {
        const int s = it % kStagesA;
        if (it >= kStagesA && !mbar_wait(&ctl.empty[s], ((it / kStagesA) - 1) & 1, wc, 0x11))
          break;
        const int n0 = (tile0 + it) * kRows;
        uint8_t* st = stages + s * 2 * kTileB;
        mbar_arrive_expect_tx(&ctl.full[s], 2 * kTileB);
        tma_load_3d(st, &tm_k, &ctl.full[s], h * kD, n0, b);
        tma_load_3d(st + kHalf, &tm_k, &ctl.full[s], h * kD + 64, n0, b);
        tma_load_3d(st + kTileB, &tm_v, &ctl.full[s], h * kD, n0, b);
        tma_load_3d(st + kTileB + kHalf, &tm_v, &ctl.full[s], h * kD + 64, n0, b);
        ++issued;
      }
      if (*abort_flag) {  // drain loads still in flight before the CTA exits
        for (int it = issued > kStagesA ? issued - kStagesA : 0; it < issued; ++it)
          mbar_drain(&ctl.full[it % kStagesA], (it / kStagesA) & 1);
      }
    }
  } else if (warp == kWarpMmaA) {
    // ---------------- MMA issuer: D[d][e] += K'[tok][d]^T V[tok][e]
    if (lane == 0) {
      // A = K' (M = d, MN-major), B = V (N = e, MN-major), both 128B-swizzled
      // [2 halves of 64][128 tokens]; LBO = distance of the 64-column halves,
      // SBO = distance of 8-token groups.
      const uint32_t idesc = idesc_bf16_f32(128, 128, 1, 1);
      // built once; stages and K steps advance the start address
      const uint64_t dk0 = smem_desc_sw128(smem_u32(stages), kHalf, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_u32(stages + kTileB), kHalf, 1024);
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % kStagesA;
        if (!mbar_wait(&ctl.kready[s], (it / kStagesA) & 1, wc, 0x12)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          umma_ss(tmem, desc_advance(dk0, s * 2 * kTileB + kk * 2048),
                  desc_advance(dv0, s * 2 * kTileB + kk * 2048), idesc, (it | kk) != 0);
        umma_commit(&ctl.empty[s]);
      }
      umma_commit(&ctl.done);
    }
  } else if (warp < 16) {
    // ---------------- workers: thread = (token row r, column quarter c4)
    const int q4 = warp & 3, c4 = warp >> 2, r = q4 * 32 + lane;
    float zacc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) zacc[i] = 0.f;
    for (int it = 0; it < ntiles; ++it) {
      const int s = it % kStagesA;
      if (!mbar_wait(&ctl.full[s], (it / kStagesA) & 1, wc, 0x13)) break;
      const int n = (tile0 + it) * kRows + r;
      if (n < g.N) {  // rows past N were zero-filled by TMA: phi = RoPE = 0
        const RowRope rr = row_rope(rs, g, n);
        uint8_t* tile = stages + s * 2 * kTileB;
        switch (c4) {  // warp-uniform
          case 0: quarter_state<NT, NH, 0>(tile, r, rr, zacc); break;
          case 1: quarter_state<NT, NH, 1>(tile, r, rr, zacc); break;
          case 2: quarter_state<NT, NH, 2>(tile, r, rr, zacc); break;
          default: quarter_state<NT, NH, 3>(tile, r, rr, zacc); break;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&ctl.kready[s]);
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&ctl.done, 0, wc, 0x14));
    tc_fence_after();
    const size_t part = ((size_t)(b * g.heads + h) * splits + split);
    if (ok) {
      float* Sout = ws_S + part * kD * kD;
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + c4 * 32, v);
      tmem_ld_wait();
      float4* dst = reinterpret_cast<float4*>(Sout + (size_t)r * kD + c4 * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                             __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
    }
    // z: reduce the per-row partial sums over the 128 rows of each column
    // quarter in a fixed order (stride 33 keeps both passes conflict-free).
    float* red = reinterpret_cast<float*>(stages);
#pragma unroll
    for (int i = 0; i < 32; ++i) red[(c4 * 128 + r) * 33 + i] = zacc[i];
    named_bar_sync(1, kWorkers);
    if (tid < 128) {
      const int cc = tid >> 5, i = tid & 31;
      float acc = 0.f;
      for (int rr = 0; rr < 128; ++rr) acc += red[(cc * 128 + rr) * 33 + i];
      ws_z[part * kD + cc * 32 + i] = acc;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMmaA) {
    if (*abort_flag) mbar_drain(&ctl.done, 0);  // MMAs in flight finish before TMEM is freed
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------------------
// combine kernel (shared with the fp32 path): fixed-order sum over splits.
// Grid (batch * heads, slices): each CTA sums one slice of one head's S.
// Every element is S_prev + p_0 + p_1 + ... in that order; a thread owns four
// consecutive elements and issues the loads of up to kCombineBatch splits
// before it adds them, so the reduction is bound by bandwidth, not by the
// latency of one load after another.
// ------------------------------------------------------------------------
constexpr int kCombineSlices = 16;
constexpr int kCombineBatch = 8;

__device__ __forceinline__ void add4(float4& a, const float4& b) {
  a.x += b.x;
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
}

__global__ void __launch_bounds__(256)
    linattn_combine_kernel(const float* __restrict__ ws_S, const float* __restrict__ ws_z,
                           int splits, int D, const float* S_prev, const float* z_prev,
                           float* S_state, float* z_state, float* __restrict__ S_f32,
                           float* __restrict__ z_out) {
  griddep_wait();  // the partials come from the previous launch
  griddep_launch_next();
  const int bh = blockIdx.x;
  const int DD = D * D;
  const size_t base = (size_t)bh * DD;
  const uintptr_t addr_bits = reinterpret_cast<uintptr_t>(ws_S) |
                              reinterpret_cast<uintptr_t>(S_prev) |
                              reinterpret_cast<uintptr_t>(S_state) | reinterpret_cast<uintptr_t>(S_f32);
  if ((DD & 3) == 0 && (addr_bits & 15u) == 0) {
    // float4 path: with DD a multiple of 4 and 16-byte aligned buffers every
    // access is aligned
    const int DD4 = DD >> 2;
    const int per = (DD4 + (int)gridDim.y - 1) / (int)gridDim.y;
    const int beg = (int)blockIdx.y * per;
    const int end = min(DD4, beg + per);
    const float4* part = reinterpret_cast<const float4*>(ws_S) + (size_t)bh * splits * DD4;
    for (int i = beg + threadIdx.x; i < end; i += blockDim.x) {
      float4 acc = S_prev ? reinterpret_cast<const float4*>(S_prev + base)[i]
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = 0; s0 < splits; s0 += kCombineBatch) {
        float4 p[kCombineBatch];
#pragma unroll
        for (int j = 0; j < kCombineBatch; ++j)
          if (s0 + j < splits) p[j] = part[(size_t)(s0 + j) * DD4 + i];
#pragma unroll
        for (int j = 0; j < kCombineBatch; ++j)
          if (s0 + j < splits) add4(acc, p[j]);
      }
      if (S_state) reinterpret_cast<float4*>(S_state + base)[i] = acc;
      if (S_f32) reinterpret_cast<float4*>(S_f32 + base)[i] = acc;
    }
  } else {
    const int per = (DD + (int)gridDim.y - 1) / (int)gridDim.y;
    const int beg = (int)blockIdx.y * per;
    const int end = min(DD, beg + per);
    for (int idx = beg + threadIdx.x; idx < end; idx += blockDim.x) {
      float acc = S_prev ? S_prev[base + idx] : 0.f;
      for (int sp = 0; sp < splits; ++sp) acc += ws_S[((size_t)bh * splits + sp) * DD + idx];
      if (S_state) S_state[base + idx] = acc;
      if (S_f32) S_f32[base + idx] = acc;
    }
  }
  if (blockIdx.y == 0)
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      float acc = z_prev ? z_prev[(size_t)bh * D + d] : 0.f;
      for (int sp = 0; sp < splits; ++sp) acc += ws_z[((size_t)bh * splits + sp) * D + d];
      if (z_state) z_state[(size_t)bh * D + d] = acc;
      if (z_out) z_out[(size_t)bh * D + d] = acc;
    }
}

// ------------------------------------------------------------------------
// output kernel
// ------------------------------------------------------------------------
struct OutSmemCtl {
  uint64_t fullQ[kStagesQ], emptyQ[kStagesQ], qready[kStagesQ];
  uint64_t fullG[kStagesG], ystaged[kStagesG];
  uint64_t mma_done[2], tmem_free[2];
  uint64_t wsync;  // reusable worker barrier (bounded waits)
  uint32_t tmem;
  int abort_flag;
  alignas(16) float den[kStagesQ][4][kRows];
  alignas(16) float z[kD];  // read as float4
};
static_assert(offsetof(OutSmemCtl, z) % 16 == 0, "z is read with 16-byte loads");

template <bool kGate, int NT, int NH>
__global__ void __launch_bounds__(kThreadsB, 1)
    linattn_out_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_g,
                       const __grid_constant__ CUtensorMap tm_y, const float* __restrict__ S_all,
                       const float* __restrict__ z_all, RopeDev rope, GridDev g, int tiles_total,
                       int splits, float eps, int prefetch, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ OutSmemCtl ctl;
  uint8_t* smem = align1024(smem_raw);
  uint8_t* s_op = smem;                             // S^T operand, 32 KB
  uint8_t* q_st = s_op + kTileB;                    // Q stages
  uint8_t* g_st = q_st + kStagesQ * kTileB;         // G / Y stages
  float2* rope_base = reinterpret_cast<float2*>(g_st + kStagesG * kTileB);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tile0 = (int)((long long)split * tiles_total / splits);
  const int ntiles = (int)((long long)(split + 1) * tiles_total / splits) - tile0;
  const int bh = b * g.heads + h;
  const WaitCtx wc{&ctl.abort_flag, status};

  if (tid == 0) {
    for (int s = 0; s < kStagesQ; ++s) {
      mbar_init(&ctl.fullQ[s], 1);
      mbar_init(&ctl.emptyQ[s], 1);
      mbar_init(&ctl.qready[s], kWorkers);
    }
    for (int s = 0; s < kStagesG; ++s) {
      mbar_init(&ctl.fullG[s], 1);
      mbar_init(&ctl.ystaged[s], kWorkers);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.mma_done[i], 1);
      mbar_init(&ctl.tmem_free[i], kWorkers);
    }
    mbar_init(&ctl.wsync, kWorkers);
    ctl.abort_flag = 0;
    mbar_fence_init();
    if (prefetch) {
      // Q and G are inputs of the whole call, complete before its first
      // kernel started: their first tiles load while the previous launch
      // (which produces S and z) finishes
      fence_proxy_async_smem();
      for (int it = 0; it < kStagesQ && it < ntiles; ++it) {
        const int n0 = (tile0 + it) * kRows;
        mbar_arrive_expect_tx(&ctl.fullQ[it], kTileB);
        tma_load_3d(q_st + it * kTileB, &tm_q, &ctl.fullQ[it], h * kD, n0, b);
        tma_load_3d(q_st + it * kTileB + kHalf, &tm_q, &ctl.fullQ[it], h * kD + 64, n0, b);
      }
      if (kGate)
        for (int it = 0; it < kStagesG && it < ntiles; ++it) {
          const int n0 = (tile0 + it) * kRows;
          mbar_arrive_expect_tx(&ctl.fullG[it], kTileB);
          tma_load_3d(g_st + it * kTileB, &tm_g, &ctl.fullG[it], h * kD, n0, b);
          tma_load_3d(g_st + it * kTileB + kHalf, &tm_g, &ctl.fullG[it], h * kD + 64, n0, b);
        }
    }
  }
  if (warp == kWarpMmaB) {
    tmem_alloc(&ctl.tmem, 256);
    tmem_relinquish();
  }
  // everything above overlaps the previous launch's tail; S and z (and Q, G)
  // are read only after it has finished.  Where the call's inputs are known
  // complete (prefetch), the RoPE tables are staged before the wait too.
  RopeSmem rs{};
  if (prefetch) rs = rope_stage(rope_base, rope, g, b, tid, kThreadsB);
  griddep_wait();
  if (tid < kD) ctl.z[tid] = z_all[(size_t)bh * kD + tid];
  if (tid < kWorkers) {
    // S^T operand: element (e, d) = S[d][e] in bf16, K-major [2 halves of
    // 64 d][128 e rows] with the 128-byte swizzle.  Thread = (row e, d quarter).
    const int e = tid & 127, qd = tid >> 7;
    const float* Sh = S_all + (size_t)bh * kD * kD + (size_t)(qd * 32) * kD + e;
    uint8_t* dst = s_op + (qd >> 1) * kHalf;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        wv[i] = f2_to_bf2(Sh[(ch * 8 + 2 * i) * kD], Sh[(ch * 8 + 2 * i + 1) * kD]);
      *reinterpret_cast<uint4*>(dst + sw128_off(e, (qd & 1) * 4 + ch)) =
          make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
    fence_proxy_async_smem();
  }
  if (!prefetch) rs = rope_stage(rope_base, rope, g, b, tid, kThreadsB);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;

  if (warp == kWarpProdQ) {
    // ---------------- Q producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      for (int it = prefetch ? kStagesQ : 0; it < ntiles; ++it) {
        const int s = it % kStagesQ;
        if (it >= kStagesQ && !mbar_wait(&ctl.emptyQ[s], ((it / kStagesQ) - 1) & 1, wc, 0x21))
          break;
        const int n0 = (tile0 + it) * kRows;
        mbar_arrive_expect_tx(&ctl.fullQ[s], kTileB);
        tma_load_3d(q_st + s * kTileB, &tm_q, &ctl.fullQ[s], h * kD, n0, b);
        tma_load_3d(q_st + s * kTileB + kHalf, &tm_q, &ctl.fullQ[s], h * kD + 64, n0, b);
      }
    }
  } else if (warp == kWarpProdG) {
    // ---------------- G producer and Y store.  Stage s holds G of a tile, the
    // workers overwrite it with that tile's Y, this thread stores Y by TMA and
    // refills the stage once the store has read it (the workers never wait
    // for a store).  Ungated, the stages only stage Y.
    if (lane == 0) {
      if (kGate) prefetch_tmap(&tm_g);
      prefetch_tmap(&tm_y);
      auto store_y = [&](int t) {  // Y of tile t, once all its rows are staged
        const int st = t % kStagesG;
        if (!mbar_wait(&ctl.ystaged[st], (t / kStagesG) & 1, wc, 0x22)) return false;
        uint8_t* src = g_st + st * kTileB;
        tma_store_3d(&tm_y, src, h * kD, (tile0 + t) * kRows, b);
        tma_store_3d(&tm_y, src + kHalf, h * kD + 64, (tile0 + t) * kRows, b);
        bulk_commit();
        return true;
      };
      bool okp = true;
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % kStagesG;
        if (it >= kStagesG) {
          okp = store_y(it - kStagesG);
          if (!okp) break;
          bulk_wait_read0();  // the stage has been read out
        }
        if (kGate && prefetch && it < kStagesG) {
          // loaded before the launch waited
        } else if (kGate) {
          const int n0 = (tile0 + it) * kRows;
          mbar_arrive_expect_tx(&ctl.fullG[s], kTileB);
          tma_load_3d(g_st + s * kTileB, &tm_g, &ctl.fullG[s], h * kD, n0, b);
          tma_load_3d(g_st + s * kTileB + kHalf, &tm_g, &ctl.fullG[s], h * kD + 64, n0, b);
        } else {
          mbar_arrive(&ctl.fullG[s]);
        }
      }
      for (int t = ntiles > kStagesG ? ntiles - kStagesG : 0; okp && t < ntiles; ++t)
        okp = store_y(t);
      bulk_wait0();
    }
  } else if (warp == kWarpMmaB) {
    // ---------------- MMA issuer: D[tok][e] = Q'[tok][d] S[d][e]
    if (lane == 0) {
      // A = Q' (K-major, [2 halves][128 tok][64 d]), B = S^T (K-major,
      // [2 halves][128 e][64 d]); a K step of 16 advances 32 bytes in a half.
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      const uint64_t ds = smem_desc_sw128(smem_u32(s_op), 16, 1024);
      const uint64_t dq0 = smem_desc_sw128(smem_u32(q_st), 16, 1024);  // stages, K steps: advance
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % kStagesQ, tb = it & 1;
        if (!mbar_wait(&ctl.qready[s], (it / kStagesQ) & 1, wc, 0x24)) break;
        if (it >= 2 && !mbar_wait(&ctl.tmem_free[tb], ((it >> 1) - 1) & 1, wc, 0x25)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_ss(tmem + tb * 128, desc_advance(dq0, s * kTileB + off), desc_advance(ds, off), idesc,
                  kk != 0);
        }
        umma_commit(&ctl.emptyQ[s]);
        umma_commit(&ctl.mma_done[tb]);
      }
    }
  } else if (warp < 16) {
    // ---------------- workers: thread = (token row r, column quarter c4)
    const int q4 = warp & 3, c4 = warp >> 2, r = q4 * 32 + lane;
    const int hf = c4 >> 1;  // the 64-column half holding this thread's columns
    bool ok = true;
    auto prologue = [&](int it) {
      const int s = it % kStagesQ;
      if (!mbar_wait(&ctl.fullQ[s], (it / kStagesQ) & 1, wc, 0x26)) {
        ok = false;
        return;
      }
      const int n = (tile0 + it) * kRows + r;
      float den = 0.f;
      if (n < g.N) {
        const RowRope rr = row_rope(rs, g, n);
        uint8_t* tile = q_st + s * kTileB;
        switch (c4) {  // warp-uniform
          case 0: den = quarter_query<NT, NH, 0>(tile, r, rr, ctl.z); break;
          case 1: den = quarter_query<NT, NH, 1>(tile, r, rr, ctl.z); break;
          case 2: den = quarter_query<NT, NH, 2>(tile, r, rr, ctl.z); break;
          default: den = quarter_query<NT, NH, 3>(tile, r, rr, ctl.z); break;
        }
      }
      ctl.den[s][c4][r] = den;
      fence_proxy_async_smem();
      mbar_arrive(&ctl.qready[s]);
    };
    uint32_t n_wsync = 0;
    auto epilogue = [&](int it) {
      const int s = it % kStagesQ, tb = it & 1, sg = it % kStagesG;
      bool okw = mbar_wait(&ctl.mma_done[tb], (it >> 1) & 1, wc, 0x27);
      // every column quarter has written its partial denominator
      mbar_arrive(&ctl.wsync);
      okw = mbar_wait(&ctl.wsync, (n_wsync++) & 1, wc, 0x29) && okw;
      okw = __all_sync(0xffffffffu, okw);  // tcgen05.ld is warp-collective
      const float inv =
          1.f / (ctl.den[s][0][r] + ctl.den[s][1][r] + ctl.den[s][2][r] + ctl.den[s][3][r] + eps);
      const uint64_t inv2 = pk2(inv, inv);
      uint32_t acc[32];
      if (okw) {
        tc_fence_after();
        tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + tb * 128 + c4 * 32, acc);
        tmem_ld_wait();
      }
      tc_fence_before();
      mbar_arrive(&ctl.tmem_free[tb]);
      okw = mbar_wait(&ctl.fullG[sg], (it / kStagesG) & 1, wc, 0x28) && okw;
      uint8_t* half = g_st + sg * kTileB + hf * kHalf;
      if (okw) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint4* p = reinterpret_cast<uint4*>(half + sw128_off(r, (c4 & 1) * 4 + ch));
          uint32_t gw[4] = {0, 0, 0, 0};
          if (kGate) {
            const uint4 graw = *p;
            gw[0] = graw.x; gw[1] = graw.y; gw[2] = graw.z; gw[3] = graw.w;
          }
          uint32_t out[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint64_t y2 = mul2(pk2(__uint_as_float(acc[ch * 8 + 2 * i]),
                                   __uint_as_float(acc[ch * 8 + 2 * i + 1])),
                               inv2);
            if (kGate) y2 = mul2(y2, sigmoid2(gw[i]));
            float y0, y1;
            up2(y2, y0, y1);
            out[i] = f2_to_bf2(y0, y1);
          }
          *p = make_uint4(out[0], out[1], out[2], out[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&ctl.ystaged[sg]);  // the G producer stores the tile
      ok = okw;
    };
    if (ntiles > 0) prologue(0);
    for (int it = 0; ok && it < ntiles; ++it) {
      if (it + 1 < ntiles) prologue(it + 1);
      if (!ok) break;
      epilogue(it);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMmaB) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

constexpr size_t kStateSmem = 1024 + kStagesA * 2 * kTileB;
constexpr size_t kOutSmem = 1024 + kTileB + kStagesQ * kTileB + kStagesG * kTileB;

// The standard split of 128-dim heads (64 rotary pairs over t / h / w).
constexpr int kStdNT = 22, kStdNH = 21;

bool is_std_split(const RopeDev& r) { return r.n_t == kStdNT && r.n_h == kStdNH && r.n_w == 21; }

template <class K>
void smem_attr(K kernel, size_t bytes) {
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

void set_smem_attrs() {
  once_per_context(kAttrLinattn, [] {
    smem_attr(linattn_state_kernel<kStdNT, kStdNH>, kStateSmem + kRopeSmemMax);
    smem_attr(linattn_state_kernel<-1, -1>, kStateSmem + kRopeSmemMax);
    smem_attr(linattn_out_kernel<true, kStdNT, kStdNH>, kOutSmem + kRopeSmemMax);
    smem_attr(linattn_out_kernel<false, kStdNT, kStdNH>, kOutSmem + kRopeSmemMax);
    smem_attr(linattn_out_kernel<true, -1, -1>, kOutSmem + kRopeSmemMax);
    smem_attr(linattn_out_kernel<false, -1, -1>, kOutSmem + kRopeSmemMax);
  });
}

}  // namespace

// ------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------

// Split reduction only: partial S and z of every (batch entry, head, split)
// into ws_S [B][heads][splits][D][D] and ws_z [B][heads][splits][D].
sana_status linattn_bf16_partials(const sana_shape& s, const LinAttnPlan& plan, const void* k,
                                  const void* v, const RopeDev& rope, const GridDev& g,
                                  float* ws_S, float* ws_z, cudaStream_t st) {
  const uint64_t C = (uint64_t)s.heads * kD, N = (uint64_t)g.N;
  CUtensorMap tk, tv;
  if (!make_tmap_bf16_3d(&tk, k, C, N, s.B, C, N * C, kRows) ||
      !make_tmap_bf16_3d(&tv, v, C, N, s.B, C, N * C, kRows))
    return fail(SANA_ERR_CUDA, "linattn: cuTensorMapEncodeTiled failed");
  set_smem_attrs();
  const size_t smem_a = kStateSmem + rope_smem_bytes(g, rope);
  const dim3 grid(plan.splits_a, s.heads, s.B);
  if (is_std_split(rope))
    linattn_state_kernel<kStdNT, kStdNH><<<grid, kThreadsA, smem_a, st>>>(
        tk, tv, rope, g, plan.tiles, plan.splits_a, ws_S, ws_z, status_word());
  else
    linattn_state_kernel<-1, -1><<<grid, kThreadsA, smem_a, st>>>(
        tk, tv, rope, g, plan.tiles, plan.splits_a, ws_S, ws_z, status_word());
  return check_launch("linattn_state_kernel");
}

// State phase: split reduction + fixed-order combine into S_f32 / z_out
// (and the carried state when committing).
sana_status linattn_bf16_state(const sana_shape& s, const LinAttnPlan& plan, const void* k,
                               const void* v, const RopeDev& rope, const GridDev& g,
                               const float* S_prev, const float* z_prev, float* S_state,
                               float* z_state, float* ws_S, float* ws_z, float* S_f32,
                               float* z_out, cudaStream_t st) {
  if (sana_status e = linattn_bf16_partials(s, plan, k, v, rope, g, ws_S, ws_z, st)) return e;
  const cudaError_t e = launch_dependent(linattn_combine_kernel, dim3(s.B * s.heads, kCombineSlices),
                                         dim3(256), 0, st, ws_S, ws_z, plan.splits_a, kD, S_prev,
                                         z_prev, S_state, z_state, S_f32, z_out);
  if (e != cudaSuccess) return fail(SANA_ERR_CUDA, "linattn_combine_kernel: %s", cudaGetErrorString(e));
  return check_launch("linattn_combine_kernel");
}

// Output phase: one kernel launch.
sana_status linattn_bf16_apply(const sana_shape& s, const LinAttnPlan& plan, const void* q,
                               const void* gt, const RopeDev& rope, const GridDev& g,
                               const float* S_f32, const float* z, float eps, void* out,
                               cudaStream_t st, bool prefetch_inputs) {
  const uint64_t C = (uint64_t)s.heads * kD, N = (uint64_t)g.N;
  CUtensorMap tq, tg, ty;
  bool okm = make_tmap_bf16_3d(&tq, q, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&ty, out, C, N, s.B, C, N * C, kRows);
  if (gt) okm = okm && make_tmap_bf16_3d(&tg, gt, C, N, s.B, C, N * C, kRows);
  else tg = tq;
  if (!okm) return fail(SANA_ERR_CUDA, "linattn: cuTensorMapEncodeTiled failed");
  set_smem_attrs();
  const size_t smem_b = kOutSmem + rope_smem_bytes(g, rope);
  const dim3 grid(plan.splits_b, s.heads, s.B);
  const bool stdsp = is_std_split(rope);
  int* sw = status_word();
  // launched as a programmatic dependent: its prologue overlaps the tail of
  // the launch that produces S and z
  auto kern = gt ? (stdsp ? linattn_out_kernel<true, kStdNT, kStdNH> : linattn_out_kernel<true, -1, -1>)
                 : (stdsp ? linattn_out_kernel<false, kStdNT, kStdNH>
                          : linattn_out_kernel<false, -1, -1>);
  const cudaError_t e = launch_dependent(kern, grid, dim3(kThreadsB), smem_b, st, tq, tg, ty, S_f32,
                                         z, rope, g, plan.tiles, plan.splits_b, eps,
                                         prefetch_inputs ? 1 : 0, sw);
  if (e != cudaSuccess) return fail(SANA_ERR_CUDA, "linattn_out_kernel: %s", cudaGetErrorString(e));
  return check_launch("linattn_out_kernel");
}

// The fp32 path reuses the combine kernel.
void launch_linattn_combine(int BH, const float* ws_S, const float* ws_z, int splits, int D,
                            const float* S_prev, const float* z_prev, float* S_state,
                            float* z_state, float* S_f32, float* z_out, cudaStream_t st) {
  linattn_combine_kernel<<<dim3(BH, kCombineSlices), 256, 0, st>>>(
      ws_S, ws_z, splits, D, S_prev, z_prev, S_state, z_state, S_f32, z_out);
}

}  // namespace sana
