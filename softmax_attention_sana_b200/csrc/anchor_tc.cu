// Gated softmax anchor, bf16 on tcgen05 ("SANA-Video 2.0" abstract: gated
// softmax anchors every fourth layer; reading: the same 3D RoPE on Q and K,
// scale 1/sqrt(D)).
//
//   Y = sigmoid(G) * softmax(Q' K'^T) V   with Q' = RoPE(Q) * scale * log2(e),
//   K' = RoPE(K) prepared by a rotation pass, so the softmax works in base 2.
//
// One CTA per (batch, head, pair of 128-query tiles).  Both query tiles share
// every K'/V tile, and their softmax warpgroups ping-pong with the tensor core:
//   producer warp : TMA Q'_0, Q'_1 once; K'_j, V_j in 2-stage rings; G at the end
//   MMA warp      : S_0 = Q'_0 K'_0^T, S_1 = Q'_1 K'_0^T, then for each key tile
//                   j: O_0 += P_0 V_j, S_0 = Q'_0 K'_{j+1}^T, O_1 += P_1 V_j,
//                   S_1 = Q'_1 K'_{j+1}^T, so one warpgroup's softmax runs while
//                   the tensor core works for the other
//   2 x 4 softmax warps (thread = query row of its tile): row max, base-2
//                   exponentials, P as bf16 written back over its S columns,
//                   lazy rescaling of O in TMEM (only when a row's max grows
//                   by more than 2^8, decided warp-uniformly), final 1/l, gate
//                   and TMA store.
// TMEM (512 columns): S_0 [0,128) S_1 [128,256) O_0 [256,384) O_1 [384,512);
// P_i occupies the first 64 columns of S_i.
//
// Block-sparse form: with a tile list, the CTA walks only the `keep` key tiles
// listed for its 256-query block (in list order) instead of all of them; the
// softmax is exact over the keys of those tiles.
#include <cuda.h>

#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {
namespace {

constexpr int kD = 128;
constexpr int kRows = 128;
constexpr int kHalf = kRows * 64 * 2;  // 16 KB
constexpr int kTileB = 2 * kHalf;      // 32 KB
constexpr int kKS = 2;                 // K' stages
constexpr int kVS = 2;                 // V stages
constexpr int kThreads = 320;          // 8 softmax warps + producer + MMA
constexpr int kWarpProd = 8, kWarpMma = 9;
constexpr float kRescaleLog2 = 8.f;    // lazy rescale threshold (base-2 units)
// Of every 8 pairs of exponentials, this many run as a polynomial on the FMA
// pipe instead of the MUFU unit (16 results per clock per SM).
constexpr int kEmuPairs = 2;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- packed fp32 (f32x2) helpers: one instruction for two lanes of math
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
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the FMA pipe, for x <= 2^22 (x below -126 gives a value below
// 2^-126, i.e. nothing in bf16).  n = round(x) comes from adding 1.5 * 2^23
// (the low mantissa bits of the sum hold n), f = x - n lies in [-1/2, 1/2],
// 2^f is a cubic fitted here for this interval (max relative error 7.5e-5,
// far below bf16 rounding), and 2^n is applied by adding n to the exponent
// field: the constant's low nine bits are zero, so the shifted sum
// contributes exactly n << 23.
//
// Two at a time with packed f32x2 arithmetic, with the max subtraction folded
// in: for a row with reference max m, x = s - m; c = 1.5 * 2^23 - m gives
// t = s + c = round(x) + 1.5 * 2^23 and f = s - (t - c) = x - round(x).
// s_lo = m - 126 is the clamp; the exponent add is one integer multiply-add.
__device__ __forceinline__ void exp2_fma2(float s0, float s1, float s_lo, uint64_t c,
                                          float& y0, float& y1) {
  const uint64_t sv = pk2(fmaxf(s0, s_lo), fmaxf(s1, s_lo));
  const uint64_t t = add2(sv, c);
  const uint64_t f = sub2(sv, sub2(t, c));
  uint64_t p = fma2(pk2(0.055170517f, 0.055170517f), f, pk2(0.24260856f, 0.24260856f));
  p = fma2(p, f, pk2(0.69326097f, 0.69326097f));
  p = fma2(p, f, pk2(0.99992824f, 0.99992824f));
  float t0, t1, p0, p1;
  up2(t, t0, t1);
  up2(p, p0, p1);
  uint32_t r0, r1;
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(r0) : "r"(__float_as_uint(t0)), "r"(__float_as_uint(p0)));
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(r1) : "r"(__float_as_uint(t1)), "r"(__float_as_uint(p1)));
  y0 = __uint_as_float(r0);
  y1 = __uint_as_float(r1);
}

struct AnchorCtl {
  uint64_t q_full, g_full;
  uint64_t k_full[kKS], k_empty[kKS];
  uint64_t v_full[kVS], v_empty[kVS];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t ysync[2];  // the 128 output rows of tile i are staged (bounded wait)
  uint32_t tmem;
  int abort_flag;
};

// 320 threads = 10 warps: three share one of the four 16K-register slices of
// the SM, which caps a thread at 168 registers.
template <bool kGate, bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
    anchor_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                  const __grid_constant__ CUtensorMap tm_y, int N, const int* __restrict__ tiles,
                  int keep, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ AnchorCtl ctl;
  uint8_t* smem = align1024(smem_raw);
  uint8_t* q_s = smem;                 // Q'_0, Q'_1 (later: Y staging)
  uint8_t* k_s = q_s + 2 * kTileB;     // K' ring (later: G tiles)
  uint8_t* v_s = k_s + kKS * kTileB;   // V ring

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qp = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int row0 = qp * 2 * kRows;  // first query row of tile 0
  const int nkv = (N + kRows - 1) / kRows;
  const int kv_tail = N - (nkv - 1) * kRows;  // valid keys in the last tile
  // key tiles this CTA visits: all of them, or the `keep` listed for its block
  const int* list = kSparse ? tiles + ((size_t)(b * gridDim.y + h) * gridDim.x + qp) * keep : nullptr;
  const int nk_all = kSparse ? keep : nkv;
  auto key_tile = [&](int j) { return kSparse ? __ldg(list + j) : j; };
  const WaitCtx wc{&ctl.abort_flag, status};

  if (tid == 0) {
    mbar_init(&ctl.q_full, 1);
    mbar_init(&ctl.g_full, 1);
    for (int i = 0; i < kKS; ++i) {
      mbar_init(&ctl.k_full[i], 1);
      mbar_init(&ctl.k_empty[i], 1);
    }
    for (int i = 0; i < kVS; ++i) {
      mbar_init(&ctl.v_full[i], 1);
      mbar_init(&ctl.v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.s_full[i], 1);
      mbar_init(&ctl.p_full[i], 128);
      mbar_init(&ctl.pv_done[i], 1);
      mbar_init(&ctl.ysync[i], 128);
    }
    ctl.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;

  if (warp == kWarpProd) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(&ctl.q_full, 2 * kTileB);
      for (int i = 0; i < 2; ++i) {
        tma_load_3d(q_s + i * kTileB, &tm_q, &ctl.q_full, h * kD, row0 + i * kRows, b);
        tma_load_3d(q_s + i * kTileB + kHalf, &tm_q, &ctl.q_full, h * kD + 64, row0 + i * kRows, b);
      }
      int nk = 0, nv = 0;
      bool ok = true;
      for (int j = 0; j < nk_all; ++j) {
        const int sk = j % kKS, sv = j % kVS;
        const int row = key_tile(j) * kRows;  // first key of the tile
        if (j >= kKS && !mbar_wait(&ctl.k_empty[sk], ((j / kKS) - 1) & 1, wc, 0x31)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&ctl.k_full[sk], kTileB);
        tma_load_3d(k_s + sk * kTileB, &tm_k, &ctl.k_full[sk], h * kD, row, b);
        tma_load_3d(k_s + sk * kTileB + kHalf, &tm_k, &ctl.k_full[sk], h * kD + 64, row, b);
        ++nk;
        if (j >= kVS && !mbar_wait(&ctl.v_empty[sv], ((j / kVS) - 1) & 1, wc, 0x32)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&ctl.v_full[sv], kTileB);
        tma_load_3d(v_s + sv * kTileB, &tm_v, &ctl.v_full[sv], h * kD, row, b);
        tma_load_3d(v_s + sv * kTileB + kHalf, &tm_v, &ctl.v_full[sv], h * kD + 64, row, b);
        ++nv;
      }
      // G goes into the K ring once the last S MMAs have read it
      if (ok && kGate) {
        for (int j = (nk_all > kKS ? nk_all - kKS : 0); j < nk_all && ok; ++j)
          ok = mbar_wait(&ctl.k_empty[j % kKS], (j / kKS) & 1, wc, 0x3c);
        if (ok) {
          mbar_arrive_expect_tx(&ctl.g_full, 2 * kTileB);
          for (int i = 0; i < 2; ++i) {
            tma_load_3d(k_s + i * kTileB, &tm_g, &ctl.g_full, h * kD, row0 + i * kRows, b);
            tma_load_3d(k_s + i * kTileB + kHalf, &tm_g, &ctl.g_full, h * kD + 64,
                        row0 + i * kRows, b);
          }
        }
      }
      if (*wc.abort_flag) {  // loads still in flight land before the CTA exits
        mbar_drain(&ctl.q_full, 0);
        for (int j = nk > kKS ? nk - kKS : 0; j < nk; ++j)
          mbar_drain(&ctl.k_full[j % kKS], (j / kKS) & 1);
        for (int j = nv > kVS ? nv - kVS : 0; j < nv; ++j)
          mbar_drain(&ctl.v_full[j % kVS], (j / kVS) & 1);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      // S = Q' K'^T: A = Q' (K-major), B = K' tile (K-major: rows = keys).
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      // O += P V: A = P in TMEM (K-major), B = V tile (MN-major: d contiguous).
      const uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);
      // operand descriptors, built once; buffers and K steps advance the address
      const uint64_t dq0 = smem_desc_sw128(smem_u32(q_s), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_u32(k_s), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_u32(v_s), kHalf, 1024);
      auto issue_s = [&](int i, int j) {  // S_i = Q'_i K'_j^T
        const uint64_t a = desc_advance(dq0, i * kTileB);
        const uint64_t bk = desc_advance(dk0, (j % kKS) * kTileB);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_ss(tmem + i * 128, desc_advance(a, off), desc_advance(bk, off), idesc_s, kk != 0);
        }
        umma_commit(&ctl.s_full[i]);
      };
      auto issue_pv = [&](int i, int j) {  // O_i += P_i V_j
        const uint64_t bv = desc_advance(dv0, (j % kVS) * kTileB);
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          umma_ts(tmem + 256 + i * 128, tmem + i * 128 + kk * 8, desc_advance(bv, kk * 2048),
                  idesc_o, (j | kk) != 0);
        umma_commit(&ctl.pv_done[i]);
      };
      bool ok = mbar_wait(&ctl.q_full, 0, wc, 0x33) && nk_all > 0 &&
                mbar_wait(&ctl.k_full[0], 0, wc, 0x36);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        umma_commit(&ctl.k_empty[0]);  // K'_0 is read by these two only
      }
      for (int j = 0; ok && j < nk_all; ++j) {
        const bool more = j + 1 < nk_all;
        if (!mbar_wait(&ctl.v_full[j % kVS], (j / kVS) & 1, wc, 0x35)) break;
        if (more && !mbar_wait(&ctl.k_full[(j + 1) % kKS], ((j + 1) / kKS) & 1, wc, 0x36)) break;
        for (int i = 0; i < 2 && ok; ++i) {
          // P_i of tile j is in TMEM; O_i has been rescaled if needed
          if (!mbar_wait(&ctl.p_full[i], j & 1, wc, 0x34)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(i, j);
          if (more) {
            // S_i is overwritten only after the MMAs that read P_i from it finish
            if (!mbar_wait(&ctl.pv_done[i], j & 1, wc, 0x37)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(i, j + 1);
          }
        }
        if (!ok) break;
        umma_commit(&ctl.v_empty[j % kVS]);
        if (more) umma_commit(&ctl.k_empty[(j + 1) % kKS]);
      }
    }
  } else {
    // ------------------------------------------------ softmax warps: thread = query row
    const int qi = warp >> 2;                 // which query tile
    const int r = (warp & 3) * 32 + lane;     // row within the tile
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tmem_s = tmem + qi * 128, tmem_o = tmem + 256 + qi * 128;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < nk_all; ++j) {
      // warp-uniform outcome: tcgen05.ld / st are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl.s_full[qi], j & 1, wc, 0x38))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool last = key_tile(j) == nkv - 1 && kv_tail < kRows;
      // pass 1: row max, 64 columns in registers at a time (four independent
      // chains of 3-input max)
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t sa[32], sb[32];
        tmem_ld32(tmem_s + lane_base + hh * 64, sa);
        tmem_ld32(tmem_s + lane_base + hh * 64 + 32, sb);
        tmem_ld_wait();
        if (last) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (hh * 64 + i >= kv_tail) sa[i] = __float_as_uint(-INFINITY);
            if (hh * 64 + 32 + i >= kv_tail) sb[i] = __float_as_uint(-INFINITY);
          }
        }
#pragma unroll
        for (int i = 0; i < 32; i += 8)
#pragma unroll
          for (int a = 0; a < 4; ++a)
            mq[a] = max3(mq[a], __uint_as_float(sa[i + 2 * a]), __uint_as_float(sb[i + 2 * a + 1]));
#pragma unroll
        for (int i = 0; i < 32; i += 8)
#pragma unroll
          for (int a = 0; a < 4; ++a)
            mq[a] = max3(mq[a], __uint_as_float(sa[i + 2 * a + 1]), __uint_as_float(sb[i + 2 * a]));
      }
      const float mx = max3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
      const float m_new = fmaxf(m, mx);
      // lazy rescaling: a row moves its reference max only when the max grew
      // by more than 2^8; the decision to touch O is warp-uniform because TMEM
      // access is warp-collective (rows that keep their max use a factor 1).
      // A moved max is rounded up to an integer so that the folded constant of
      // the FMA-pipe exponential (1.5 * 2^23 - m) is exact.
      const bool grow = m_new > m + kRescaleLog2;
      const bool any_grow = __any_sync(0xffffffffu, grow);
      const float m_use = grow ? ceilf(m_new) : m;
      const float corr = ex2(m - m_use);  // 0 on the first tile
      // pass 2: P = 2^(s - m) over 32-column chunks, the next chunk's load in
      // flight while this one is exponentiated (MUFU for most pairs, the
      // FMA-pipe polynomial for kEmuPairs of every 8).  P of chunk c goes to
      // columns [16c, 16c + 16), inside S chunks already read.
      const uint64_t neg_m = pk2(-m_use, -m_use);
      const uint64_t cfold = pk2(12582912.f - m_use, 12582912.f - m_use);
      const float s_lo = m_use - 126.f;
      uint64_t rs2 = pk2(0.f, 0.f);
      uint32_t sc[2][32];
      uint32_t pk[32];
      tmem_ld32(tmem_s + lane_base, sc[0]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c < 3) tmem_ld32(tmem_s + lane_base + (c + 1) * 32, sc[(c + 1) & 1]);
        uint32_t* cur = sc[c & 1];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float s0 = __uint_as_float(cur[i]), s1 = __uint_as_float(cur[i + 1]);
          if (last) {
            if (c * 32 + i >= kv_tail) s0 = -INFINITY;
            if (c * 32 + i + 1 >= kv_tail) s1 = -INFINITY;
          }
          float p0, p1;
          if (((i >> 1) & 7) >= 8 - kEmuPairs) {
            exp2_fma2(s0, s1, s_lo, cfold, p0, p1);
          } else {
            float x0, x1;
            up2(add2(pk2(s0, s1), neg_m), x0, x1);
            p0 = ex2(x0);
            p1 = ex2(x1);
          }
          rs2 = add2(rs2, pk2(p0, p1));
          pk[(c & 1) * 16 + i / 2] = f2_to_bf2(p0, p1);
        }
        if (c & 1) tmem_st32(tmem_s + lane_base + (c >> 1) * 32, pk);
        if (c < 3) tmem_ld_wait();
      }
      float rs0, rs1;
      up2(rs2, rs0, rs1);
      l = l * corr + (rs0 + rs1);
      m = m_use;
      if (any_grow && j >= 1) {
        // O_i holds the sum over tiles < j (their PV MMAs finished before S_i
        // of this tile was issued); scale it before the next PV accumulates
        if (!__all_sync(0xffffffffu, mbar_wait(&ctl.pv_done[qi], (j - 1) & 1, wc, 0x39))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem_o + lane_base + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
          tmem_st32(tmem_o + lane_base + c * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctl.p_full[qi]);
    }
    // ---------------- epilogue: Y = O / l * sigmoid(G)
    ok = __all_sync(0xffffffffu,
                    ok && nk_all > 0 && mbar_wait(&ctl.pv_done[qi], (nk_all - 1) & 1, wc, 0x3a));
    if (kGate) ok = ok && __all_sync(0xffffffffu, mbar_wait(&ctl.g_full, 0, wc, 0x3d));
    uint8_t* ybuf = q_s + qi * kTileB;  // Q'_i is no longer read
    const uint8_t* gbuf = k_s + qi * kTileB;
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_base + c * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // 8 columns per 16-byte chunk
          const int ch = (c & 1) * 4 + q;
          const uint32_t off = (c >> 1) * kHalf + sw128_off(r, ch);
          uint32_t gw[4] = {0, 0, 0, 0};
          if (kGate) {
            const uint4 gr = *reinterpret_cast<const uint4*>(gbuf + off);
            gw[0] = gr.x; gw[1] = gr.y; gw[2] = gr.z; gw[3] = gr.w;
          }
          uint32_t out[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float y0 = __uint_as_float(o[q * 8 + 2 * i]) * inv;
            float y1 = __uint_as_float(o[q * 8 + 2 * i + 1]) * inv;
            if (kGate) {
              const float2 gg = bf2_to_f2(gw[i]);
              y0 *= sigmoid_fast(gg.x);
              y1 *= sigmoid_fast(gg.y);
            }
            out[i] = f2_to_bf2(y0, y1);
          }
          *reinterpret_cast<uint4*>(ybuf + off) = make_uint4(out[0], out[1], out[2], out[3]);
        }
      }
      fence_proxy_async_smem();
    }
    mbar_arrive(&ctl.ysync[qi]);
    ok = mbar_wait(&ctl.ysync[qi], 0, wc, 0x3b) && ok;
    if (ok && r == 0 && row0 + qi * kRows < N) {  // a tile past N has nothing to store
      tma_store_3d(&tm_y, ybuf, h * kD, row0 + qi * kRows, b);
      tma_store_3d(&tm_y, ybuf + kHalf, h * kD + 64, row0 + qi * kRows, b);
      bulk_commit();
      bulk_wait0();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    if (*wc.abort_flag) {  // MMAs in flight finish before TMEM is freed
      mbar_drain(&ctl.pv_done[0], (nk_all - 1) & 1);
      mbar_drain(&ctl.pv_done[1], (nk_all - 1) & 1);
    }
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

constexpr size_t kAnchorSmem = 1024 + 2 * kTileB + kKS * kTileB + kVS * kTileB;

}  // namespace

sana_status anchor_bf16_run(const sana_shape& s, const void* qr, const void* kr, const void* v,
                            const void* gt, const GridDev& g, const int* tiles, int keep,
                            void* out, cudaStream_t st) {
  const uint64_t C = (uint64_t)s.heads * kD, N = (uint64_t)g.N;
  CUtensorMap tq, tk, tv, tg, ty;
  bool okm = make_tmap_bf16_3d(&tq, qr, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&tk, kr, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&tv, v, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&ty, out, C, N, s.B, C, N * C, kRows);
  if (gt) okm = okm && make_tmap_bf16_3d(&tg, gt, C, N, s.B, C, N * C, kRows);
  else tg = tq;
  if (!okm) return fail(SANA_ERR_CUDA, "anchor: cuTensorMapEncodeTiled failed");
  once_per_context(kAttrAnchor, [] {
    const int bytes = (int)kAnchorSmem;
    cudaFuncSetAttribute(anchor_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    cudaFuncSetAttribute(anchor_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    cudaFuncSetAttribute(anchor_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    cudaFuncSetAttribute(anchor_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
  const int qtiles = (g.N + kRows - 1) / kRows;
  const dim3 grid((qtiles + 1) / 2, s.heads, s.B);
  int* sw = status_word();
  if (gt && tiles)
    anchor_kernel<true, true><<<grid, kThreads, kAnchorSmem, st>>>(tq, tk, tv, tg, ty, g.N, tiles, keep, sw);
  else if (gt)
    anchor_kernel<true, false><<<grid, kThreads, kAnchorSmem, st>>>(tq, tk, tv, tg, ty, g.N, nullptr, 0, sw);
  else if (tiles)
    anchor_kernel<false, true><<<grid, kThreads, kAnchorSmem, st>>>(tq, tk, tv, tg, ty, g.N, tiles, keep, sw);
  else
    anchor_kernel<false, false><<<grid, kThreads, kAnchorSmem, st>>>(tq, tk, tv, tg, ty, g.N, nullptr, 0, sw);
  return check_launch("anchor_kernel");
}

}  // namespace sana
