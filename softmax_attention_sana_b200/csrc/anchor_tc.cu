// Gated softmax anchor, bf16 on tcgen05 ("SANA-Video 2.0" abstract: gated
// softmax anchors every fourth layer; reading: the same 3D RoPE on Q and K,
// scale 1/sqrt(D)).
//
//   Y = sigmoid(G) * softmax(Q' K'^T) V   with Q' = RoPE(Q) * scale * log2(e),
//   K' = RoPE(K) prepared by a rotation pass, so the softmax works in base 2.
//
// One CTA per (batch, head, 128-query tile):
//   producer warp : TMA Q' and G once, then K' and V tiles (128 keys) in a ring
//   MMA warp      : S_b = Q' K'_j^T into TMEM buffer b = j % 2 (SS MMA), then
//                   O += P_{j-1} V_{j-1} with P read from TMEM (TS MMA)
//   4 softmax warps (thread = query row): online softmax over each S_b row,
//                   P written back as bf16 into the S_b columns, O rescaled
//                   in TMEM only when the running max grows by more than
//                   2^8 (values of P stay <= 256); the epilogue divides by
//                   the row sum, applies the gate and stores through TMA.
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
constexpr int kThreads = 192;          // 4 softmax warps + producer + MMA
constexpr float kRescaleLog2 = 8.f;    // lazy rescale threshold (base-2 units)

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct AnchorCtl {
  uint64_t q_full;
  uint64_t k_full[kKS], k_empty[kKS];
  uint64_t v_full[kVS], v_empty[kVS];
  uint64_t s_full[2], s_free[2], p_full[2];
  uint64_t pv_done;
  uint64_t ysync;  // the 128 output rows are staged (bounded wait)
  uint32_t tmem;
  int abort_flag;
};

template <bool kGate>
__global__ void __launch_bounds__(kThreads, 1)
    anchor_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                  const __grid_constant__ CUtensorMap tm_y, int N, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ AnchorCtl ctl;
  uint8_t* smem = align1024(smem_raw);
  uint8_t* q_s = smem;                 // Q' tile (later: Y staging when ungated)
  uint8_t* g_s = q_s + kTileB;         // G tile (Y staging when gated)
  uint8_t* k_s = g_s + kTileB;         // K' ring
  uint8_t* v_s = k_s + kKS * kTileB;   // V ring

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nkv = (N + kRows - 1) / kRows;
  const int kv_tail = N - (nkv - 1) * kRows;  // valid keys in the last tile
  const WaitCtx wc{&ctl.abort_flag, status};

  if (tid == 0) {
    mbar_init(&ctl.q_full, 1);
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
      mbar_init(&ctl.s_free[i], 1);
      mbar_init(&ctl.p_full[i], 128);
    }
    mbar_init(&ctl.pv_done, 1);
    mbar_init(&ctl.ysync, 128);
    ctl.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 5) {
    tmem_alloc(&ctl.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;          // S_0: cols [0,128), S_1: [128,256)
  const uint32_t tmem_o = tmem + 256;      // O: cols [256, 384)

  if (warp == 4) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(&ctl.q_full, kGate ? 2 * kTileB : kTileB);
      tma_load_3d(q_s, &tm_q, &ctl.q_full, h * kD, qt * kRows, b);
      tma_load_3d(q_s + kHalf, &tm_q, &ctl.q_full, h * kD + 64, qt * kRows, b);
      if (kGate) {
        tma_load_3d(g_s, &tm_g, &ctl.q_full, h * kD, qt * kRows, b);
        tma_load_3d(g_s + kHalf, &tm_g, &ctl.q_full, h * kD + 64, qt * kRows, b);
      }
      // K' and V rings advance together; a stage is refilled once the MMAs
      // that read it have completed.
      int nk = 0, nv = 0;
      for (int j = 0; j < nkv; ++j) {
        const int sk = j % kKS, sv = j % kVS;
        if (j >= kKS && !mbar_wait(&ctl.k_empty[sk], ((j / kKS) - 1) & 1, wc, 0x31)) break;
        mbar_arrive_expect_tx(&ctl.k_full[sk], kTileB);
        tma_load_3d(k_s + sk * kTileB, &tm_k, &ctl.k_full[sk], h * kD, j * kRows, b);
        tma_load_3d(k_s + sk * kTileB + kHalf, &tm_k, &ctl.k_full[sk], h * kD + 64, j * kRows, b);
        ++nk;
        if (j >= kVS && !mbar_wait(&ctl.v_empty[sv], ((j / kVS) - 1) & 1, wc, 0x32)) break;
        mbar_arrive_expect_tx(&ctl.v_full[sv], kTileB);
        tma_load_3d(v_s + sv * kTileB, &tm_v, &ctl.v_full[sv], h * kD, j * kRows, b);
        tma_load_3d(v_s + sv * kTileB + kHalf, &tm_v, &ctl.v_full[sv], h * kD + 64, j * kRows, b);
        ++nv;
      }
      if (*wc.abort_flag) {  // loads still in flight land before the CTA exits
        mbar_drain(&ctl.q_full, 0);
        for (int j = nk > kKS ? nk - kKS : 0; j < nk; ++j) mbar_drain(&ctl.k_full[j % kKS], (j / kKS) & 1);
        for (int j = nv > kVS ? nv - kVS : 0; j < nv; ++j) mbar_drain(&ctl.v_full[j % kVS], (j / kVS) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      // S = Q' K'^T: A = Q' (K-major), B = K' tile (K-major: rows = keys).
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      // O += P V: A = P in TMEM (K-major), B = V tile (MN-major: d contiguous).
      const uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t qb = smem_u32(q_s);
      bool ok = mbar_wait(&ctl.q_full, 0, wc, 0x33);
      auto issue_pv = [&](int j) -> bool {  // O += P_j V_j
        const int bb = j & 1, sv = j % kVS;
        if (!mbar_wait(&ctl.p_full[bb], (j >> 1) & 1, wc, 0x34)) return false;
        if (!mbar_wait(&ctl.v_full[sv], (j / kVS) & 1, wc, 0x35)) return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(v_s + sv * kTileB);
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          umma_ts(tmem_o, tmem + bb * 128 + kk * 8, smem_desc_sw128(vb + kk * 2048, kHalf, 1024),
                  idesc_o, (j | kk) != 0);
        umma_commit(&ctl.pv_done);
        umma_commit(&ctl.v_empty[sv]);
        umma_commit(&ctl.s_free[bb]);
        return true;
      };
      for (int j = 0; ok && j < nkv; ++j) {
        const int bb = j & 1, sk = j % kKS;
        if (!mbar_wait(&ctl.k_full[sk], (j / kKS) & 1, wc, 0x36)) break;
        if (j >= 2 && !mbar_wait(&ctl.s_free[bb], ((j >> 1) - 1) & 1, wc, 0x37)) break;
        tc_fence_after();
        const uint32_t kb = smem_u32(k_s + sk * kTileB);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_ss(tmem + bb * 128, smem_desc_sw128(qb + off, 16, 1024),
                  smem_desc_sw128(kb + off, 16, 1024), idesc_s, kk != 0);
        }
        umma_commit(&ctl.s_full[bb]);
        umma_commit(&ctl.k_empty[sk]);
        if (j >= 1 && !issue_pv(j - 1)) ok = false;
      }
      if (ok && nkv > 0) issue_pv(nkv - 1);
    }
  } else {
    // ------------------------------------------------ softmax warps: thread = query row
    const int r = warp * 32 + lane;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < nkv; ++j) {
      const int bb = j & 1;
      // warp-uniform outcome: tcgen05.ld / st are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl.s_full[bb], (j >> 1) & 1, wc, 0x38))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + bb * 128 + c * 32, sr[c]);
      tmem_ld_wait();
      const int valid = (j == nkv - 1) ? kv_tail : kRows;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float s = __uint_as_float(sr[c][i]);
          if (c * 32 + i >= valid) s = -INFINITY;
          sr[c][i] = __float_as_uint(s);
          mx = fmaxf(mx, s);
        }
      const float m_new = fmaxf(m, mx);
      // rescale O when any row of the warp needs it (collective TMEM access)
      const bool grow = m_new > m + kRescaleLog2;
      if (__any_sync(0xffffffffu, grow)) {
        const float m_use = grow ? m_new : m;
        const float corr = ex2(m - m_use);  // 0 on the first tile, 1 for rows that keep m
        if (j >= 1) {
          // O holds the sum over tiles < j; wait for the last PV before touching it
          if (!__all_sync(0xffffffffu, mbar_wait(&ctl.pv_done, (j - 1) & 1, wc, 0x39))) {
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
          tmem_st_wait();
        }
        l *= corr;
        m = m_use;
      }
      float rs = 0.f;
      uint32_t pk[2][32];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = ex2(__uint_as_float(sr[c][i]) - m);
          const float p1 = ex2(__uint_as_float(sr[c][i + 1]) - m);
          rs += p0 + p1;
          pk[c >> 1][(c & 1) * 16 + i / 2] = f2_to_bf2(p0, p1);
        }
      l += rs;
      tmem_st32(tmem + lane_base + bb * 128, pk[0]);
      tmem_st32(tmem + lane_base + bb * 128 + 32, pk[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctl.p_full[bb]);
    }
    // ---------------- epilogue: Y = O / l * sigmoid(G)
    ok = __all_sync(0xffffffffu, ok && nkv > 0 && mbar_wait(&ctl.pv_done, (nkv - 1) & 1, wc, 0x3a));
    uint8_t* ybuf = kGate ? g_s : q_s;
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_base + c * 32, o);
        tmem_ld_wait();
        uint8_t* hb = ybuf + (c >> 1) * kHalf;
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // 8 columns per 16-byte chunk
          const int ch = (c & 1) * 4 + q;
          uint4* p = reinterpret_cast<uint4*>(hb + sw128_off(r, ch));
          uint32_t gw[4] = {0, 0, 0, 0};
          if (kGate) {
            const uint4 gr = *p;
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
          *p = make_uint4(out[0], out[1], out[2], out[3]);
        }
      }
      fence_proxy_async_smem();
    }
    mbar_arrive(&ctl.ysync);
    ok = mbar_wait(&ctl.ysync, 0, wc, 0x3b) && ok;
    if (ok && tid == 0) {
      tma_store_3d(&tm_y, ybuf, h * kD, qt * kRows, b);
      tma_store_3d(&tm_y, ybuf + kHalf, h * kD + 64, qt * kRows, b);
      bulk_commit();
      bulk_wait0();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    if (*wc.abort_flag) mbar_drain(&ctl.pv_done, (nkv - 1) & 1);
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

constexpr size_t kAnchorSmem = 1024 + 2 * kTileB + kKS * kTileB + kVS * kTileB;

}  // namespace

sana_status anchor_bf16_run(const sana_shape& s, const void* qr, const void* kr, const void* v,
                            const void* gt, const GridDev& g, void* out, cudaStream_t st) {
  const uint64_t C = (uint64_t)s.heads * kD, N = (uint64_t)g.N;
  CUtensorMap tq, tk, tv, tg, ty;
  bool okm = make_tmap_bf16_3d(&tq, qr, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&tk, kr, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&tv, v, C, N, s.B, C, N * C, kRows) &&
             make_tmap_bf16_3d(&ty, out, C, N, s.B, C, N * C, kRows);
  if (gt) okm = okm && make_tmap_bf16_3d(&tg, gt, C, N, s.B, C, N * C, kRows);
  else tg = tq;
  if (!okm) return fail(SANA_ERR_CUDA, "anchor: cuTensorMapEncodeTiled failed");
  static bool attr[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr[dev]) {
    cudaFuncSetAttribute(anchor_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kAnchorSmem);
    cudaFuncSetAttribute(anchor_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kAnchorSmem);
    attr[dev] = true;
  }
  const dim3 grid((g.N + kRows - 1) / kRows, s.heads, s.B);
  if (gt)
    anchor_kernel<true><<<grid, kThreads, kAnchorSmem, st>>>(tq, tk, tv, tg, ty, g.N, status_word());
  else
    anchor_kernel<false><<<grid, kThreads, kAnchorSmem, st>>>(tq, tk, tv, tg, ty, g.N, status_word());
  return check_launch("anchor_kernel");
}

}  // namespace sana
