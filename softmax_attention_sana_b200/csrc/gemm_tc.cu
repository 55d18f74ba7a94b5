// bf16 GEMM on tcgen05 for the stack's projections:
//   out[M][N] = epilogue(A[M][K] . W[N][K]^T), fp32 accumulation in TMEM.
// Persistent: one CTA per SM walks 128 x 256 output tiles; a TMA producer
// warp fills a 4-stage ring of (A 128x64, W 256x64) K-blocks, one thread
// issues the MMAs into one of two TMEM accumulators, and four epilogue warps
// drain the other accumulator (identity, SiLU, or residual add) while the
// next tile's mainloop runs.  The output columns may be split into equal
// parts written to separate tensors (the Q, K, V, G projection).
#include <cuda.h>

#include "pair.cuh"
#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {
namespace {

constexpr int BM = 256, BN = 256, BK = 64;  // tile of a CTA pair
constexpr int kRowsCta = BM / 2;              // A rows (and B rows) one CTA holds
constexpr int kStages = 6;
constexpr int kABytes = kRowsCta * BK * 2;    // 16 KB
constexpr int kBBytes = (BN / 2) * BK * 2;    // 16 KB: this CTA's half of W's rows
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;  // producer, MMA, 4 epilogue warps

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

struct GemmOut {
  __nv_bfloat16* part[4];
  int part_cols;  // columns per part (== N when not split)
  long long ldo;  // row stride of each part in elements
};

struct GemmCtl {
  uint64_t full[kStages], empty[kStages];
  uint64_t tfull[2], tempty[2];
  uint64_t mma_end;
  uint32_t tmem;
  int abort_flag;
};

// A cluster of two CTAs walks 256 x 256 output tiles: each CTA loads its 128
// rows of A and its 128 of the tile's 256 W rows; the leader (rank 0) issues
// M = 256, N = 256 MMAs over both, and each CTA's epilogue drains its own 128
// accumulator rows.  Per MMA clock each CTA reads half the W bytes of a
// one-CTA 128 x 256 tile.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                long long M, int N, int K, GemmOut out, int epilogue, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ GemmCtl ctl;
  uint8_t* smem = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int tiles_n = (N + BN - 1) / BN;
  const long long tiles_m = (M + BM - 1) / BM;
  const long long ntiles = tiles_m * tiles_n;
  const int kblocks = K / BK;
  const WaitCtx wc{&ctl.abort_flag, status};

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.tfull[i], 1);
      mbar_init(&ctl.tempty[i], 8);  // one arrival per epilogue warp of the pair
    }
    mbar_init(&ctl.mma_end, 1);
    ctl.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&ctl.tmem, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any arrival crosses over
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs; bytes counted on the leader's barriers)
    if (lane == 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      long long it = 0;
      bool ok = true;
      for (long long t = pair; ok && t < ntiles; t += npairs) {
        const int m0 = (int)(t / tiles_n) * BM + (int)rank * kRowsCta;
        const int n0 = (int)(t % tiles_n) * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = (int)(it % kStages);
          if (it >= kStages &&
              !mbar_wait(&ctl.empty[s], (uint32_t)((it / kStages) - 1) & 1, wc, 0x41)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          if (rank == 0) mbar_arrive_expect_tx(&ctl.full[s], 2 * kStageBytes);
          const uint32_t lf = cluster_addr(&ctl.full[s], 0);
          tma_load_2d_pair(st, &tm_a, lf, kb * BK, m0);
          tma_load_2d_pair(st + kABytes, &tm_b, lf, kb * BK, n0);
        }
      }
      // the last stages' release arrivals land here before the CTA may exit
      for (long long j = it > kStages ? it - kStages : 0; ok && j < it; ++j)
        ok = mbar_wait(&ctl.empty[j % kStages], (uint32_t)(j / kStages) & 1, wc, 0x45);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
      // built once; stages and K steps advance the start address
      const uint64_t da0 = smem_desc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t db0 = smem_desc_sw128(smem_u32(smem + kABytes), 16, 1024);
      long long it = 0;
      int local = 0;
      bool ok = true;
      for (long long t = pair; ok && t < ntiles; t += npairs, ++local) {
        const int tb = local & 1;
        if (local >= 2 &&
            !mbar_wait_cluster(&ctl.tempty[tb], ((local >> 1) - 1) & 1, wc, 0x42))
          break;
        tc_fence_after();
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = (int)(it % kStages);
          if (!mbar_wait_cluster(&ctl.full[s], (uint32_t)(it / kStages) & 1, wc, 0x43)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_ss_pair(tmem + tb * BN, desc_advance(da0, s * kStageBytes + kk * 32),
                         desc_advance(db0, s * kStageBytes + kk * 32), idesc, (kb | kk) != 0);
          umma_commit_pair_both(&ctl.empty[s]);
        }
        if (ok) umma_commit_pair_both(&ctl.tfull[tb]);
      }
      umma_commit_pair_self(&ctl.mma_end);
      mbar_drain(&ctl.mma_end, 0);  // nothing of the pair's MMAs is in flight past here
    }
  } else {
    // ---------------- epilogue warps 2..5 (both CTAs): TMEM lane quarter = warp % 4
    const int q4 = warp & 3, r = q4 * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t leader_tempty[2] = {cluster_addr(&ctl.tempty[0], 0),
                                       cluster_addr(&ctl.tempty[1], 0)};
    int local = 0;
    for (long long t = pair; t < ntiles; t += npairs, ++local) {
      const int tb = local & 1;
      // warp-uniform: tcgen05.ld is a warp-collective instruction
      const bool okw = __all_sync(0xffffffffu, mbar_wait(&ctl.tfull[tb], (local >> 1) & 1, wc, 0x44));
      tc_fence_after();
      const long long row = (t / tiles_n) * BM + rank * kRowsCta + r;
      const int n0 = (int)(t % tiles_n) * BN;
      const int part = n0 / out.part_cols;
      const int pc0 = n0 - part * out.part_cols;
      __nv_bfloat16* orow = out.part[part] + row * out.ldo + pc0;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        if (okw) tmem_ld32(tmem + lane_base + tb * BN + c * 32, v);
        tmem_ld_wait();
        if (!okw || row >= M) continue;
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (n0 + c * 32 + q * 8 >= N) break;  // N is a multiple of 16
          float f[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(v[q * 8 + i]);
          if (epilogue == 1) {
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = f[i] / (1.f + __expf(-f[i]));
          } else if (epilogue == 2) {
            const uint4 old = dst[q];
            const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 o2 = bf2_to_f2(ow[i]);
              f[2 * i] += o2.x;
              f[2 * i + 1] += o2.y;
            }
          }
          dst[q] = make_uint4(f2_to_bf2(f[0], f[1]), f2_to_bf2(f[2], f[3]), f2_to_bf2(f[4], f[5]),
                              f2_to_bf2(f[6], f[7]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tempty[tb]);
      if (!okw) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the pair's MMAs or arrivals may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

constexpr size_t kGemmSmem = 1024 + kStages * kStageBytes;

}  // namespace

// out may be split column-wise into `nparts` tensors of N / nparts columns each
// (each a multiple of 256); otherwise nparts = 1 and ldo is its row stride.
sana_status gemm_run_parts(long long M, int N, int K, const void* A, long long lda, const void* W,
                           void* const* outs, int nparts, long long ldo, int epilogue,
                           cudaStream_t st) {
  if (M == 0) return SANA_OK;
  if (K % BK != 0 || N % 16 != 0)
    return fail(SANA_ERR_UNSUPPORTED, "gemm: K=%d must be a multiple of 64 and N=%d of 16", K, N);
  if (nparts < 1 || nparts > 4 || N % nparts != 0 || (nparts > 1 && (N / nparts) % BN != 0))
    return fail(SANA_ERR_UNSUPPORTED, "gemm: bad output split");
  CUtensorMap ta, tb;
  if (!make_tmap_bf16_2d(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda, BK, kRowsCta) ||
      !make_tmap_bf16_2d(&tb, W, (uint64_t)K, (uint64_t)N, (uint64_t)K, BK, BN / 2))
    return fail(SANA_ERR_CUDA, "gemm: cuTensorMapEncodeTiled failed");
  GemmOut o{};
  for (int i = 0; i < nparts; ++i) o.part[i] = static_cast<__nv_bfloat16*>(outs[i]);
  o.part_cols = N / nparts;
  o.ldo = ldo;
  once_per_context(kAttrGemm, [] {
    cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
  });
  const long long tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int pairs = (int)(tiles < kNumSMs / 2 ? tiles : kNumSMs / 2);
  gemm_kernel<<<2 * pairs, kThreads, kGemmSmem, st>>>(ta, tb, M, N, K, o, epilogue, status_word());
  return check_launch("gemm_kernel");
}

sana_status gemm_run(long long M, int N, int K, const void* A, long long lda, const void* W,
                     void* out, long long ldo, int epilogue, cudaStream_t st) {
  void* outs[1] = {out};
  return gemm_run_parts(M, N, K, A, lda, W, outs, 1, ldo, epilogue, st);
}

}  // namespace sana
