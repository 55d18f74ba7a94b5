// MX block-scaled projection GEMM ("SANA-Video 2.0" hyper.ai summary,
// Experiments: low-precision inference quantises only the linear GEMM
// layers, weights to MXFP4 and activations to MXFP8; attention stays bf16).
//
//   y[M][N] = Q8(x)[M][K] . Q4(w)[N][K]^T,  fp32 accumulation, bf16 out.
//
// The formats are the OCP Microscaling v1.0 ones: blocks of 32 elements
// along K share one E8M0 scale 2^s with s = floor(log2 max|x|) - emax of the
// element format (8 for E4M3, 2 for E2M1), clamped to [-127, 127] (an
// all-zero block takes -127); each element is x / 2^s rounded to nearest
// even and saturated (cvt.rn.satfinite).
//
// Storage (what the quantisers write and the GEMM reads):
//   * E4M3 elements: one byte each, row-major [rows][K].
//   * E2M1 elements: two per byte, element 2i in the low nibble, row-major
//     [rows][K/2].
//   * scales: E8M0 bytes (s + 127) in 512-byte atoms, one per 128 rows x 128
//     K-elements (4 blocks), atoms ordered [rows/128][K/128]; inside an atom
//     row r, block b sits at byte 16 (r % 32) + 4 (r / 32) + b.  This is the
//     layout tcgen05.cp.32x128b.warpx4 copies to TMEM so that each row's four
//     block scales form one 32-bit TMEM word.
//
// GEMM: persistent, 128 x 256 output tiles (128 x 128 when N is not a
// multiple of 256); a TMA producer warp fills a ring of stages of (A 128 x 128
// E4M3, B BN x 128 E2M1 unpacked to the 8-bit shared-memory footprint by the
// 16U4_ALIGN16B tensor map, the scale atoms by bulk copy); one thread copies
// the scale atoms to TMEM and issues tcgen05.mma kind::mxf8f6f4 (block scale
// 1X, K = 32 per instruction); epilogue warps drain the accumulator (the
// 128-wide form keeps two, so its epilogue overlaps the next tile).
#include <cuda.h>

#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {
namespace {

constexpr int BM = 128, BK = 128;  // BK in elements
constexpr int kABytes = BM * BK;   // E4M3: 16 KB
constexpr int kSFBytes = 512;      // one scale atom
constexpr int kSfCol = 256;        // TMEM column of the scale slots (after the accumulators)

// Two tile widths.  BN = 256 (N a multiple of 256) doubles the work of every
// block-scaled MMA instruction; its 256-column accumulator leaves no room for
// a second one next to the scale slots, so eight epilogue warps drain it.
// BN = 128 keeps two accumulators (the epilogue overlaps the next tile).
template <int BN>
struct MxCfg {
  static constexpr int kStages = BN == 128 ? 6 : 4;
  static constexpr int kAccBufs = BN == 128 ? 2 : 1;
  static constexpr int kEpiWarps = BN / 32;                   // lane quarter x 128 columns
  static constexpr int kThreads = 64 + 32 * kEpiWarps;        // producer, MMA, epilogue
  static constexpr int kBBytes = BN * BK;                     // E2M1 in the 8-bit footprint
  static constexpr int kSFB = BN / 128 * kSFBytes;            // scale atoms of the B tile
  static constexpr int kStageBytes = kABytes + kBBytes + kSFBytes + kSFB;
  // bytes the stage's copies deliver: B arrives as packed nibbles
  static constexpr uint32_t kStageTx = kABytes + BN * BK / 2 + kSFBytes + kSFB;
  static constexpr int kSlotCols = 16;                        // A: 4 columns, B: 4 per atom
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// ---------------------------------------------------------------- quantisers
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Byte offset of (row, 32-element block) in the scale-atom layout.
__device__ __forceinline__ size_t sf_offset(long long row, int blk, int K) {
  const size_t atom = (size_t)(row >> 7) * (size_t)(K >> 7) + (size_t)(blk >> 2);
  return atom * 512 + 16 * (row & 31) + 4 * ((row >> 5) & 3) + (blk & 3);
}

// One thread per 32-element block: max |x|, the block exponent, 32 element
// codes and one scale byte.  Rows in [rows, rows_pad) only get a zero scale
// byte (their elements are never read: the GEMM's row tiles past M are
// zero-filled by TMA).
template <bool kFp4>
__global__ void __launch_bounds__(256)
    mx_quant_kernel(const __nv_bfloat16* __restrict__ x, long long rows, long long rows_pad, int K,
                    uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  const int nblk = K >> 5;
  const long long total = rows_pad * nblk;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / nblk;
    const int blk = (int)(i - row * nblk);
    if (row >= rows) {
      sf[sf_offset(row, blk, K)] = 0;
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + row * K + blk * 32);
    uint32_t w[16];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = src[c];
      w[4 * c] = v.x;
      w[4 * c + 1] = v.y;
      w[4 * c + 2] = v.z;
      w[4 * c + 3] = v.w;
    }
    // max |x| on the magnitude bits of both bf16 halves (order-preserving)
    uint32_t amax = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      amax = max(amax, w[k] & 0x7FFFu);
      amax = max(amax, (w[k] >> 16) & 0x7FFFu);
    }
    const int e = (int)(amax >> 7);          // biased exponent of max |x|
    const int emax = kFp4 ? 2 : 8;
    int s = e == 0 ? -127 : e - 127 - emax;  // zero or subnormal max: smallest scale
    s = s < -127 ? -127 : (s > 127 ? 127 : s);
    const float mul = __uint_as_float((uint32_t)(127 - s) << 23);  // 2^-s, s <= 125 here
    if (kFp4) {
      uint32_t packed[4] = {0, 0, 0, 0};
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float2 f = bf2_to_f2(w[k]);
        packed[k >> 2] |= cvt_e2m1x2(f.x * mul, f.y * mul) << (8 * (k & 3));
      }
      *reinterpret_cast<uint4*>(q + row * (K / 2) + blk * 16) =
          make_uint4(packed[0], packed[1], packed[2], packed[3]);
    } else {
      uint32_t packed[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float2 a = bf2_to_f2(w[2 * k]), b = bf2_to_f2(w[2 * k + 1]);
        packed[k] = cvt_e4m3x2(a.x * mul, a.y * mul) | (cvt_e4m3x2(b.x * mul, b.y * mul) << 16);
      }
      uint4* dst = reinterpret_cast<uint4*>(q + row * K + blk * 32);
      dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    }
    sf[sf_offset(row, blk, K)] = (uint8_t)(s + 127);
  }
}

// ---------------------------------------------------------------- GEMM
// Instruction descriptor of tcgen05.mma kind::mxf8f6f4: A E4M3, B E2M1, both
// K-major, E8M0 scales, dense, K = 32; the scale-factor ids pick the byte
// (the 32-element block) inside each row's 32-bit TMEM word.
__host__ __device__ constexpr uint32_t idesc_mxf8f6f4(int M, int N, int sf_id) {
  return ((uint32_t)sf_id << 4)        // B scale-factor id
         | (0u << 7)                   // A format: E4M3
         | (5u << 10)                  // B format: E2M1
         | ((uint32_t)(N >> 3) << 17)  // N / 8
         | (1u << 23)                  // scale format: E8M0
         | ((uint32_t)(M >> 4) << 24)  // M / 16
         | ((uint32_t)sf_id << 29);    // A scale-factor id
}

// D[tmem] (+)= (A[smem] * 2^sfa) (B[smem] * 2^sfb)
__device__ __forceinline__ void umma_mx(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Shared-memory descriptor of a 512-byte scale atom as the source of
// tcgen05.cp.32x128b: no swizzle, K-major, 32 rows of 16 bytes, eight-row
// groups 128 bytes apart.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;            // leading byte offset: 16 B (one core matrix wide)
  d |= (uint64_t)(128 >> 4) << 32;   // stride byte offset: 128 B
  d |= (uint64_t)1 << 46;            // descriptor version for sm_100
  return d;                          // layout type 0: no swizzle
}
// 32 lanes x 128 bits from shared memory into TMEM, broadcast to the four
// lane quarters (each row's word lands in every quarter).
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}
// Untiled bulk copy global -> shared (both 16-byte aligned, size multiple of 16).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Output columns, optionally split into equal parts written to separate
// tensors (the Q, K, V, G projection).
struct MxOut {
  __nv_bfloat16* part[4];
  int part_cols;  // columns per part (== N when not split), a multiple of BN
  long long ldo;  // row stride of each part in elements
};

struct MxCtl {
  uint64_t full[6], empty[6];
  uint64_t tfull[2], tempty[2];
  uint64_t drain;  // teardown after an abort: all issued tcgen05 ops finished
  uint32_t tmem;
  int abort_flag;
};

template <int BN>
__global__ void __launch_bounds__(MxCfg<BN>::kThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb, long long M,
                   int N, int K, MxOut out, int epilogue, int* status) {
  using Cfg = MxCfg<BN>;
  constexpr int kStages = Cfg::kStages, kAccBufs = Cfg::kAccBufs;
  constexpr int kBBytes = Cfg::kBBytes, kStageBytes = Cfg::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  __shared__ MxCtl ctl;
  uint8_t* smem = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tiles_n = N / BN;
  const long long tiles_m = (M + BM - 1) / BM;
  const long long ntiles = tiles_m * tiles_n;
  const int kblocks = K / BK;
  const WaitCtx wc{&ctl.abort_flag, status};

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(&ctl.tfull[i], 1);
      mbar_init(&ctl.tempty[i], 32 * Cfg::kEpiWarps);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      long long it = 0;
      bool ok = true;
      for (long long t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
        const long long mt = t / tiles_n;
        const int nt = (int)(t % tiles_n);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = (int)(it % kStages);
          if (it >= kStages &&
              !mbar_wait(&ctl.empty[s], (uint32_t)((it / kStages) - 1) & 1, wc, 0x51)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&ctl.full[s], Cfg::kStageTx);
          tma_load_2d(st, &tm_a, &ctl.full[s], kb * BK, (int)(mt * BM));
          tma_load_2d(st + kABytes, &tm_b, &ctl.full[s], kb * BK, nt * BN);
          bulk_load(st + kABytes + kBBytes, sfa + ((size_t)mt * kblocks + kb) * kSFBytes, kSFBytes,
                    &ctl.full[s]);
#pragma unroll
          for (int a = 0; a < BN / 128; ++a)  // B's scale atoms: 128 rows each
            bulk_load(st + kABytes + kBBytes + (1 + a) * kSFBytes,
                      sfb + ((size_t)(nt * (BN / 128) + a) * kblocks + kb) * kSFBytes, kSFBytes,
                      &ctl.full[s]);
        }
      }
      if (!ok)  // loads in flight land before the CTA exits
        for (long long j = it > kStages ? it - kStages : 0; j < it; ++j)
          mbar_drain(&ctl.full[j % kStages], (uint32_t)(j / kStages) & 1);
    }
  } else if (warp == 1) {
    // ---------------- scale copies and MMA issue
    if (lane == 0) {
      const uint64_t da0 = smem_desc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t db0 = smem_desc_sw128(smem_u32(smem + kABytes), 16, 1024);
      const uint64_t dsf0 = sf_atom_desc(smem_u32(smem + kABytes + kBBytes));
      long long it = 0;
      int local = 0;
      bool ok = true;
      for (long long t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++local) {
        const int tb = local % kAccBufs;
        if (local >= kAccBufs &&
            !mbar_wait(&ctl.tempty[tb], ((local / kAccBufs) - 1) & 1, wc, 0x52))
          break;
        tc_fence_after();
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = (int)(it % kStages);
          if (!mbar_wait(&ctl.full[s], (uint32_t)(it / kStages) & 1, wc, 0x53)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // four scale slots (A: 4 columns, B: 4 per atom), rotated per K-block
          const uint32_t slot = tmem + kSfCol + (uint32_t)(it & 3) * Cfg::kSlotCols;
#pragma unroll
          for (int a = 0; a <= BN / 128; ++a)
            tmem_cp_sf(slot + 4 * a, desc_advance(dsf0, s * kStageBytes + a * kSFBytes));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // the scale-factor id (byte of the TMEM word) is also carried in
            // the top two bits of the scale address
            const uint32_t sel = (uint32_t)kk << 30;
            umma_mx(tmem + tb * BN, desc_advance(da0, s * kStageBytes + kk * 32),
                    desc_advance(db0, s * kStageBytes + kk * 32), idesc_mxf8f6f4(BM, BN, kk),
                    slot | sel, (slot + 4) | sel, (kb | kk) != 0);
          }
          umma_commit(&ctl.empty[s]);
        }
        if (ok) umma_commit(&ctl.tfull[tb]);
      }
    }
  } else {
    // ---------------- epilogue warps: TMEM lane quarter = warp % 4, and
    // 128 columns per warp of the same quarter
    const int q4 = warp & 3, r = q4 * 32 + lane;
    const int cbase = ((warp - 2) >> 2) * 128;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    int local = 0;
    for (long long t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
      const int tb = local % kAccBufs;
      const bool okw = __all_sync(
          0xffffffffu, mbar_wait(&ctl.tfull[tb], (local / kAccBufs) & 1, wc, 0x54));
      tc_fence_after();
      const long long row = (t / tiles_n) * BM + r;
      const int nt0 = (int)(t % tiles_n) * BN;
      const int part = nt0 / out.part_cols;
      __nv_bfloat16* orow = out.part[part] + row * out.ldo + (nt0 - part * out.part_cols) + cbase;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        if (okw) tmem_ld32(tmem + lane_base + tb * BN + cbase + c * 32, v);
        tmem_ld_wait();
        if (!okw || row >= M) continue;
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float f[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(v[q * 8 + i]);
          if (epilogue == 1) {
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] *= sigmoid_fast(f[i]);
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
      mbar_arrive(&ctl.tempty[tb]);
      if (!okw) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*wc.abort_flag) {  // MMAs and scale copies in flight finish before TMEM is freed
      if (lane == 0) umma_commit(&ctl.drain);
      __syncwarp();
      mbar_drain(&ctl.drain, 0);
    }
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

size_t mx_scale_bytes(long long rows, int K) {
  return (size_t)((rows + 127) / 128) * (size_t)(K / 128) * 512;
}

sana_status mx_quantize_run(const void* x, long long rows, int K, bool fp4, void* q, void* sf,
                            cudaStream_t st) {
  if (rows == 0) return SANA_OK;
  const long long rows_pad = (rows + 127) / 128 * 128;
  const long long total = rows_pad * (K / 32);
  long long blocks = (total + 255) / 256;
  if (blocks > 16 * kNumSMs) blocks = 16 * kNumSMs;
  if (fp4)
    mx_quant_kernel<true><<<(unsigned)blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), rows, rows_pad, K, static_cast<uint8_t*>(q),
        static_cast<uint8_t*>(sf));
  else
    mx_quant_kernel<false><<<(unsigned)blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), rows, rows_pad, K, static_cast<uint8_t*>(q),
        static_cast<uint8_t*>(sf));
  return check_launch("mx_quant_kernel");
}

template <int BN>
sana_status mx_gemm_launch(long long M, int N, int K, const void* xq, const void* xsf,
                           const void* wq, const void* wsf, const MxOut& out, int epilogue,
                           cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!make_tmap_2d_typed(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)K, (uint64_t)M,
                          (uint64_t)K, BK, BM) ||
      !make_tmap_2d_typed(&tb, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, wq, (uint64_t)K, (uint64_t)N,
                          (uint64_t)K / 2, BK, BN))
    return fail(SANA_ERR_CUDA, "mx gemm: cuTensorMapEncodeTiled failed");
  once_per_context(BN == 256 ? kAttrMx256 : kAttrMx128, [] {
    cudaFuncSetAttribute(mx_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)MxCfg<BN>::kSmem);
  });
  const long long tiles = ((M + BM - 1) / BM) * (N / BN);
  const int grid = (int)(tiles < kNumSMs ? tiles : kNumSMs);
  mx_gemm_kernel<BN><<<grid, MxCfg<BN>::kThreads, MxCfg<BN>::kSmem, st>>>(
      ta, tb, static_cast<const uint8_t*>(xsf), static_cast<const uint8_t*>(wsf), M, N, K, out,
      epilogue, status_word());
  return check_launch("mx_gemm_kernel");
}

sana_status mx_gemm_run_parts(long long M, int N, int K, const void* xq, const void* xsf,
                              const void* wq, const void* wsf, void* const* outs, int nparts,
                              long long ldo, int epilogue, cudaStream_t st) {
  if (M == 0) return SANA_OK;
  if (nparts < 1 || nparts > 4 || N % nparts != 0)
    return fail(SANA_ERR_UNSUPPORTED, "mx gemm: bad output split");
  MxOut o{};
  for (int i = 0; i < nparts; ++i) o.part[i] = static_cast<__nv_bfloat16*>(outs[i]);
  o.part_cols = N / nparts;
  o.ldo = ldo;
  // the 256-wide tile when every part is a whole number of them
  if (N % 256 == 0 && o.part_cols % 256 == 0)
    return mx_gemm_launch<256>(M, N, K, xq, xsf, wq, wsf, o, epilogue, st);
  if (o.part_cols % 128 != 0) return fail(SANA_ERR_UNSUPPORTED, "mx gemm: bad output split");
  return mx_gemm_launch<128>(M, N, K, xq, xsf, wq, wsf, o, epilogue, st);
}

sana_status mx_gemm_run(long long M, int N, int K, const void* xq, const void* xsf,
                        const void* wq, const void* wsf, void* out, long long ldo, int epilogue,
                        cudaStream_t st) {
  void* outs[1] = {out};
  return mx_gemm_run_parts(M, N, K, xq, xsf, wq, wsf, outs, 1, ldo, epilogue, st);
}

}  // namespace sana
