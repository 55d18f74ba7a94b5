// Tile selection of the block-sparse softmax anchor.
//
// "SANA-Video 2.0" (Experiments, Sol-Engine figures; abstract) applies sparse
// attention to the softmax anchors without giving the pattern.  Reading:
// queries in blocks of 256 tokens (one anchor CTA), keys in tiles of 128; each
// block keeps the `keep` key tiles with the largest pooled logit
//   score(block, tile) = mean(Q') . mean(K')
// over the block's / tile's tokens (Q', K' the rotated, scaled operands the
// anchor kernel reads, so this equals the mean logit of the block pair), ties
// going to the lower tile index; the kept indices are written in ascending
// order so that the anchor kernels of one head stream K and V in the same
// direction.
//
//   tile_sums_kernel    per 128-token tile: fixed-order column sums of Q' / K'
//   block_select_kernel per (batch, head, group of query blocks): scores by
//                       warp-cooperative dot products, then per block a bitonic
//                       sort of 64-bit keys (score bits, then inverted index),
//                       the first `keep` flagged and compacted in index order.
#include <cuda_bf16.h>

#include "sana_internal.h"

namespace sana {
namespace {

constexpr int kTile = 128;   // keys per tile; a query block is two tiles
constexpr int kSelThreads = 256;

__global__ void __launch_bounds__(256)
    tile_sums_kernel(const __nv_bfloat16* __restrict__ x, int N, int C, int ntiles,
                     float* __restrict__ sums) {
  const int t = blockIdx.x, b = blockIdx.y;
  const int n0 = t * kTile, n1 = min(N, n0 + kTile);
  const int C2 = C / 2;
  const __nv_bfloat162* xb = reinterpret_cast<const __nv_bfloat162*>(x) + (size_t)b * N * C2;
  for (int c2 = threadIdx.x; c2 < C2; c2 += blockDim.x) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
    for (int n = n0; n < n1; ++n) {
      const float2 f = __bfloat1622float2(xb[(size_t)n * C2 + c2]);
      a0 += f.x;
      a1 += f.y;
    }
    float* o = sums + ((size_t)b * ntiles + t) * C + 2 * c2;
    o[0] = a0;
    o[1] = a1;
  }
}

__device__ __forceinline__ int tile_rows(int t, int N) { return min(N, (t + 1) * kTile) - t * kTile; }

// Larger key = larger score, or equal score and smaller index.
__device__ __forceinline__ unsigned long long sort_key(float score, int idx) {
  const uint32_t u = __float_as_uint(score);
  const uint32_t ordered = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)ordered << 32) | (0xFFFFFFFFu - (uint32_t)idx);
}

__global__ void __launch_bounds__(kSelThreads)
    block_select_kernel(const float* __restrict__ qsums, const float* __restrict__ ksums, int N,
                        int C, int heads, int ntiles, int nqb, int qpc, int keep, int npow2,
                        int* __restrict__ tiles_out) {
  extern __shared__ __align__(16) unsigned char sel_smem[];
  unsigned long long* key = reinterpret_cast<unsigned long long*>(sel_smem);  // [npow2]
  float* qbar = reinterpret_cast<float*>(key + npow2);                          // [qpc][128]
  float* score = qbar + qpc * 128;                                              // [qpc][ntiles]
  int* scan = reinterpret_cast<int*>(score + qpc * ntiles);                     // [kSelThreads]
  unsigned char* flag = reinterpret_cast<unsigned char*>(scan + kSelThreads);   // [ntiles]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int qb0 = blockIdx.x * qpc;
  const int nq = min(qpc, nqb - qb0);
  // pooled queries of the group's blocks (two tiles each, the second may be absent)
  for (int i = tid; i < nq * 128; i += kSelThreads) {
    const int r = i >> 7, d = i & 127;
    const int t0 = 2 * (qb0 + r), t1 = t0 + 1;
    float sum = qsums[((size_t)b * ntiles + t0) * C + h * 128 + d];
    int rows = tile_rows(t0, N);
    if (t1 < ntiles) {
      sum += qsums[((size_t)b * ntiles + t1) * C + h * 128 + d];
      rows += tile_rows(t1, N);
    }
    qbar[r * 128 + d] = sum / (float)rows;
  }
  __syncthreads();
  // scores: warp w takes tiles w, w + 8, ...; lane holds dims 4 lane .. +3
  for (int t = warp; t < ntiles; t += kSelThreads / 32) {
    const float4 kv =
        *reinterpret_cast<const float4*>(ksums + ((size_t)b * ntiles + t) * C + h * 128 + lane * 4);
    const float inv = 1.f / (float)tile_rows(t, N);
    for (int r = 0; r < nq; ++r) {
      const float4 qv = *reinterpret_cast<const float4*>(qbar + r * 128 + lane * 4);
      float d = qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      if (lane == 0) score[r * ntiles + t] = d * inv;
    }
  }
  __syncthreads();
  for (int r = 0; r < nq; ++r) {
    for (int i = tid; i < npow2; i += kSelThreads)
      key[i] = i < ntiles ? sort_key(score[r * ntiles + i], i) : 0ull;
    for (int i = tid; i < ntiles; i += kSelThreads) flag[i] = 0;
    __syncthreads();
    // bitonic sort, descending
    for (int k = 2; k <= npow2; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < npow2; i += kSelThreads) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const unsigned long long a = key[i], c = key[ixj];
            const bool up = (i & k) == 0;
            if (up ? (a < c) : (a > c)) {
              key[i] = c;
              key[ixj] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int i = tid; i < keep; i += kSelThreads)
      flag[0xFFFFFFFFu - (uint32_t)(key[i] & 0xFFFFFFFFull)] = 1;
    __syncthreads();
    // compaction in index order: contiguous ranges per thread + block scan
    const int per = (ntiles + kSelThreads - 1) / kSelThreads;
    const int lo = min(ntiles, tid * per), hi = min(ntiles, lo + per);
    int cnt = 0;
    for (int i = lo; i < hi; ++i) cnt += flag[i];
    scan[tid] = cnt;
    __syncthreads();
    for (int o = 1; o < kSelThreads; o <<= 1) {  // inclusive Hillis-Steele scan
      const int v = tid >= o ? scan[tid - o] : 0;
      __syncthreads();
      scan[tid] += v;
      __syncthreads();
    }
    int off = scan[tid] - cnt;
    int* out = tiles_out + (((size_t)b * heads + h) * nqb + qb0 + r) * keep;
    for (int i = lo; i < hi; ++i)
      if (flag[i]) out[off++] = i;
    __syncthreads();
  }
}

// At least 2, so that the float arrays after the keys stay 16-byte aligned.
int pow2_at_least(int n) {
  int p = 2;
  while (p < n) p <<= 1;
  return p;
}

}  // namespace

int anchor_select_qpc(int ntiles) {
  int q = 16384 / (ntiles > 0 ? ntiles : 1);
  return q < 1 ? 1 : (q > 8 ? 8 : q);
}

size_t anchor_select_smem(int ntiles) {
  const int qpc = anchor_select_qpc(ntiles);
  return (size_t)pow2_at_least(ntiles) * 8 + (size_t)qpc * 128 * 4 + (size_t)qpc * ntiles * 4 +
         kSelThreads * 4 + (size_t)ntiles + 16;
}

sana_status anchor_select_run(int B, int N, int heads, const void* qr, const void* kr, int keep,
                              float* qsums, float* ksums, int* tiles, cudaStream_t st) {
  const int C = heads * 128;
  const int ntiles = (N + kTile - 1) / kTile;
  const int nqb = (ntiles + 1) / 2;
  tile_sums_kernel<<<dim3(ntiles, B), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(qr), N, C,
                                                    ntiles, qsums);
  tile_sums_kernel<<<dim3(ntiles, B), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(kr), N, C,
                                                    ntiles, ksums);
  if (sana_status e = check_launch("tile_sums_kernel")) return e;
  const int qpc = anchor_select_qpc(ntiles);
  const size_t smem = anchor_select_smem(ntiles);
  cudaFuncSetAttribute(block_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  block_select_kernel<<<dim3((nqb + qpc - 1) / qpc, heads, B), kSelThreads, smem, st>>>(
      qsums, ksums, N, C, heads, ntiles, nqb, qpc, keep, pow2_at_least(ntiles), tiles);
  return check_launch("block_select_kernel");
}

}  // namespace sana
