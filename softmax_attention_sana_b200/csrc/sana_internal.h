// Host-side internals of libsana: error reporting, TMA tensor-map encoding,
// workspace carving and the launchers each entry point dispatches to.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>

#include "../../include/sana.h"

namespace sana {

// Fixed SM count of the target part.  Work partitions (and therefore the
// summation order of split reductions) depend only on the problem shape.
constexpr int kNumSMs = 148;

sana_status fail(sana_status st, const char* fmt, ...);
sana_status check_launch(const char* what);
// Unique id of the calling thread's current CUDA context (cuCtxGetId), 0 if
// there is none yet or the driver does not provide it.
unsigned long long current_context_id();
// Function attributes (the dynamic shared-memory opt-in) belong to a CUDA
// context: once_per_context runs `set` for a kernel family the first time a
// call reaches it on a device in a given context (again after a device reset
// gives the device a new context), under a lock, so no launch of that family
// runs before its attributes are set.
enum AttrKey : int {
  kAttrLinattn = 0, kAttrLinattnBwd, kAttrAnchor, kAttrGemm, kAttrMx128, kAttrMx256, kAttrKeys
};
void once_per_context(int key, void (*set)());
// Device address of the status word of the current device.
int* status_word();

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over a caller-provided workspace.
struct Carver {
  char* base;
  size_t cap;
  size_t used = 0;
  Carver(void* b, size_t c) : base(static_cast<char*>(b)), cap(c) {}
  template <class T>
  T* take(size_t count) {
    used = align_up(used, 256);
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += count * sizeof(T);
    return p;
  }
  bool fits() const { return used <= cap; }
};

// TMA descriptors (bf16, 128-byte swizzle, zero fill out of bounds).
// 3D view of a (B, rows, cols) tensor with a row stride of `row_stride` elements
// and a batch stride of `batch_stride` elements; box = (64 cols, box_rows rows, 1).
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                       uint64_t batches, uint64_t row_stride, uint64_t batch_stride,
                       uint32_t box_rows);
// 2D view of a (rows, cols) tensor with row stride `row_stride` elements.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                       uint64_t row_stride, uint32_t box_cols, uint32_t box_rows);

// 2D view of a (rows, cols) tensor of any TMA element type, 128-byte swizzle;
// row stride in bytes; box = (box_cols elements, box_rows rows).
bool make_tmap_2d_typed(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                        uint64_t cols, uint64_t rows, uint64_t row_stride_bytes, uint32_t box_cols,
                        uint32_t box_rows);

// Grid of one call, as the kernels see it.  Batch entry b covers frames
// [t_offset + b * t_stride, + T): t_stride is 0 for independent sequences and
// the block length when consecutive blocks of one sequence are batched.
struct GridDev {
  int T, H, W;
  int t_offset;
  int N;
  int heads;
  int t_stride = 0;
};
// RoPE tables, as the kernels see them.
struct RopeDev {
  const float *cos_t, *sin_t, *cos_h, *sin_h, *cos_w, *sin_w;
  int n_t, n_h, n_w;
};

inline int odd_up(int n) { return n | 1; }
inline size_t rope_smem_bytes(const GridDev& g, const RopeDev& r) {
  return 8 * ((size_t)g.T * odd_up(r.n_t) + (size_t)g.H * odd_up(r.n_h) +
              (size_t)g.W * odd_up(r.n_w));
}
// The tcgen05 kernels stage the rotary tables of one grid in shared memory.
constexpr size_t kRopeSmemMax = 26 * 1024;

// ---------------------------------------------------------------- linear attention
struct LinAttnPlan {
  int splits_a;  // CTAs per (batch, head) of the state reduction
  int splits_b;  // CTAs per (batch, head) of the output pass
  int tiles;     // 128-token tiles per (batch, head)
};
LinAttnPlan linattn_plan(const sana_shape& s, sana_dtype dt);
size_t linattn_ws_bytes(const sana_shape& s, sana_dtype dt);
size_t linattn_state_ws_bytes(const sana_shape& s, sana_dtype dt);
sana_status linattn_state_run(const sana_shape& s, sana_dtype dt, const void* k, const void* v,
                              const RopeDev& rope, float* S_out, float* z_out, void* ws,
                              size_t ws_bytes, cudaStream_t st);
sana_status linattn_apply_run(const sana_shape& s, sana_dtype dt, const void* q, const void* gt,
                              const RopeDev& rope, const float* S, const float* z, float eps,
                              void* out, cudaStream_t st);

// Launchers of the two precisions (linattn_tc.cu for bf16, simt_f32.cu for fp32).
// The partial launchers run the split reduction only; ws_S / ws_z receive
// [B][heads][splits][D][D] / [B][heads][splits][D].
sana_status linattn_bf16_partials(const sana_shape& s, const LinAttnPlan& plan, const void* k,
                                  const void* v, const RopeDev& rope, const GridDev& g,
                                  float* ws_S, float* ws_z, cudaStream_t st);
sana_status linattn_f32_partials(const sana_shape& s, const float* k, const float* v,
                                 const RopeDev& rope, const GridDev& g, int splits, float* ws_S,
                                 float* ws_z, cudaStream_t st);
sana_status linattn_bf16_state(const sana_shape& s, const LinAttnPlan& plan, const void* k,
                               const void* v, const RopeDev& rope, const GridDev& g,
                               const float* S_prev, const float* z_prev, float* S_state,
                               float* z_state, float* ws_S, float* ws_z, float* S_f32,
                               float* z_out, cudaStream_t st);
// prefetch_inputs: the first Q / G tiles may be loaded before the launch
// waits for the previous one (only where q and gt are known to be complete
// when the call's first, ordinarily launched kernel starts).
sana_status linattn_bf16_apply(const sana_shape& s, const LinAttnPlan& plan, const void* q,
                               const void* gt, const RopeDev& rope, const GridDev& g,
                               const float* S_f32, const float* z, float eps, void* out,
                               cudaStream_t st, bool prefetch_inputs = false);
int linattn_f32_splits(const sana_shape& s, int N);
sana_status linattn_f32_state(const sana_shape& s, const float* k, const float* v,
                              const RopeDev& rope, const GridDev& g, int splits,
                              const float* S_prev, const float* z_prev, float* S_state,
                              float* z_state, float* ws_S, float* ws_z, float* S_f32,
                              float* z_comb, cudaStream_t st);
sana_status linattn_f32_apply(const sana_shape& s, const float* q, const float* gt,
                              const RopeDev& rope, const GridDev& g, const float* S_f32,
                              const float* z, float eps, float* out, cudaStream_t st);


// Fixed-order sum of split partials (+ an optional carried state), any D.
void launch_linattn_combine(int BH, const float* ws_S, const float* ws_z, int splits, int D,
                            const float* S_prev, const float* z_prev, float* S_state,
                            float* z_state, float* S_f32, float* z_out, cudaStream_t st);
// Backward of the bf16 layer given S, z (linattn_bwd_tc.cu).
sana_status linattn_bf16_backward(const sana_shape& s, const LinAttnPlan& plan, const void* q,
                                  const void* k, const void* v, const void* gt, const void* dy,
                                  const RopeDev& rope, const GridDev& g, float eps,
                                  const float* S, const float* z, float* ws_dS, float* ws_dz,
                                  float* dS, float* dz, void* dq, void* dk, void* dv, void* dg,
                                  cudaStream_t st);
size_t linattn_bwd_ws_bytes(const sana_shape& s);
sana_status linattn_bwd_run(const sana_shape& s, const void* q, const void* k, const void* v,
                            const void* gt, const void* dy, const RopeDev& rope, float eps,
                            const float* S_saved, const float* z_saved, void* dq, void* dk,
                            void* dv, void* dg, void* ws, size_t ws_bytes, cudaStream_t st);

// Bidirectional (S_prev == nullptr) or block-causal step.
sana_status linattn_run(const sana_shape& s, sana_dtype dt, const void* q, const void* k,
                        const void* v, const void* g, const RopeDev& rope, float eps,
                        float* state_S, float* state_z, bool causal, bool commit, void* out,
                        void* ws, size_t ws_bytes, cudaStream_t st);

// A whole sequence of blocks of `chunk_frames` frames (the last block takes
// the remaining frames): per-block states in parallel, a fixed-order prefix
// over blocks, then every block's output.
size_t linattn_scan_ws_bytes(const sana_shape& s, int chunk_frames, sana_dtype dt);
sana_status linattn_scan_run(const sana_shape& s, int chunk_frames, sana_dtype dt, const void* q,
                             const void* k, const void* v, const void* g, const RopeDev& rope,
                             float eps, float* state_S, float* state_z, bool commit, void* out,
                             void* ws, size_t ws_bytes, cudaStream_t st);

// ---------------------------------------------------------------- softmax anchor
size_t anchor_ws_bytes(const sana_shape& s, sana_dtype dt);
sana_status anchor_run(const sana_shape& s, sana_dtype dt, const void* q, const void* k,
                       const void* v, const void* g, const RopeDev* rope, float scale,
                       void* out, void* ws, size_t ws_bytes, cudaStream_t st);

// Block-sparse anchor: tile selection (anchor_select.cu) and the anchor kernel
// over listed key tiles (anchor_tc.cu; tiles == nullptr visits every tile).
constexpr int kAnchorMaxTiles = 16384;  // key tiles the selection supports (N <= 2M)
size_t anchor_select_smem(int ntiles);
sana_status anchor_select_run(int B, int N, int heads, const void* qr, const void* kr, int keep,
                              float* qsums, float* ksums, int* tiles, cudaStream_t st);
sana_status anchor_bf16_run(const sana_shape& s, const void* qr, const void* kr, const void* v,
                            const void* gt, const GridDev& g, const int* tiles, int keep,
                            void* out, cudaStream_t st);
size_t anchor_sparse_ws_bytes(const sana_shape& s);
sana_status anchor_sparse_run(const sana_shape& s, const void* q, const void* k, const void* v,
                              const void* g, const RopeDev* rope, float scale, int keep, int* tiles,
                              bool select, void* out, void* ws, size_t ws_bytes, cudaStream_t st);

// ---------------------------------------------------------------- AttnRes / norm / GEMM
sana_status attnres_run(int B, long long N, int C, sana_dtype dt, const void* const* sources,
                        int S, const float* w, float eps, void* h, float* alpha, bool normed_out,
                        void* h_norm, cudaStream_t st);
size_t attnres_bwd_ws_bytes(long long tokens, int C);
sana_status attnres_bwd_run(long long tokens, int C, const void* const* sources, int S,
                            const float* w, float eps, const void* dh, void* const* d_sources,
                            float* dw, void* ws, size_t ws_bytes, cudaStream_t st);
sana_status rmsnorm_run(long long rows, int C, sana_dtype dt, const void* x, float eps, void* y,
                        cudaStream_t st);
sana_status gemm_run(long long M, int N, int K, const void* A, long long lda, const void* W,
                     void* out, long long ldo, int epilogue, cudaStream_t st);

// ---------------------------------------------------------------- MX projection GEMM
// Scale bytes of a (rows, K) operand: 512-byte atoms of 128 rows x 128 K-elements.
size_t mx_scale_bytes(long long rows, int K);
// bf16 (rows, K) -> E4M3 bytes (fp4 = false) or packed E2M1 (fp4 = true) + scales.
sana_status mx_quantize_run(const void* x, long long rows, int K, bool fp4, void* q, void* sf,
                            cudaStream_t st);
// out[M][N] = epilogue(Q8(x) . Q4(w)^T) from quantised operands.
sana_status mx_gemm_run(long long M, int N, int K, const void* xq, const void* xsf,
                        const void* wq, const void* wsf, void* out, long long ldo, int epilogue,
                        cudaStream_t st);
// The same with the output columns split into nparts equal tensors.
sana_status mx_gemm_run_parts(long long M, int N, int K, const void* xq, const void* xsf,
                              const void* wq, const void* wsf, void* const* outs, int nparts,
                              long long ldo, int epilogue, cudaStream_t st);

}  // namespace sana
