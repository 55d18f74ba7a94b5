// libsana C ABI: argument validation, workspace sizing, dispatch to the
// kernels, RoPE tables, error strings and the device status word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {

__device__ int g_status_word;

namespace {
thread_local std::string g_err = "ok";
}

sana_status fail(sana_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

sana_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SANA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return SANA_OK;
}

unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

void once_per_context(int key, void (*set)()) {
  static unsigned long long done[kAttrKeys][64] = {};
  static std::mutex mu;
  int dev = 0;
  const bool have_dev = cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (have_dev && ctx != 0 && done[key][dev] == ctx) return;
  set();
  if (have_dev) done[key][dev] = current_context_id();
}

int* status_word() {
  // One slot per device, valid for the context it was looked up in: a device
  // reset gives the device a new context whose copy of the word may sit at a
  // new address, so a changed context id forces a new lookup.
  struct Slot {
    unsigned long long ctx;
    int* addr;
  };
  static Slot slots[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (ctx != 0 && slots[dev].ctx == ctx && slots[dev].addr) return slots[dev].addr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
  // the lookup makes the primary context current when none was
  slots[dev] = Slot{current_context_id(), static_cast<int*>(p)};
  return slots[dev].addr;
}

// ---------------------------------------------------------------- failure-detection self-test
namespace {
// Waits on an mbarrier that nothing ever arrives on, through the same bounded
// wait every pipeline uses; after limit_ns it records a timeout and returns.
__global__ void bounded_wait_selftest_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  const WaitCtx wc{&abort_flag, status};
  mbar_wait(&bar, 0, wc, 0x7f, limit_ns);
}
}  // namespace

// ---------------------------------------------------------------- tensor maps
namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}
}  // namespace

bool make_tmap_2d_typed(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                        uint64_t cols, uint64_t rows, uint64_t row_stride_bytes, uint32_t box_cols,
                        uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                       uint64_t batches, uint64_t row_stride, uint64_t batch_stride,
                       uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {cols, rows, batches};
  const cuuint64_t strides[2] = {row_stride * 2, batch_stride * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                       uint64_t row_stride, uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- validation helpers
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

size_t esize(sana_dtype dt) { return dt == SANA_BF16 ? 2 : 4; }

sana_status check_shape(const sana_shape* s, sana_dtype dt, const char* who) {
  if (!s) return fail(SANA_ERR_INVALID_ARG, "%s: shape is NULL", who);
  if (dt != SANA_F32 && dt != SANA_BF16) return fail(SANA_ERR_INVALID_ARG, "%s: bad dtype %d", who, (int)dt);
  if (s->B < 1 || s->T < 0 || s->H < 1 || s->W < 1 || s->heads < 1 || s->t_offset < 0)
    return fail(SANA_ERR_INVALID_ARG, "%s: bad shape B=%d T=%d H=%d W=%d heads=%d t_offset=%d", who,
                s->B, s->T, s->H, s->W, s->heads, s->t_offset);
  const long long N = (long long)s->T * s->H * s->W;
  if (N >= (1LL << 31) / 2) return fail(SANA_ERR_UNSUPPORTED, "%s: N=%lld too large", who, N);
  const int D = s->head_dim;
  if (dt == SANA_BF16 && D != 128)
    return fail(SANA_ERR_UNSUPPORTED, "%s: bf16 needs head_dim 128 (got %d)", who, D);
  if (dt == SANA_F32 && D != 16 && D != 32 && D != 64 && D != 128)
    return fail(SANA_ERR_UNSUPPORTED, "%s: fp32 head_dim must be 16/32/64/128 (got %d)", who, D);
  return SANA_OK;
}

sana_status check_rope(const sana_rope* r, const sana_shape* s, const char* who) {
  if (!r) return fail(SANA_ERR_INVALID_ARG, "%s: rope is NULL", who);
  if (r->n_t < 0 || r->n_h < 0 || r->n_w < 0 || r->n_t + r->n_h + r->n_w != s->head_dim / 2)
    return fail(SANA_ERR_INVALID_ARG, "%s: rope split %d/%d/%d does not cover head_dim/2=%d", who,
                r->n_t, r->n_h, r->n_w, s->head_dim / 2);
  if (r->H != s->H || r->W != s->W || r->T_total < s->t_offset + s->T)
    return fail(SANA_ERR_INVALID_ARG,
                "%s: rope tables (T_total=%d, H=%d, W=%d) do not cover frames [%d, %d) of %dx%d", who,
                r->T_total, r->H, r->W, s->t_offset, s->t_offset + s->T, s->H, s->W);
  if ((r->n_t && (!r->cos_t || !r->sin_t)) || (r->n_h && (!r->cos_h || !r->sin_h)) ||
      (r->n_w && (!r->cos_w || !r->sin_w)))
    return fail(SANA_ERR_INVALID_ARG, "%s: rope table pointer is NULL", who);
  return SANA_OK;
}

RopeDev to_dev(const sana_rope& r) {
  return RopeDev{r.cos_t, r.sin_t, r.cos_h, r.sin_h, r.cos_w, r.sin_w, r.n_t, r.n_h, r.n_w};
}

GridDev to_grid(const sana_shape& s) {
  return GridDev{s.T, s.H, s.W, s.t_offset, s.T * s.H * s.W, s.heads};
}

}  // namespace

// ---------------------------------------------------------------- linear attention
LinAttnPlan linattn_plan(const sana_shape& s, sana_dtype dt) {
  LinAttnPlan p{};
  const int N = s.T * s.H * s.W;
  const int bh = s.B * s.heads;
  if (dt == SANA_BF16) {
    p.tiles = (N + 127) / 128;
    int sp = kNumSMs / bh;
    if (sp < 1) sp = 1;
    if (sp > p.tiles) sp = p.tiles;
    if (sp < 1) sp = 1;
    p.splits_a = p.splits_b = sp;
  } else {
    p.tiles = (N + 31) / 32;
    p.splits_a = p.splits_b = linattn_f32_splits(s, N > 0 ? N : 1);
  }
  return p;
}

namespace {
struct LinWs {
  float* ws_S;   // split partials of S
  float* ws_z;   // split partials of z
  float* S_f32;  // combined S
  float* z_comb; // combined z
  size_t partial_bytes;  // what the state phase alone needs
  size_t bytes;          // what the whole layer needs
};
LinWs carve_linattn(const sana_shape& s, sana_dtype dt, void* ws) {
  const LinAttnPlan p = linattn_plan(s, dt);
  const size_t bh = (size_t)s.B * s.heads, D = s.head_dim;
  Carver cv(ws, ~size_t(0));
  LinWs w{};
  w.ws_S = cv.take<float>(bh * p.splits_a * D * D);
  w.ws_z = cv.take<float>(bh * p.splits_a * D);
  w.partial_bytes = align_up(cv.used, 256);
  w.S_f32 = cv.take<float>(bh * D * D);
  w.z_comb = cv.take<float>(bh * D);
  w.bytes = align_up(cv.used, 256);
  return w;
}

sana_status state_phase(const sana_shape& s, sana_dtype dt, const void* k, const void* v,
                        const RopeDev& rope, const GridDev& g, const float* S_prev,
                        const float* z_prev, float* S_state, float* z_state, const LinWs& w,
                        float* S_out, float* z_out, cudaStream_t st) {
  const LinAttnPlan p = linattn_plan(s, dt);
  if (dt == SANA_BF16)
    return linattn_bf16_state(s, p, k, v, rope, g, S_prev, z_prev, S_state, z_state, w.ws_S,
                              w.ws_z, S_out, z_out, st);
  return linattn_f32_state(s, static_cast<const float*>(k), static_cast<const float*>(v), rope, g,
                           p.splits_a, S_prev, z_prev, S_state, z_state, w.ws_S, w.ws_z, S_out,
                           z_out, st);
}

sana_status apply_phase(const sana_shape& s, sana_dtype dt, const void* q, const void* gt,
                        const RopeDev& rope, const GridDev& g, const float* S, const float* z,
                        float eps, void* out, cudaStream_t st, bool prefetch_inputs) {
  if (dt == SANA_BF16) {
    if (rope_smem_bytes(g, rope) > kRopeSmemMax)
      return fail(SANA_ERR_UNSUPPORTED,
                  "linear attention: grid %dx%dx%d needs %zu B of RoPE tables (max %zu)", g.T, g.H,
                  g.W, rope_smem_bytes(g, rope), kRopeSmemMax);
    return linattn_bf16_apply(s, linattn_plan(s, dt), q, gt, rope, g, S, z, eps, out, st,
                              prefetch_inputs);
  }
  return linattn_f32_apply(s, static_cast<const float*>(q), static_cast<const float*>(gt), rope,
                           g, S, z, eps, static_cast<float*>(out), st);
}
}  // namespace

size_t linattn_ws_bytes(const sana_shape& s, sana_dtype dt) {
  return carve_linattn(s, dt, nullptr).bytes;
}
size_t linattn_state_ws_bytes(const sana_shape& s, sana_dtype dt) {
  return carve_linattn(s, dt, nullptr).partial_bytes;
}

sana_status linattn_run(const sana_shape& s, sana_dtype dt, const void* q, const void* k,
                        const void* v, const void* gt, const RopeDev& rope, float eps,
                        float* state_S, float* state_z, bool causal, bool commit, void* out,
                        void* ws, size_t ws_bytes, cudaStream_t st) {
  const GridDev g = to_grid(s);
  if (g.N == 0) return SANA_OK;
  const LinWs w = carve_linattn(s, dt, ws);
  if (ws_bytes < w.bytes)
    return fail(SANA_ERR_WORKSPACE, "linear attention: workspace %zu < %zu bytes", ws_bytes, w.bytes);
  if (dt == SANA_BF16 && rope_smem_bytes(g, rope) > kRopeSmemMax)
    return fail(SANA_ERR_UNSUPPORTED,
                "linear attention: grid %dx%dx%d needs %zu B of RoPE tables (max %zu)", g.T, g.H,
                g.W, rope_smem_bytes(g, rope), kRopeSmemMax);
  const float* S_prev = causal ? state_S : nullptr;
  const float* z_prev = causal ? state_z : nullptr;
  float* S_commit = causal && commit ? state_S : nullptr;
  float* z_commit = causal && commit ? state_z : nullptr;
  if (sana_status e = state_phase(s, dt, k, v, rope, g, S_prev, z_prev, S_commit, z_commit, w,
                                  w.S_f32, w.z_comb, st))
    return e;
  // the state phase's first kernel is an ordinary launch: q and gt are
  // complete when the output kernel starts
  return apply_phase(s, dt, q, gt, rope, g, w.S_f32, w.z_comb, eps, out, st, true);
}

sana_status linattn_state_run(const sana_shape& s, sana_dtype dt, const void* k, const void* v,
                              const RopeDev& rope, float* S_out, float* z_out, void* ws,
                              size_t ws_bytes, cudaStream_t st) {
  const GridDev g = to_grid(s);
  const LinWs w = carve_linattn(s, dt, ws);
  if (ws_bytes < w.partial_bytes)
    return fail(SANA_ERR_WORKSPACE, "linear attention state: workspace %zu < %zu bytes", ws_bytes,
                w.partial_bytes);
  if (g.N == 0) {
    cudaMemsetAsync(S_out, 0, (size_t)s.B * s.heads * s.head_dim * s.head_dim * 4, st);
    cudaMemsetAsync(z_out, 0, (size_t)s.B * s.heads * s.head_dim * 4, st);
    return check_launch("linear attention state (empty)");
  }
  if (dt == SANA_BF16 && rope_smem_bytes(g, rope) > kRopeSmemMax)
    return fail(SANA_ERR_UNSUPPORTED, "linear attention: grid needs too many RoPE table bytes");
  return state_phase(s, dt, k, v, rope, g, nullptr, nullptr, nullptr, nullptr, w, S_out, z_out, st);
}

sana_status linattn_apply_run(const sana_shape& s, sana_dtype dt, const void* q, const void* gt,
                              const RopeDev& rope, const float* S, const float* z, float eps,
                              void* out, cudaStream_t st) {
  const GridDev g = to_grid(s);
  if (g.N == 0) return SANA_OK;
  return apply_phase(s, dt, q, gt, rope, g, S, z, eps, out, st, false);
}

// ---------------------------------------------------------------- backward (bf16)
// Workspace: the forward state phase's partials and combined (S, z), then the
// same again for (dS, dz).
size_t linattn_bwd_ws_bytes(const sana_shape& s) {
  const size_t one = carve_linattn(s, SANA_BF16, nullptr).bytes;
  return 2 * one;
}

// S_saved / z_saved: the forward's combined state, or NULL to rebuild it from k, v.
sana_status linattn_bwd_run(const sana_shape& s, const void* q, const void* k, const void* v,
                            const void* gt, const void* dy, const RopeDev& rope, float eps,
                            const float* S_saved, const float* z_saved, void* dq, void* dk,
                            void* dv, void* dg, void* ws, size_t ws_bytes, cudaStream_t st) {
  const GridDev g = to_grid(s);
  if (g.N == 0) return SANA_OK;
  const size_t one = carve_linattn(s, SANA_BF16, nullptr).bytes;
  if (ws_bytes < 2 * one)
    return fail(SANA_ERR_WORKSPACE, "linear attention backward: workspace %zu < %zu bytes",
                ws_bytes, 2 * one);
  if (rope_smem_bytes(g, rope) > kRopeSmemMax)
    return fail(SANA_ERR_UNSUPPORTED, "linear attention backward: grid needs too many RoPE table bytes");
  const LinWs fw = carve_linattn(s, SANA_BF16, ws);
  const LinWs bw = carve_linattn(s, SANA_BF16, static_cast<char*>(ws) + one);
  const LinAttnPlan plan = linattn_plan(s, SANA_BF16);
  const float* S = S_saved;
  const float* z = z_saved;
  if (!S) {
    if (sana_status e = linattn_bf16_state(s, plan, k, v, rope, g, nullptr, nullptr, nullptr,
                                           nullptr, fw.ws_S, fw.ws_z, fw.S_f32, fw.z_comb, st))
      return e;
    S = fw.S_f32;
    z = fw.z_comb;
  }
  return linattn_bf16_backward(s, plan, q, k, v, gt, dy, rope, g, eps, S, z, bw.ws_S, bw.ws_z,
                               bw.S_f32, bw.z_comb, dq, dk, dv, dg, st);
}

// ---------------------------------------------------------------- anchor
sana_status rope_rotate_run(const void* x, bool bf16, const RopeDev* rope, const GridDev& g, int B,
                            int D, float mul, void* out, cudaStream_t st);
sana_status anchor_f32_run(const sana_shape& s, const float* qr, const float* kr, const float* v,
                           const float* gt, const GridDev& g, float scale, float* out,
                           cudaStream_t st);

size_t anchor_ws_bytes(const sana_shape& s, sana_dtype dt) {
  const size_t n = (size_t)s.B * s.T * s.H * s.W * s.heads * s.head_dim;
  Carver cv(nullptr, ~size_t(0));
  cv.take<char>(n * esize(dt));
  cv.take<char>(n * esize(dt));
  return align_up(cv.used, 256);
}

sana_status anchor_run(const sana_shape& s, sana_dtype dt, const void* q, const void* k,
                       const void* v, const void* gt, const RopeDev* rope, float scale, void* out,
                       void* ws, size_t ws_bytes, cudaStream_t st) {
  const GridDev g = to_grid(s);
  if (g.N == 0) return SANA_OK;
  const size_t need = anchor_ws_bytes(s, dt);
  if (ws_bytes < need)
    return fail(SANA_ERR_WORKSPACE, "softmax anchor: workspace %zu < %zu bytes", ws_bytes, need);
  const size_t n = (size_t)s.B * g.N * s.heads * s.head_dim;
  Carver cv(ws, ws_bytes);
  void* qr = cv.take<char>(n * esize(dt));
  void* kr = cv.take<char>(n * esize(dt));
  const int D = s.head_dim;
  if (scale <= 0.f) scale = 1.f / sqrtf((float)D);
  if (dt == SANA_BF16) {
    // Q is pre-scaled by scale * log2(e) so the kernel's softmax works in base 2.
    const float qmul = scale * 1.4426950408889634f;
    if (sana_status e = rope_rotate_run(q, true, rope, g, s.B, D, qmul, qr, st)) return e;
    if (sana_status e = rope_rotate_run(k, true, rope, g, s.B, D, 1.f, kr, st)) return e;
    return anchor_bf16_run(s, qr, kr, v, gt, g, nullptr, 0, out, st);
  }
  if (sana_status e = rope_rotate_run(q, false, rope, g, s.B, D, 1.f, qr, st)) return e;
  if (sana_status e = rope_rotate_run(k, false, rope, g, s.B, D, 1.f, kr, st)) return e;
  return anchor_f32_run(s, static_cast<const float*>(qr), static_cast<const float*>(kr),
                        static_cast<const float*>(v), static_cast<const float*>(gt), g, scale,
                        static_cast<float*>(out), st);
}

// Sparse form (bf16): the same prepass, then (if select) the tile selection,
// then the anchor kernel over the listed tiles.
size_t anchor_sparse_ws_bytes(const sana_shape& s) {
  const size_t N = (size_t)s.T * s.H * s.W;
  const size_t ntiles = (N + 127) / 128;
  Carver cv(nullptr, ~size_t(0));
  cv.take<char>(anchor_ws_bytes(s, SANA_BF16));
  cv.take<float>((size_t)s.B * ntiles * s.heads * s.head_dim);
  cv.take<float>((size_t)s.B * ntiles * s.heads * s.head_dim);
  return align_up(cv.used, 256);
}

sana_status anchor_sparse_run(const sana_shape& s, const void* q, const void* k, const void* v,
                              const void* gt, const RopeDev* rope, float scale, int keep, int* tiles,
                              bool select, void* out, void* ws, size_t ws_bytes, cudaStream_t st) {
  const GridDev g = to_grid(s);
  if (g.N == 0) return SANA_OK;
  const size_t need = anchor_sparse_ws_bytes(s);
  if (ws_bytes < need)
    return fail(SANA_ERR_WORKSPACE, "sparse anchor: workspace %zu < %zu bytes", ws_bytes, need);
  const size_t n = (size_t)s.B * g.N * s.heads * s.head_dim;
  const size_t ntiles = ((size_t)g.N + 127) / 128;
  Carver cv(ws, ws_bytes);
  void* qr = cv.take<char>(n * 2);
  void* kr = cv.take<char>(n * 2);
  cv.used = align_up(anchor_ws_bytes(s, SANA_BF16), 256);
  float* qsums = cv.take<float>((size_t)s.B * ntiles * s.heads * s.head_dim);
  float* ksums = cv.take<float>((size_t)s.B * ntiles * s.heads * s.head_dim);
  if (scale <= 0.f) scale = 1.f / sqrtf((float)s.head_dim);
  const float qmul = scale * 1.4426950408889634f;
  if (sana_status e = rope_rotate_run(q, true, rope, g, s.B, s.head_dim, qmul, qr, st)) return e;
  if (sana_status e = rope_rotate_run(k, true, rope, g, s.B, s.head_dim, 1.f, kr, st)) return e;
  if (select)
    if (sana_status e = anchor_select_run(s.B, g.N, s.heads, qr, kr, keep, qsums, ksums, tiles, st))
      return e;
  return anchor_bf16_run(s, qr, kr, v, gt, g, tiles, keep, out, st);
}

}  // namespace sana

// ============================================================================
// extern "C" entry points
// ============================================================================
using namespace sana;

extern "C" {

const char* sana_version(void) { return "libsana 0.1 (sm_100a)"; }

const char* sana_last_error_string(void) { return g_err.c_str(); }

size_t sana_rope_tables_count(int T_total, int H, int W, int n_t, int n_h, int n_w) {
  if (T_total < 0 || H < 0 || W < 0 || n_t < 0 || n_h < 0 || n_w < 0) return 0;
  return 2 * ((size_t)T_total * n_t + (size_t)H * n_h + (size_t)W * n_w);
}

sana_status sana_rope_tables_host(int T_total, int H, int W, int n_t, int n_h, int n_w,
                                  double theta, float* out) {
  if (!out) return fail(SANA_ERR_INVALID_ARG, "rope tables: output buffer is NULL");
  if (T_total < 0 || H < 0 || W < 0 || n_t < 0 || n_h < 0 || n_w < 0 || !(theta > 0.0))
    return fail(SANA_ERR_INVALID_ARG, "rope tables: bad sizes or theta");
  float* p = out;
  const int npos[3] = {T_total, H, W};
  const int npair[3] = {n_t, n_h, n_w};
  for (int ax = 0; ax < 3; ++ax) {
    float* c = p;
    float* s = p + (size_t)npos[ax] * npair[ax];
    for (int pos = 0; pos < npos[ax]; ++pos)
      for (int k = 0; k < npair[ax]; ++k) {
        const double ang = (double)pos * std::pow(theta, -(double)k / npair[ax]);
        c[(size_t)pos * npair[ax] + k] = (float)std::cos(ang);
        s[(size_t)pos * npair[ax] + k] = (float)std::sin(ang);
      }
    p += 2 * (size_t)npos[ax] * npair[ax];
  }
  return SANA_OK;
}

sana_status sana_rope_bind(const float* t, int T_total, int H, int W, int n_t, int n_h, int n_w,
                           sana_rope* out) {
  if (!t || !out) return fail(SANA_ERR_INVALID_ARG, "rope bind: NULL argument");
  if (T_total < 0 || H < 0 || W < 0 || n_t < 0 || n_h < 0 || n_w < 0)
    return fail(SANA_ERR_INVALID_ARG, "rope bind: bad sizes");
  out->cos_t = t;
  out->sin_t = t + (size_t)T_total * n_t;
  t += 2 * (size_t)T_total * n_t;
  out->cos_h = t;
  out->sin_h = t + (size_t)H * n_h;
  t += 2 * (size_t)H * n_h;
  out->cos_w = t;
  out->sin_w = t + (size_t)W * n_w;
  out->n_t = n_t;
  out->n_h = n_h;
  out->n_w = n_w;
  out->T_total = T_total;
  out->H = H;
  out->W = W;
  return SANA_OK;
}

size_t sana_linattn_workspace_size(const sana_shape* s, sana_dtype dt) {
  if (check_shape(s, dt, "sana_linattn_workspace_size") != SANA_OK) return 0;
  return linattn_ws_bytes(*s, dt);
}

static sana_status linattn_common(const char* who, const sana_shape* s, sana_dtype dt,
                                  const void* q, const void* k, const void* v, const void* g,
                                  const sana_rope* rope, float eps, float* S, float* z,
                                  bool causal, int commit, void* out, void* ws, size_t ws_bytes,
                                  sana_stream_t stream) {
  if (sana_status e = check_shape(s, dt, who)) return e;
  if (sana_status e = check_rope(rope, s, who)) return e;
  if (!std::isfinite(eps) || eps < 0.f) return fail(SANA_ERR_INVALID_ARG, "%s: eps must be finite and >= 0", who);
  if (s->T == 0) return SANA_OK;  // empty grid: nothing to read or write, state unchanged
  if (!q || !k || !v || !out) return fail(SANA_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
  const void* ptrs[5] = {q, k, v, g, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t n = (size_t)s->B * s->T * s->H * s->W * s->heads * s->head_dim * esize(dt);
  if (overlap(out, n, q, n) || overlap(out, n, k, n) || overlap(out, n, v, n) || overlap(out, n, g, n))
    return fail(SANA_ERR_INVALID_ARG, "%s: out aliases an input", who);
  if (causal) {
    if (!S || !z) return fail(SANA_ERR_INVALID_ARG, "%s: state pointers are NULL", who);
    const size_t sb = (size_t)s->B * s->heads * s->head_dim * s->head_dim * 4;
    const size_t zb = (size_t)s->B * s->heads * s->head_dim * 4;
    if (overlap(S, sb, out, n) || overlap(z, zb, out, n) || overlap(S, sb, z, zb))
      return fail(SANA_ERR_INVALID_ARG, "%s: state aliases the output", who);
    if (!aligned16(S) || !aligned16(z)) return fail(SANA_ERR_INVALID_ARG, "%s: state must be 16-byte aligned", who);
  }
  const size_t need = linattn_ws_bytes(*s, dt);
  if (need && (!ws || ws_bytes < need))
    return fail(SANA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws ? ws_bytes : 0, need);
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(SANA_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
  return linattn_run(*s, dt, q, k, v, g, to_dev(*rope), eps, S, z, causal, commit != 0, out, ws,
                     ws_bytes, stream);
}

sana_status sana_linattn_fwd(const sana_shape* s, sana_dtype dt, const void* q, const void* k,
                             const void* v, const void* g, const sana_rope* rope, float eps,
                             void* out, void* ws, size_t ws_bytes, sana_stream_t stream) {
  return linattn_common("sana_linattn_fwd", s, dt, q, k, v, g, rope, eps, nullptr, nullptr, false,
                        0, out, ws, ws_bytes, stream);
}

sana_status sana_linattn_block_causal_step(const sana_shape* s, sana_dtype dt, const void* q,
                                           const void* k, const void* v, const void* g,
                                           const sana_rope* rope, float eps, float* S, float* z,
                                           int commit, void* out, void* ws, size_t ws_bytes,
                                           sana_stream_t stream) {
  return linattn_common("sana_linattn_block_causal_step", s, dt, q, k, v, g, rope, eps, S, z, true,
                        commit, out, ws, ws_bytes, stream);
}

size_t sana_linattn_bwd_workspace_size(const sana_shape* s, sana_dtype dt) {
  if (check_shape(s, dt, "sana_linattn_bwd_workspace_size") != SANA_OK || dt != SANA_BF16) return 0;
  return linattn_bwd_ws_bytes(*s);
}

// Validation shared by both backward entry points (S, z NULL for the first).
static sana_status bwd_checked_run(const char* who, bool saved, const sana_shape* s, sana_dtype dt,
                            const void* q, const void* k, const void* v, const void* g,
                            const sana_rope* rope, float eps, const float* S, const float* z,
                            const void* dy, void* dq, void* dk, void* dv, void* dg, void* ws,
                            size_t ws_bytes, cudaStream_t stream) {
  if (sana_status e = check_shape(s, dt, who)) return e;
  if (dt != SANA_BF16) return fail(SANA_ERR_UNSUPPORTED, "%s: bf16 only", who);
  if (sana_status e = check_rope(rope, s, who)) return e;
  if (!std::isfinite(eps) || eps < 0.f) return fail(SANA_ERR_INVALID_ARG, "%s: eps must be finite and >= 0", who);
  if (s->T == 0) return SANA_OK;
  if (!q || !k || !v || !dy || !dq || !dk || !dv)
    return fail(SANA_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
  if ((g == nullptr) != (dg == nullptr))
    return fail(SANA_ERR_INVALID_ARG, "%s: gate_logits and d_gate must both be given or both be NULL", who);
  const void* ins[5] = {q, k, v, g, dy};
  const void* outs[4] = {dq, dk, dv, dg};
  for (const void* p : ins)
    if (p && !aligned16(p)) return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  for (const void* p : outs)
    if (p && !aligned16(p)) return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t n = (size_t)s->B * s->T * s->H * s->W * s->heads * s->head_dim * 2;
  for (const void* o : outs) {
    for (const void* i : ins)
      if (overlap(o, n, i, n)) return fail(SANA_ERR_INVALID_ARG, "%s: a gradient aliases an input", who);
    for (const void* o2 : outs)
      if (o2 != o && overlap(o, n, o2, n)) return fail(SANA_ERR_INVALID_ARG, "%s: gradients alias each other", who);
  }
  if (saved) {
    if (!S || !z) return fail(SANA_ERR_INVALID_ARG, "%s: saved state S, z must be given", who);
    if (!aligned16(S) || !aligned16(z))
      return fail(SANA_ERR_INVALID_ARG, "%s: state must be 16-byte aligned", who);
    const size_t sb = (size_t)s->B * s->heads * s->head_dim * s->head_dim * 4;
    const size_t zb = (size_t)s->B * s->heads * s->head_dim * 4;
    for (const void* o : outs)
      if (o && (overlap(o, n, S, sb) || overlap(o, n, z, zb)))
        return fail(SANA_ERR_INVALID_ARG, "%s: a gradient aliases the saved state", who);
  }
  const size_t need = linattn_bwd_ws_bytes(*s);
  if (!ws || ws_bytes < need)
    return fail(SANA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws ? ws_bytes : 0, need);
  if (reinterpret_cast<uintptr_t>(ws) & 255u)
    return fail(SANA_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
  if (saved) {
    const size_t sb = (size_t)s->B * s->heads * s->head_dim * s->head_dim * 4;
    if (overlap(ws, ws_bytes, S, sb) || overlap(ws, ws_bytes, z, (size_t)s->B * s->heads * s->head_dim * 4))
      return fail(SANA_ERR_INVALID_ARG, "%s: the workspace overlaps the saved state", who);
  }
  return linattn_bwd_run(*s, q, k, v, g, dy, to_dev(*rope), eps, saved ? S : nullptr,
                         saved ? z : nullptr, dq, dk, dv, dg, ws, ws_bytes, stream);
}

sana_status sana_linattn_bwd(const sana_shape* s, sana_dtype dt, const void* q, const void* k,
                             const void* v, const void* g, const sana_rope* rope, float eps,
                             const void* dy, void* dq, void* dk, void* dv, void* dg, void* ws,
                             size_t ws_bytes, sana_stream_t stream) {
  return bwd_checked_run("sana_linattn_bwd", false, s, dt, q, k, v, g, rope, eps, nullptr, nullptr,
                         dy, dq, dk, dv, dg, ws, ws_bytes, stream);
}

sana_status sana_linattn_bwd_saved_state(const sana_shape* s, sana_dtype dt, const void* q,
                                         const void* k, const void* v, const void* g,
                                         const sana_rope* rope, float eps, const float* S,
                                         const float* z, const void* dy, void* dq, void* dk,
                                         void* dv, void* dg, void* ws, size_t ws_bytes,
                                         sana_stream_t stream) {
  return bwd_checked_run("sana_linattn_bwd_saved_state", true, s, dt, q, k, v, g, rope, eps, S, z,
                         dy, dq, dk, dv, dg, ws, ws_bytes, stream);
}

size_t sana_linattn_block_causal_scan_workspace_size(const sana_shape* s, int chunk_frames,
                                                     sana_dtype dt) {
  if (check_shape(s, dt, "sana_linattn_block_causal_scan_workspace_size") != SANA_OK ||
      chunk_frames < 1)
    return 0;
  return linattn_scan_ws_bytes(*s, chunk_frames, dt);
}

sana_status sana_linattn_block_causal_scan(const sana_shape* s, int chunk_frames, sana_dtype dt,
                                           const void* q, const void* k, const void* v,
                                           const void* g, const sana_rope* rope, float eps,
                                           float* S, float* z, int commit, void* out, void* ws,
                                           size_t ws_bytes, sana_stream_t stream) {
  const char* who = "sana_linattn_block_causal_scan";
  if (sana_status e = check_shape(s, dt, who)) return e;
  if (sana_status e = check_rope(rope, s, who)) return e;
  if (chunk_frames < 1) return fail(SANA_ERR_INVALID_ARG, "%s: chunk_frames=%d", who, chunk_frames);
  if (!std::isfinite(eps) || eps < 0.f) return fail(SANA_ERR_INVALID_ARG, "%s: eps must be finite and >= 0", who);
  if (!S || !z) return fail(SANA_ERR_INVALID_ARG, "%s: state pointers are NULL", who);
  if (!aligned16(S) || !aligned16(z)) return fail(SANA_ERR_INVALID_ARG, "%s: state must be 16-byte aligned", who);
  if (s->T == 0) return SANA_OK;  // no blocks: nothing to read or write, state unchanged
  if (!q || !k || !v || !out) return fail(SANA_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
  const void* ptrs[5] = {q, k, v, g, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t n = (size_t)s->B * s->T * s->H * s->W * s->heads * s->head_dim * esize(dt);
  if (overlap(out, n, q, n) || overlap(out, n, k, n) || overlap(out, n, v, n) || overlap(out, n, g, n))
    return fail(SANA_ERR_INVALID_ARG, "%s: out aliases an input", who);
  const size_t sb = (size_t)s->B * s->heads * s->head_dim * s->head_dim * 4;
  const size_t zb = (size_t)s->B * s->heads * s->head_dim * 4;
  if (overlap(S, sb, out, n) || overlap(z, zb, out, n) || overlap(S, sb, z, zb))
    return fail(SANA_ERR_INVALID_ARG, "%s: state aliases the output", who);
  const size_t need = linattn_scan_ws_bytes(*s, chunk_frames, dt);
  if (!ws || ws_bytes < need)
    return fail(SANA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws ? ws_bytes : 0, need);
  if (reinterpret_cast<uintptr_t>(ws) & 255u)
    return fail(SANA_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
  if (overlap(ws, need, out, n) || overlap(ws, need, S, sb) || overlap(ws, need, z, zb))
    return fail(SANA_ERR_INVALID_ARG, "%s: workspace aliases the output or the state", who);
  return linattn_scan_run(*s, chunk_frames, dt, q, k, v, g, to_dev(*rope), eps, S, z, commit != 0,
                          out, ws, ws_bytes, stream);
}

size_t sana_linattn_state_workspace_size(const sana_shape* s, sana_dtype dt) {
  if (check_shape(s, dt, "sana_linattn_state_workspace_size") != SANA_OK) return 0;
  return linattn_state_ws_bytes(*s, dt);
}

sana_status sana_linattn_state(const sana_shape* s, sana_dtype dt, const void* k, const void* v,
                               const sana_rope* rope, float* S_out, float* z_out, void* ws,
                               size_t ws_bytes, sana_stream_t stream) {
  const char* who = "sana_linattn_state";
  if (sana_status e = check_shape(s, dt, who)) return e;
  if (sana_status e = check_rope(rope, s, who)) return e;
  if (!S_out || !z_out) return fail(SANA_ERR_INVALID_ARG, "%s: NULL state pointer", who);
  if (s->T > 0 && (!k || !v)) return fail(SANA_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
  const void* ptrs[4] = {k, v, S_out, z_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t n = (size_t)s->B * s->T * s->H * s->W * s->heads * s->head_dim * esize(dt);
  const size_t sb = (size_t)s->B * s->heads * s->head_dim * s->head_dim * 4;
  const size_t zb = (size_t)s->B * s->heads * s->head_dim * 4;
  if (overlap(S_out, sb, k, n) || overlap(S_out, sb, v, n) || overlap(z_out, zb, k, n) ||
      overlap(z_out, zb, v, n) || overlap(S_out, sb, z_out, zb))
    return fail(SANA_ERR_INVALID_ARG, "%s: outputs alias inputs", who);
  const size_t need = linattn_state_ws_bytes(*s, dt);
  if (need && (!ws || ws_bytes < need))
    return fail(SANA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws ? ws_bytes : 0, need);
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(SANA_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
  return linattn_state_run(*s, dt, k, v, to_dev(*rope), S_out, z_out, ws, ws_bytes, stream);
}

sana_status sana_linattn_apply(const sana_shape* s, sana_dtype dt, const void* q, const void* g,
                               const sana_rope* rope, const float* S, const float* z, float eps,
                               void* out, sana_stream_t stream) {
  const char* who = "sana_linattn_apply";
  if (sana_status e = check_shape(s, dt, who)) return e;
  if (sana_status e = check_rope(rope, s, who)) return e;
  if (!std::isfinite(eps) || eps < 0.f) return fail(SANA_ERR_INVALID_ARG, "%s: eps must be finite and >= 0", who);
  if (s->T == 0) return SANA_OK;
  if (!q || !S || !z || !out) return fail(SANA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  const void* ptrs[5] = {q, g, S, z, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t n = (size_t)s->B * s->T * s->H * s->W * s->heads * s->head_dim * esize(dt);
  const size_t sb = (size_t)s->B * s->heads * s->head_dim * s->head_dim * 4;
  if (overlap(out, n, q, n) || overlap(out, n, g, n) || overlap(out, n, S, sb))
    return fail(SANA_ERR_INVALID_ARG, "%s: out aliases an input", who);
  return linattn_apply_run(*s, dt, q, g, to_dev(*rope), S, z, eps, out, stream);
}

size_t sana_softmax_anchor_workspace_size(const sana_shape* s, sana_dtype dt) {
  if (check_shape(s, dt, "sana_softmax_anchor_workspace_size") != SANA_OK) return 0;
  return anchor_ws_bytes(*s, dt);
}

sana_status sana_softmax_anchor_fwd(const sana_shape* s, sana_dtype dt, const void* q,
                                    const void* k, const void* v, const void* g,
                                    const sana_rope* rope, float scale, void* out, void* ws,
                                    size_t ws_bytes, sana_stream_t stream) {
  const char* who = "sana_softmax_anchor_fwd";
  if (sana_status e = check_shape(s, dt, who)) return e;
  if (rope)
    if (sana_status e = check_rope(rope, s, who)) return e;
  if (!std::isfinite(scale)) return fail(SANA_ERR_INVALID_ARG, "%s: scale is not finite", who);
  if (s->T == 0) return SANA_OK;
  if (!q || !k || !v || !out) return fail(SANA_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
  const void* ptrs[5] = {q, k, v, g, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t n = (size_t)s->B * s->T * s->H * s->W * s->heads * s->head_dim * esize(dt);
  if (overlap(out, n, q, n) || overlap(out, n, k, n) || overlap(out, n, v, n) || overlap(out, n, g, n))
    return fail(SANA_ERR_INVALID_ARG, "%s: out aliases an input", who);
  const size_t need = anchor_ws_bytes(*s, dt);
  if (need && (!ws || ws_bytes < need))
    return fail(SANA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws ? ws_bytes : 0, need);
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(SANA_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
  RopeDev rd{};
  if (rope) rd = to_dev(*rope);
  return anchor_run(*s, dt, q, k, v, g, rope ? &rd : nullptr, scale, out, ws, ws_bytes, stream);
}

sana_status sana_rope_apply(const sana_shape* s, sana_dtype dt, const void* x,
                           const sana_rope* rope, float mul, void* out, sana_stream_t stream) {
  const char* who = "sana_rope_apply";
  if (sana_status e = check_shape(s, dt, who)) return e;
  if (rope)
    if (sana_status e = check_rope(rope, s, who)) return e;
  if (!std::isfinite(mul)) return fail(SANA_ERR_INVALID_ARG, "%s: mul is not finite", who);
  if (s->T == 0) return SANA_OK;
  if (!x || !out) return fail(SANA_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
  if (!aligned16(x) || !aligned16(out))
    return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t n = (size_t)s->B * s->T * s->H * s->W * s->heads * s->head_dim * esize(dt);
  if (overlap(out, n, x, n)) return fail(SANA_ERR_INVALID_ARG, "%s: out aliases x", who);
  RopeDev rd{};
  if (rope) rd = to_dev(*rope);
  return rope_rotate_run(x, dt == SANA_BF16, rope ? &rd : nullptr, to_grid(*s), s->B,
                         s->head_dim, mul, out, stream);
}

sana_status sana_softmax_anchor_rotated_fwd(const sana_shape* s, const void* q_rot,
                                            const void* k_rot, const void* v, const void* g,
                                            void* out, sana_stream_t stream) {
  const char* who = "sana_softmax_anchor_rotated_fwd";
  if (sana_status e = check_shape(s, SANA_BF16, who)) return e;
  if (s->T == 0) return SANA_OK;
  if (!q_rot || !k_rot || !v || !out) return fail(SANA_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
  const void* ptrs[5] = {q_rot, k_rot, v, g, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t n = (size_t)s->B * s->T * s->H * s->W * s->heads * s->head_dim * 2;
  if (overlap(out, n, q_rot, n) || overlap(out, n, k_rot, n) || overlap(out, n, v, n) ||
      overlap(out, n, g, n))
    return fail(SANA_ERR_INVALID_ARG, "%s: out aliases an input", who);
  return anchor_bf16_run(*s, q_rot, k_rot, v, g, to_grid(*s), nullptr, 0, out, stream);
}

size_t sana_softmax_anchor_sparse_workspace_size(const sana_shape* s, sana_dtype dt) {
  if (check_shape(s, dt, "sana_softmax_anchor_sparse_workspace_size") != SANA_OK ||
      dt != SANA_BF16)
    return 0;
  return anchor_sparse_ws_bytes(*s);
}

sana_status sana_softmax_anchor_sparse_fwd(const sana_shape* s, sana_dtype dt, const void* q,
                                           const void* k, const void* v, const void* g,
                                           const sana_rope* rope, float scale, int keep_tiles,
                                           int* tiles, int select_tiles, void* out, void* ws,
                                           size_t ws_bytes, sana_stream_t stream) {
  const char* who = "sana_softmax_anchor_sparse_fwd";
  if (sana_status e = check_shape(s, dt, who)) return e;
  if (dt != SANA_BF16) return fail(SANA_ERR_UNSUPPORTED, "%s: bf16 only", who);
  if (rope)
    if (sana_status e = check_rope(rope, s, who)) return e;
  if (!std::isfinite(scale)) return fail(SANA_ERR_INVALID_ARG, "%s: scale is not finite", who);
  if (s->T == 0) return SANA_OK;
  const long long N = (long long)s->T * s->H * s->W;
  const long long ntiles = (N + 127) / 128;
  if (ntiles > kAnchorMaxTiles)
    return fail(SANA_ERR_UNSUPPORTED, "%s: %lld key tiles (max %d)", who, ntiles, kAnchorMaxTiles);
  if (keep_tiles < 1 || keep_tiles > ntiles)
    return fail(SANA_ERR_INVALID_ARG, "%s: keep_tiles=%d outside [1, %lld]", who, keep_tiles, ntiles);
  if (!q || !k || !v || !out || !tiles)
    return fail(SANA_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
  const void* ptrs[6] = {q, k, v, g, out, tiles};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t n = (size_t)s->B * N * s->heads * s->head_dim * 2;
  const size_t tb = (size_t)s->B * s->heads * ((ntiles + 1) / 2) * keep_tiles * 4;
  if (overlap(out, n, q, n) || overlap(out, n, k, n) || overlap(out, n, v, n) || overlap(out, n, g, n))
    return fail(SANA_ERR_INVALID_ARG, "%s: out aliases an input", who);
  if (overlap(tiles, tb, out, n) || overlap(tiles, tb, q, n) || overlap(tiles, tb, k, n) ||
      overlap(tiles, tb, v, n) || overlap(tiles, tb, g, n))
    return fail(SANA_ERR_INVALID_ARG, "%s: tiles alias a tensor", who);
  const size_t need = anchor_sparse_ws_bytes(*s);
  if (!ws || ws_bytes < need)
    return fail(SANA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws ? ws_bytes : 0, need);
  if (reinterpret_cast<uintptr_t>(ws) & 255u)
    return fail(SANA_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
  if (overlap(ws, need, tiles, tb) || overlap(ws, need, out, n))
    return fail(SANA_ERR_INVALID_ARG, "%s: workspace aliases the output or the tiles", who);
  RopeDev rd{};
  if (rope) rd = to_dev(*rope);
  return anchor_sparse_run(*s, q, k, v, g, rope ? &rd : nullptr, scale, keep_tiles, tiles,
                           select_tiles != 0, out, ws, ws_bytes, stream);
}

sana_status sana_attnres_route(int B, long long N, int C, sana_dtype dt, const void* const* sources,
                               int num_sources, const float* w, float rms_eps, void* h_out,
                               float* alpha_out, sana_stream_t stream) {
  const char* who = "sana_attnres_route";
  if (dt != SANA_F32 && dt != SANA_BF16) return fail(SANA_ERR_INVALID_ARG, "%s: bad dtype", who);
  if (B < 1 || N < 0 || C < 1) return fail(SANA_ERR_INVALID_ARG, "%s: bad sizes", who);
  if (num_sources < 1 || num_sources > 16)
    return fail(SANA_ERR_UNSUPPORTED, "%s: num_sources=%d (1..16)", who, num_sources);
  if (N == 0) return SANA_OK;
  if (!sources || !w || !h_out) return fail(SANA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (num_sources < 1 || num_sources > 16)
    return fail(SANA_ERR_UNSUPPORTED, "%s: num_sources=%d (1..16)", who, num_sources);
  if (!std::isfinite(rms_eps) || rms_eps < 0.f) return fail(SANA_ERR_INVALID_ARG, "%s: bad rms_eps", who);
  const size_t n = (size_t)B * N * C * esize(dt);
  for (int i = 0; i < num_sources; ++i) {
    if (!sources[i] || !aligned16(sources[i]))
      return fail(SANA_ERR_INVALID_ARG, "%s: source %d is NULL or not 16-byte aligned", who, i);
    if (overlap(h_out, n, sources[i], n)) return fail(SANA_ERR_INVALID_ARG, "%s: h_out aliases source %d", who, i);
  }
  if (!aligned16(h_out) || !aligned16(w)) return fail(SANA_ERR_INVALID_ARG, "%s: h_out / w not 16-byte aligned", who);
  return attnres_run(B, N, C, dt, sources, num_sources, w, rms_eps, h_out, alpha_out, false,
                     nullptr, stream);
}

size_t sana_attnres_route_bwd_workspace_size(int B, long long N, int C) {
  if (B < 1 || N < 0 || C < 1) return 0;
  return attnres_bwd_ws_bytes((long long)B * N, C);
}

sana_status sana_attnres_route_bwd(int B, long long N, int C, sana_dtype dt,
                                   const void* const* sources, int num_sources, const float* w,
                                   float rms_eps, const void* dh, void* const* d_sources,
                                   float* dw, void* ws, size_t ws_bytes, sana_stream_t stream) {
  const char* who = "sana_attnres_route_bwd";
  if (dt != SANA_BF16) return fail(SANA_ERR_UNSUPPORTED, "%s: bf16 only", who);
  if (B < 1 || N < 0 || C < 1) return fail(SANA_ERR_INVALID_ARG, "%s: bad sizes", who);
  if (num_sources < 1 || num_sources > 4)
    return fail(SANA_ERR_UNSUPPORTED, "%s: num_sources=%d (1..4)", who, num_sources);
  if (!std::isfinite(rms_eps) || rms_eps < 0.f) return fail(SANA_ERR_INVALID_ARG, "%s: bad rms_eps", who);
  if (!w || !dw) return fail(SANA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (N == 0)  // no tokens: dw = 0, nothing else is read or written
    return attnres_bwd_run(0, C, nullptr, num_sources, w, rms_eps, nullptr, nullptr, dw, nullptr,
                           0, stream);
  if (!sources || !d_sources || !dh) return fail(SANA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  const size_t n = (size_t)B * N * C * 2;
  for (int i = 0; i < num_sources; ++i) {
    if (!sources[i] || !aligned16(sources[i]) || !d_sources[i] || !aligned16(d_sources[i]))
      return fail(SANA_ERR_INVALID_ARG, "%s: source or gradient %d is NULL or not 16-byte aligned", who, i);
    if (overlap(d_sources[i], n, dh, n)) return fail(SANA_ERR_INVALID_ARG, "%s: gradient %d aliases dh", who, i);
    for (int j = 0; j < num_sources; ++j) {
      if (overlap(d_sources[i], n, sources[j], n))
        return fail(SANA_ERR_INVALID_ARG, "%s: gradient %d aliases source %d", who, i, j);
      if (j != i && overlap(d_sources[i], n, d_sources[j], n))
        return fail(SANA_ERR_INVALID_ARG, "%s: gradients %d and %d alias", who, i, j);
    }
  }
  if (!aligned16(w) || !aligned16(dh)) return fail(SANA_ERR_INVALID_ARG, "%s: w / dh not 16-byte aligned", who);
  const size_t need = attnres_bwd_ws_bytes((long long)B * N, C);
  if (!ws || ws_bytes < need)
    return fail(SANA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws ? ws_bytes : 0, need);
  return attnres_bwd_run((long long)B * N, C, sources, num_sources, w, rms_eps, dh, d_sources, dw,
                         ws, ws_bytes, stream);
}

sana_status sana_rmsnorm(long long rows, int C, sana_dtype dt, const void* x, float eps, void* y,
                         sana_stream_t stream) {
  if (dt != SANA_F32 && dt != SANA_BF16) return fail(SANA_ERR_INVALID_ARG, "sana_rmsnorm: bad dtype");
  if (rows < 0 || C < 1 || !x || !y) return fail(SANA_ERR_INVALID_ARG, "sana_rmsnorm: bad arguments");
  if (!aligned16(x) || !aligned16(y)) return fail(SANA_ERR_INVALID_ARG, "sana_rmsnorm: pointers not 16-byte aligned");
  return rmsnorm_run(rows, C, dt, x, eps, y, stream);
}

sana_status sana_gemm_bf16(long long M, int N, int K, const void* A, long long lda, const void* W,
                           void* out, long long ldo, int epilogue, sana_stream_t stream) {
  const char* who = "sana_gemm_bf16";
  if (M < 0 || N < 1 || K < 1 || !A || !W || !out) return fail(SANA_ERR_INVALID_ARG, "%s: bad arguments", who);
  if (K % 64 != 0 || N % 8 != 0 || lda < K || ldo < N || lda % 8 || ldo % 8)
    return fail(SANA_ERR_UNSUPPORTED, "%s: needs K %% 64 == 0, N %% 8 == 0, lda >= K, ldo >= N (multiples of 8)", who);
  if (epilogue < 0 || epilogue > 2) return fail(SANA_ERR_INVALID_ARG, "%s: bad epilogue %d", who, epilogue);
  if (!aligned16(A) || !aligned16(W) || !aligned16(out)) return fail(SANA_ERR_INVALID_ARG, "%s: pointers not 16-byte aligned", who);
  return gemm_run(M, N, K, A, lda, W, out, ldo, epilogue, stream);
}

// ---------------------------------------------------------------- MX projection GEMM
size_t sana_mx_scale_bytes(long long rows, int K) {
  if (rows < 0 || K < 128 || K % 128 != 0) return 0;
  return mx_scale_bytes(rows, K);
}

sana_status sana_mx_quantize(const void* x, long long rows, int K, int fp4, void* q, void* scales,
                             sana_stream_t stream) {
  const char* who = "sana_mx_quantize";
  if (rows < 0 || K < 128 || K % 128 != 0 || (fp4 != 0 && fp4 != 1))
    return fail(SANA_ERR_INVALID_ARG, "%s: needs rows >= 0, K a positive multiple of 128, fp4 0/1",
                who);
  if (rows == 0) return SANA_OK;
  if (!x || !q || !scales) return fail(SANA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (!aligned16(x) || !aligned16(q) || !aligned16(scales))
    return fail(SANA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t nx = (size_t)rows * K * 2, nq = (size_t)rows * K / (fp4 ? 2 : 1);
  const size_t ns = mx_scale_bytes(rows, K);
  if (overlap(q, nq, x, nx) || overlap(scales, ns, x, nx) || overlap(scales, ns, q, nq))
    return fail(SANA_ERR_INVALID_ARG, "%s: buffers overlap", who);
  return mx_quantize_run(x, rows, K, fp4 != 0, q, scales, stream);
}

sana_status sana_mx_gemm(long long M, int N, int K, const void* xq, const void* x_scales,
                         const void* wq, const void* w_scales, void* out, long long ldo,
                         int epilogue, sana_stream_t stream) {
  const char* who = "sana_mx_gemm";
  if (M < 0 || N < 128 || N % 128 != 0 || K < 128 || K % 128 != 0)
    return fail(SANA_ERR_UNSUPPORTED, "%s: needs N and K positive multiples of 128 (N=%d K=%d)",
                who, N, K);
  if (ldo < N || ldo % 8 != 0) return fail(SANA_ERR_INVALID_ARG, "%s: ldo must be >= N and a multiple of 8", who);
  if (epilogue < 0 || epilogue > 2) return fail(SANA_ERR_INVALID_ARG, "%s: bad epilogue %d", who, epilogue);
  if (M == 0) return SANA_OK;
  if (!xq || !x_scales || !wq || !w_scales || !out)
    return fail(SANA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (!aligned16(xq) || !aligned16(x_scales) || !aligned16(w_scales) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(wq) & 31u))
    return fail(SANA_ERR_INVALID_ARG,
                "%s: pointers must be 16-byte aligned (the E2M1 weights 32-byte aligned)", who);
  const size_t no = (size_t)M * ldo * 2;
  if (overlap(out, no, xq, (size_t)M * K) || overlap(out, no, wq, (size_t)N * K / 2) ||
      overlap(out, no, x_scales, mx_scale_bytes(M, K)) ||
      overlap(out, no, w_scales, mx_scale_bytes(N, K)))
    return fail(SANA_ERR_INVALID_ARG, "%s: out aliases an operand", who);
  return mx_gemm_run(M, N, K, xq, x_scales, wq, w_scales, out, ldo, epilogue, stream);
}

size_t sana_mx_linear_workspace_size(long long M, int K) {
  if (M < 0 || K < 128 || K % 128 != 0) return 0;
  return align_up((size_t)M * K, 256) + align_up(mx_scale_bytes(M, K), 256);
}

sana_status sana_mx_linear(long long M, int N, int K, const void* x, const void* wq,
                           const void* w_scales, void* out, long long ldo, int epilogue, void* ws,
                           size_t ws_bytes, sana_stream_t stream) {
  const char* who = "sana_mx_linear";
  if (M < 0 || N < 128 || N % 128 != 0 || K < 128 || K % 128 != 0)
    return fail(SANA_ERR_UNSUPPORTED, "%s: needs N and K positive multiples of 128 (N=%d K=%d)",
                who, N, K);
  if (M == 0) return SANA_OK;
  const size_t need = sana_mx_linear_workspace_size(M, K);
  if (!ws || ws_bytes < need)
    return fail(SANA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", who, ws ? ws_bytes : 0, need);
  if (reinterpret_cast<uintptr_t>(ws) & 255u)
    return fail(SANA_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
  if (out && overlap(ws, need, out, (size_t)M * ldo * 2))
    return fail(SANA_ERR_INVALID_ARG, "%s: workspace aliases the output", who);
  char* xq = static_cast<char*>(ws);
  char* xs = xq + align_up((size_t)M * K, 256);
  if (sana_status e = sana_mx_quantize(x, M, K, 0, xq, xs, stream)) return e;
  return sana_mx_gemm(M, N, K, xq, xs, wq, w_scales, out, ldo, epilogue, stream);
}

sana_status sana_selftest_bounded_wait(unsigned int limit_ms, sana_stream_t stream) {
  if (limit_ms == 0 || limit_ms > 2000)
    return fail(SANA_ERR_INVALID_ARG, "sana_selftest_bounded_wait: limit_ms must be in 1..2000");
  int* sw = status_word();
  if (!sw) return fail(SANA_ERR_CUDA, "sana_selftest_bounded_wait: no status word on this device");
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(sw, 1000000ull * limit_ms);
  return check_launch("bounded_wait_selftest_kernel");
}

sana_status sana_sync_status(sana_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(SANA_ERR_CUDA, "sana_sync_status: %s", cudaGetErrorString(e));
  int* sw = status_word();
  if (!sw) return fail(SANA_ERR_CUDA, "sana_sync_status: no status word on this device");
  int v = 0;
  e = cudaMemcpy(&v, sw, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(SANA_ERR_CUDA, "sana_sync_status: %s", cudaGetErrorString(e));
  if (v != 0) {
    const int zero = 0;
    cudaMemcpy(sw, &zero, sizeof(int), cudaMemcpyHostToDevice);
    return fail(SANA_ERR_TIMEOUT, "a kernel gave up a bounded wait (code 0x%x)", v);
  }
  return SANA_OK;
}

}  // extern "C"
