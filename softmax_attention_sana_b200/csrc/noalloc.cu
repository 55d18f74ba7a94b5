// Allocation-free variant of sana_linattn_fwd.
//
// Some callers cannot allocate device memory at all: runtimes whose device
// memory is owned and pre-partitioned by a framework they do not control,
// plugins that may only use buffers they are handed, or code paths where a
// cudaMalloc would synchronise the device at the wrong moment.  For them this
// entry point takes its scratch space (the split partial sums of the state and
// the combined state) from one file-scope device array instead of a
// caller-provided workspace.  It allocates nothing: no cudaMalloc, no
// cudaFree, no allocating library call.
//
// The array is kNoAllocScratchBytes (16 MiB) on every GPU that loads the
// library and stays resident until the process exits.  Every call shares it,
// so calls whose kernels overlap on the GPU (other streams, other host
// threads) race on it.  The kernels fully overwrite the parts they read, so
// nothing needs clearing between calls.  The first call on a device (and the
// first after a device reset) looks up the array's device address with
// cudaGetSymbolAddress; make that first call before any stream capture.
//
// Under lazy module loading (the CUDA 12 default) the library's device code,
// and with it this array, is loaded onto a device by the first library call
// made there, and that load may synchronise the device.  Callers for whom this
// matters should make one call at initialisation time.
#include <mutex>

#include "sana_common.cuh"
#include "sana_internal.h"

namespace sana {
namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress with that device current.  It is looked up once per
// device and context: after a device reset the device gets a new context in
// which the array may sit elsewhere, and a changed context id forces a new
// lookup.  The mutex makes first calls from several host threads safe.
void* scratch_ptr(sana_status* st) {
  struct Slot {
    unsigned long long ctx;
    void* addr;
  };
  static Slot slots[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *st = fail(SANA_ERR_CUDA, "sana_linattn_fwd_noalloc: no current device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (ctx == 0 || slots[dev].ctx != ctx || !slots[dev].addr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      *st = fail(SANA_ERR_CUDA, "sana_linattn_fwd_noalloc: cudaGetSymbolAddress: %s",
                 cudaGetErrorString(e));
      return nullptr;
    }
    // the lookup makes the primary context current when none was
    slots[dev] = Slot{current_context_id(), p};
  }
  *st = SANA_OK;
  return slots[dev].addr;
}

}  // namespace
}  // namespace sana

using namespace sana;

extern "C" size_t sana_linattn_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" sana_status sana_linattn_fwd_noalloc(const sana_shape* s, sana_dtype dt, const void* q,
                                                const void* k, const void* v,
                                                const void* gate_logits, const sana_rope* rope,
                                                float eps, void* out, sana_stream_t stream) {
  // 0 for a shape sana_linattn_fwd rejects; it then reports the error itself
  const size_t need = s ? sana_linattn_workspace_size(s, dt) : 0;
  if (need > kNoAllocScratchBytes)
    return fail(SANA_ERR_UNSUPPORTED,
                "sana_linattn_fwd_noalloc: this shape needs %zu bytes of scratch, more than the "
                "built-in %zu; use sana_linattn_fwd with a caller workspace",
                need, kNoAllocScratchBytes);
  sana_status st = SANA_OK;
  void* ws = scratch_ptr(&st);
  if (!ws) return st;
  return sana_linattn_fwd(s, dt, q, k, v, gate_logits, rope, eps, out, ws, kNoAllocScratchBytes,
                          stream);
}
