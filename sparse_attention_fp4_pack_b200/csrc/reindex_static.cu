// csa2_reindex_static: the Reindex call with its key scratch in a fixed device array
// compiled into the library, so the caller hands over no scratch memory at all.
//
// Who needs it: a host that has no device allocator of its own to draw scratch from (a
// plain C program driving the library next to a framework that owns all device memory),
// or an engine whose device memory is planned once before decoding starts and which
// must not ask for more inside the decode loop.  Such callers cannot supply the
// workspace that csa2_reindex takes.
//
// How: g_reindex_scratch below is a file-scope __device__ array of
// CSA2_STATIC_SCRATCH_BYTES.  Every GPU on which the library's device code is loaded
// holds that array until the process exits.  In host code the array's name is only a
// host-side stand-in, so the call looks up its device address with cudaGetSymbolAddress,
// with the device current, the first time it runs in a device context, and caches it
// keyed by the device and the context's unique id.  A context that is destroyed and
// created again (cudaDeviceReset) gets a new id, so the next call looks the address up
// again instead of reusing a stale one.  This set-up runs inside the call, so the first
// call on each device (and the first after a reset) should come before any stream
// capture.  The call then runs csa2_reindex unchanged with the array as its workspace.
// Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library routine.
//
// The scratch holds the per-candidate keys that the Reindex scan writes and the Top-K
// selection reads back; the scan writes every key the selection reads, so nothing in
// the array has to start at zero.  There is one array per device: two calls whose
// kernels overlap on the same device (two streams, or two host threads) race on it
// and their results are undefined.  Serialise the calls (one stream) on each device.
#include <cuda.h>

#include <mutex>

#include "csa2_device.cuh"

namespace {

static __device__ __align__(256) uint8_t g_reindex_scratch[CSA2_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchSlot {
  unsigned long long ctx_id;  // unique id of the context the address belongs to (0: none)
  void* addr;                 // device address of the array in that context
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// Driver entry points for the current context's unique id, fetched through the runtime
// (so the library needs no link against the driver library).  Null when unavailable.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
std::once_flag g_driver_once;

void load_driver_entry_points() {
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f);
  f = nullptr;
  if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f);
  cudaGetLastError();
}

// Unique id of the current context, or 0 if there is none yet or the driver cannot say.
unsigned long long current_ctx_id() {
  std::call_once(g_driver_once, load_driver_entry_points);
  if (!g_ctx_get_current || !g_ctx_get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (g_ctx_get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the array in the current device's current context.
csa2_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return CSA2_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return CSA2_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long id = current_ctx_id();
  ScratchSlot& slot = g_scratch[dev];
  if (id == 0 || slot.ctx_id != id || !slot.addr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_reindex_scratch) != cudaSuccess || !p) {
      cudaGetLastError();  // clear the error so a later launch check does not report it
      return CSA2_ERR_CUDA;
    }
    // the lookup makes the context current if the runtime had not yet; take its id now
    slot.ctx_id = id != 0 ? id : current_ctx_id();
    slot.addr = p;
  }
  *out = slot.addr;
  return CSA2_OK;
}

}  // namespace

extern "C" size_t csa2_static_scratch_bytes(void) { return CSA2_STATIC_SCRATCH_BYTES; }

extern "C" csa2_status csa2_reindex_static(const float* q, const float* w, const uint8_t* ik_pool,
                                           int64_t pool_entries, const int64_t* seq_base,
                                           const int32_t* n_vis, const int32_t* blocks, int n_blocks,
                                           int block, int B, int Q, int HI, int K, int32_t* topk,
                                           float* topk_score, uint32_t* dev_status, cudaStream_t stream) {
  // the size check comes first and touches no device state
  const size_t need = csa2_reindex_workspace_size(B, Q, HI, n_blocks, block, K);
  if (need > (size_t)CSA2_STATIC_SCRATCH_BYTES) return CSA2_ERR_UNSUPPORTED;
  if ((int64_t)B * Q <= 0 || need == 0)  // nothing to scan, or arguments csa2_reindex rejects
    return csa2_reindex(q, w, ik_pool, pool_entries, seq_base, n_vis, blocks, n_blocks, block, B, Q, HI, K,
                        topk, topk_score, nullptr, 0, dev_status, stream);
  void* ws = nullptr;
  const csa2_status st = scratch_on_current_device(&ws);
  if (st != CSA2_OK) return st;
  return csa2_reindex(q, w, ik_pool, pool_entries, seq_base, n_vis, blocks, n_blocks, block, B, Q, HI, K, topk,
                      topk_score, ws, (size_t)CSA2_STATIC_SCRATCH_BYTES, dev_status, stream);
}
