// noalloc.cu -- ic_sparse_attn_noalloc: the absorbed-MLA sparse attention with
// its split-KV scratch held in a fixed device array of this library instead of
// a caller-supplied workspace, for callers that cannot allocate device memory.
//
// The scratch is the partial output and softmax state that the split form writes
// before its merge kernel combines them: per piece of a query, 16 heads x (512
// output floats + running max + running sum).  The entry point accepts at most
// IC_NOALLOC_MAX_QUERIES queries (batch * rows).  The split plan cuts their
// (query, 32-key tile) pairs into G <= SMs equal contiguous ranges, so one query
// spans at most ceil(G / queries) + 1 pieces, and every query gets that many
// slots (maxp): queries * maxp <= G + 2 * queries, at most 276 slots on a 148-SM
// B200.  The array holds IC_NOALLOC_MAX_QUERIES x 8 = 512 slots; the exact need
// (attn_mla_ws_bytes) is checked on every call and a larger one is refused with
// IC_ERR_WORKSPACE, which only a part with far more SMs could reach.
#include <cudaTypedefs.h>

#include <mutex>

#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

static_assert(IC_NOALLOC_SCRATCH_BYTES ==
                  static_cast<size_t>(IC_NOALLOC_MAX_QUERIES) * 8 * 16 * (512 + 2) * sizeof(float),
              "scratch sized for the largest accepted call");

// Held on every device that loads this library, from module load until exit.
// In host code this name is a stand-in for the symbol, not a device address:
// the address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) float g_attn_noalloc_scratch[IC_NOALLOC_SCRATCH_BYTES / 4];

constexpr int kNoallocMaxDevices = 64;
static std::mutex g_noalloc_mu;
struct NoallocSlot {
  unsigned long long ctx_id;  // context the address belongs to (0 = none yet)
  void* ptr;
};
static NoallocSlot g_noalloc_slot[kNoallocMaxDevices];

// Unique id of the calling thread's current context, or 0 if it has none.  A
// device reset ends the context and the next one gets a new id, with the module
// (and so the array) loaded again, possibly at another address.
static unsigned long long current_ctx_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_cur || !get_id) return 0;
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array in the calling thread's current context.
// It is looked up (cudaGetSymbolAddress, with the device current) on the first
// call in a context and cached with that context's id; a call from a later
// context (after a device reset, say) looks it up again.
static ic_status noalloc_scratch(void** out) {
  int dev = -1;
  ic_status st = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st) return st;
  if (dev < 0 || dev >= kNoallocMaxDevices)
    return fail(IC_ERR_UNSUPPORTED, "sparse_attn_noalloc: device ordinal %d above %d", dev,
                kNoallocMaxDevices - 1);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc_slot[dev];
  const unsigned long long id = current_ctx_id();
  if (!slot.ptr || id == 0 || id != slot.ctx_id) {
    void* p = nullptr;
    st = cuda_check(cudaGetSymbolAddress(&p, g_attn_noalloc_scratch),
                    "cudaGetSymbolAddress(sparse_attn_noalloc scratch)");
    if (st) return st;
    if (!p) return fail(IC_ERR_CUDA, "sparse_attn_noalloc: scratch symbol has no address");
    slot.ptr = p;
    slot.ctx_id = current_ctx_id();  // the lookup above made the context current if needed
  }
  *out = slot.ptr;
  return IC_OK;
}

}  // namespace ic

extern "C" {

ic_status ic_sparse_attn_noalloc(const void* q, const void* kv, long ld_kv, const void* v,
                                 const int* idx, ic_dtype dt, int batch, int rows, int heads,
                                 int dk, int dv, int Lkv, int k, float scale, void* out,
                                 float* lse, void* stream) {
  using namespace ic;
  if (v)
    return fail(IC_ERR_UNSUPPORTED,
                "sparse_attn_noalloc: only the absorbed MLA form (v = NULL); the MQA form uses "
                "no scratch, call ic_sparse_attn");
  ic_status st = check_attn(q, kv, ld_kv, v, idx, dt, batch, rows, heads, dk, dv, Lkv, k, out);
  if (st) return st;
  const long queries = static_cast<long>(batch) * rows;
  if (queries > IC_NOALLOC_MAX_QUERIES)
    return fail(IC_ERR_UNSUPPORTED,
                "sparse_attn_noalloc: %ld queries (batch * rows) above the fixed scratch's "
                "maximum of %d; call ic_sparse_attn with a workspace",
                queries, IC_NOALLOC_MAX_QUERIES);
  if (queries == 0) return IC_OK;
  const size_t need = attn_mla_ws_bytes(batch, rows, k);
  if (need > IC_NOALLOC_SCRATCH_BYTES)
    return fail(IC_ERR_WORKSPACE,
                "sparse_attn_noalloc: needs %zu bytes of split scratch, above the fixed %zu",
                need, static_cast<size_t>(IC_NOALLOC_SCRATCH_BYTES));
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st) return st;
  // Every split item writes its whole partial before the merge reads it, so the
  // previous call's contents need no clearing.
  return launch_attn_mla(q, kv, ld_kv, idx, batch, rows, Lkv, k, scale, out, lse, scratch,
                         IC_NOALLOC_SCRATCH_BYTES, -1, static_cast<cudaStream_t>(stream),
                         dt == IC_E4M3);
}

}  // extern "C"
