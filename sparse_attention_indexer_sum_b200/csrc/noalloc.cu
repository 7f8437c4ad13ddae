// noalloc.cu -- ic_sparse_attn_noalloc: the absorbed-MLA sparse attention with
// its split-KV scratch held in a fixed device array of this library instead of
// a caller-supplied workspace, for callers that cannot allocate device memory.
//
// The scratch is the partial output and softmax state that the split form writes
// before its merge kernel combines them: per piece of a query, 16 heads x (512
// output floats + running max + running sum).  The entry point accepts at most
// IC_NOALLOC_MAX_QUERIES queries (batch * rows).  The split plan cuts their
// (query, 32-key tile) pairs into one contiguous range per SM, so a call makes at
// most SMs + 2 x queries pieces (276 on a 148-SM B200); the array holds
// IC_NOALLOC_MAX_QUERIES x 8 pieces and a call that would need more is refused.
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
static void* g_noalloc_ptr[kNoallocMaxDevices];

// Device address of the scratch array on the calling thread's current device;
// looked up on the first call for that device and cached.
static ic_status noalloc_scratch(void** out) {
  int dev = -1;
  ic_status st = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st) return st;
  if (dev < 0 || dev >= kNoallocMaxDevices)
    return fail(IC_ERR_UNSUPPORTED, "sparse_attn_noalloc: device ordinal %d above %d", dev,
                kNoallocMaxDevices - 1);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    st = cuda_check(cudaGetSymbolAddress(&p, g_attn_noalloc_scratch),
                    "cudaGetSymbolAddress(sparse_attn_noalloc scratch)");
    if (st) return st;
    if (!p) return fail(IC_ERR_CUDA, "sparse_attn_noalloc: scratch symbol has no address");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
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
                         IC_NOALLOC_SCRATCH_BYTES, -1, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
