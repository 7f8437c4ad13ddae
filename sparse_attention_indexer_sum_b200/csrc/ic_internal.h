// ic_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/ic.h"

namespace ic {

// Launches `kernel` with programmatic stream serialization (the kernel calls
// grid_dep_wait() before it touches global memory) and, for cluster > 1, in
// clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_dep(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Records a formatted message for ic_last_error() and returns `code`.
ic_status fail(ic_status code, const char* fmt, ...);
// Checks a CUDA runtime result; on failure records it and returns IC_ERR_CUDA.
ic_status cuda_check(cudaError_t e, const char* what);
int num_sms();

// Launch kinds reported by the tracing hook (ic_trace_begin / ic_trace_end).
enum LaunchKind : int {
  kKindIndexerBf16 = 1,
  kKindIndexerE4m3 = 2,
  kKindIndexerF32 = 3,
  kKindFillMasked = 4,
  kKindTopk = 5,
  kKindAttnMla = 6,
  kKindAttnCombine = 7,
  kKindAttnF32 = 8,
  kKindQuant = 9,
  kKindTopkMerge = 10,
  kKindIndexerTopkBf16 = 11,
  kKindIndexerTopkE4m3 = 12,
  kKindAttnMlaKv8 = 13,
  kKindPackKv = 14,
  kKindFillValid = 15,
};
// Called after every kernel launch: when tracing is on for this host thread,
// records an event on `stream` with the launch's kind and algorithmic work
// (flops for the indexer, bytes for the memory-bound kernels).
void trace_launch(int kind, cudaStream_t stream, double work);
// Number of (query, key) pairs with key < Lk and key <= pos0 + r over rows r < R.
long long causal_pairs(long R, long Lk, long pos0);

// Indexer on tensor cores (H = 64, D = 128).  fp8 = e4m3 inputs with scales.
// Packed sequences of different lengths: at most IC_MAXSEG per launch.  An
// indexer segment is described beside IdxTcArgs (indexer_tc.cu); an attention
// segment's query rows q0.. (up to the next segment's q0) attend over latent rows
// k0 .. k0 + len - 1, which their index lists address as 0 .. len - 1.
constexpr int IC_MAXSEG = 64;
struct IdxSeg {
  long qrow0, krow0, orow0, pos0;
  int R, Lk, qb0, pad;
};
struct AttnSeg {
  long q0, k0;
  int len, pad;
};
// The multi-token tensor-core indexer over nseg packed segments in one launch
// (q_rows, k_rows: rows of the packed query and key tensors).
ic_status launch_indexer_tc_segs(bool fp8, const void* q, const float* q_scale, const void* k,
                                 const float* k_scale, const float* w, const IdxSeg* segs,
                                 int nseg, long q_rows, long k_rows, float* scores, long ld,
                                 cudaStream_t stream);
// The fp32 indexer over packed segments: launch row r is row r of q and w and of
// scores; the segments' orow0 / pos0 / krow0 / Lk place it (qrow0 is unused).
ic_status launch_indexer_f32_segs(const float* q, const float* k, const float* w, int H, int D,
                                  const IdxSeg* segs, int nseg, long rows, float* scores, long ld,
                                  cudaStream_t stream);
// valid_len[r] of the rows of a block of packed segments (their positions + 1).
ic_status launch_fill_valid_len(const IdxSeg* segs, int nseg, long rows, int* out,
                                cudaStream_t stream);
ic_status launch_indexer_tc(bool fp8, const void* q, const float* q_scale, const void* k,
                            const float* k_scale, const float* w, int batch, int rows, int Lk,
                            long pos0, float* scores, long ld, bool fill_tail,
                            cudaStream_t stream);
// Indexer on CUDA cores for fp32 inputs (small H, D).
ic_status launch_indexer_f32(const float* q, const float* k, const float* w, int batch, int H,
                             int D, int rows, int Lk, long pos0, float* scores, long ld,
                             cudaStream_t stream);
// Fused indexer -> top-k for batch sequences of one query each (at position pos0,
// keys 0..Lk-1): the indexer kernel keeps each row's candidates in workspace slots
// (never writing the scores), then topk_merge_kernel writes idx [batch, topk].
ic_status launch_indexer_topk_fused(bool fp8, const void* q, const float* q_scale, const void* k,
                                    const float* k_scale, const float* w, int batch, int Lk,
                                    long pos0, int topk, int* idx, void* ws, size_t ws_bytes,
                                    cudaStream_t stream);
size_t indexer_topk_fused_ws_bytes(int batch, int Lk, long pos0);
ic_status launch_topk_merge(const uint8_t* slots, long rows, long nt, long total, int G, int maxp,
                            size_t slot_bytes, int cb, int nv, int k, int* idx,
                            cudaStream_t stream);
// valid_len (device int32 [rows], or NULL): row r's candidate count, clamped to
// [0, n]; NULL means min(n, pos0 + r + 1), or n when pos0 < 0.
ic_status launch_topk(const float* scores, long rows, int n, long ld, long pos0, int k, int* idx,
                      cudaStream_t stream, const int* valid_len = nullptr);
// valid_entries: number of index entries >= 0 over all rows if the caller knows
// it (the causal stack does), else -1 (rows * k is assumed for tracing only).
// kv8: kv holds fp8 latent rows (KV8_ROW_BYTES, ld_kv in bytes), else bf16 rows
// (ld_kv in elements).
// segs (nseg <= IC_MAXSEG, host array): packed sequences, with batch = 1 and rows =
// all their query rows; Lkv is then ignored.
ic_status launch_attn_mla(const void* q, const void* kv, long ld_kv, const int* idx, int batch,
                          int rows, int Lkv, int k, float scale, void* out, float* lse,
                          void* ws, size_t ws_bytes, long long valid_entries, cudaStream_t stream,
                          bool kv8 = false, const AttnSeg* segs = nullptr, int nseg = 0);
size_t attn_mla_ws_bytes(int batch, int rows, int k);
// segs: as launch_attn_mla's.
ic_status launch_attn_f32(const float* q, const float* kv, long ld_kv, const float* v,
                          const int* idx, int batch, int rows, int heads, int dk, int dv,
                          int Lkv, int k, float scale, float* out, float* lse,
                          cudaStream_t stream, const AttnSeg* segs = nullptr, int nseg = 0);
ic_status launch_quant_e4m3(const void* x, bool bf16, long rows, int n, uint8_t* codes,
                            float* scales, cudaStream_t stream);
// fp8 latent-KV cache rows (656 bytes: 512 e4m3 codes, 4 fp32 group scales, 64 bf16
// rope dims) of bf16 latent rows [rows, ld_kv >= 576].
constexpr int KV8_ROW_BYTES = 656;
ic_status launch_pack_kv_e4m3(const void* kv, long rows, long ld_kv, uint8_t* out, long ld_out,
                              cudaStream_t stream);

}  // namespace ic
