/*
 * ic.h -- C ABI of libic_b200.so: the hot path of DeepSeek Sparse Attention
 * with IndexCache (lightning indexer -> per-row top-k -> sparse attention, and
 * the F/S layer stack that shares the index set), hand-written for sm_100a.
 *
 * Sources.  "IndexCache: Wie DeepSeek O(NL^2)-Kosten in Sparse Attention um
 * 75% reduziert" (itoverdose.com): the intro (k = 2048 positions per query;
 * attention cost O(Lk)), the second paragraph (the indexer scores all previous
 * tokens), the F/S list and the rule that the first layer is F, the routing loop of
 * "Einfache Implementierung, enorme Effizienzgewinne" (I <- Indexer(X);
 * T <- top-k(I); T_cache <- T / T <- T_cache; X <- SparseAttn(X, T)), the
 * T_cache paragraph right after it (one buffer, overwritten by every F layer,
 * no extra memory), "Wie der Indexer funktioniert" (score, ReLU gate, top-k)
 * and the MLA paragraph (one latent vector shared by all heads).  The
 * parapluman.nl article, "Aandacht cachen met IndexCache": an S layer reuses
 * the indices of the nearest preceding F layer.
 *
 * Conventions for every entry point:
 *  - Pointers named in the argument lists are DEVICE pointers unless marked
 *    "host".  The caller owns every buffer; the library never allocates device
 *    memory and keeps no state besides a thread-local error message and one
 *    device error word.
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and the call returns without synchronising.  The kernels are
 *    launched with programmatic dependent launch: each may be scheduled while
 *    the previous kernel of the stream drains, and each waits for it
 *    (griddepcontrol.wait) before touching global memory.  None signals its
 *    dependents early, so stream order is unchanged for whatever the caller
 *    enqueues before or after.  ic_decode_step is captured in a CUDA graph and
 *    replayed in the tests; this note says nothing about the other calls.
 *  - Tensors are dense, row-major, with the layouts given per function.
 *  - Errors are returned as negative ic_status codes; arguments are checked
 *    before anything is launched, so a failed call has launched nothing.
 *    ic_last_error() describes the last failure of the calling thread.
 *  - Kernels never trap: a device-side wait that runs out of time (2 s)
 *    records a code in the device error word, abandons its work and returns;
 *    ic_device_status() reports it (IC_ERR_TIMEOUT).
 *  - libic_b200_debug.so, the same library built with -DIC_DEBUG_BOUNDS, also
 *    checks the indices its kernels compute (index-list entries against their
 *    cache, TMA tile coordinates, top-k and merge output slots) before using
 *    them; a failed check skips the access and ic_device_status() reports
 *    IC_ERR_BOUNDS.  (Index-list entries outside the cache are skipped in every
 *    build; only the debug build reports them.)
 */
#ifndef IC_H_
#define IC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int ic_status;
#define IC_OK 0
#define IC_ERR_INVALID_ARG (-1) /* bad pointer, size, layout or pattern        */
#define IC_ERR_UNSUPPORTED (-2) /* valid request this build does not implement */
#define IC_ERR_WORKSPACE (-3)   /* workspace missing or too small              */
#define IC_ERR_CUDA (-4)        /* a CUDA runtime/driver call failed           */
#define IC_ERR_TIMEOUT (-5)     /* a device-side bounded wait gave up          */
#define IC_ERR_BOUNDS (-6)      /* a debug-bounds build caught an index out of range */

typedef enum { IC_F32 = 0, IC_BF16 = 1, IC_E4M3 = 2 } ic_dtype;

/* Message of the last failed call on this host thread ("" if none). */
const char* ic_last_error(void);

/* Library ABI version (major * 100 + minor). */
int ic_version(void);

/* Synchronise `stream`, then read and clear the device error word.
 * Returns IC_OK, IC_ERR_TIMEOUT (a bounded device wait gave up since the last
 * check), IC_ERR_BOUNDS (debug-bounds build: an index check failed) or
 * IC_ERR_CUDA. */
ic_status ic_device_status(void* stream);

/*
 * Launch tracing, for timing each kernel on the device.  ic_trace_begin records
 * a start event on `stream`; from then on, every kernel this library launches
 * from the calling host thread is followed by an event record on its stream
 * (all calls must use that same stream for the intervals to be meaningful).
 * ic_trace_end waits for the last event and fills, for launch i (i < capacity):
 *   ms[i]    device time from the previous event to this launch's event (ms),
 *   kinds[i] IC_K_* of the launch,
 *   work[i]  its algorithmic work: flops for the indexer, bytes for the
 *            memory-bound kernels (each input byte read once, output written once).
 * Any of ms/kinds/work may be NULL.  Returns the number of launches made while
 * recording (launches beyond `capacity` are counted but not timed), or a
 * negative ic_status.  The library creates its events once and keeps them.
 */
#define IC_K_INDEXER_BF16 1
#define IC_K_INDEXER_E4M3 2
#define IC_K_INDEXER_F32 3
#define IC_K_FILL_MASKED 4
#define IC_K_TOPK 5
#define IC_K_ATTN_MLA 6
#define IC_K_ATTN_COMBINE 7
#define IC_K_ATTN_F32 8
#define IC_K_QUANT 9
#define IC_K_TOPK_MERGE 10
#define IC_K_INDEXER_TOPK_BF16 11
#define IC_K_INDEXER_TOPK_E4M3 12
#define IC_K_ATTN_MLA_KV8 13
#define IC_K_PACK_KV 14
#define IC_K_FILL_VALID 15
ic_status ic_trace_begin(void* stream, int capacity);
long ic_trace_end(float* ms, int* kinds, double* work, int capacity);

/*
 * Per-row e4m3 quantisation (the fp8 variant of the indexer inputs, one fp32
 * scale per token; OCP 8-bit floating point, E4M3).  For each row of n values:
 * scale = amax / 448 (1 for an all-zero row), code = E4M3_rne_satfinite(x / scale),
 * computed in fp32.
 *   x      [rows, n] of x_dtype (IC_BF16 or IC_F32)
 *   codes  [rows, n] uint8 (e4m3 bit patterns)
 *   scales [rows] float
 * n must be a multiple of 8 and <= 1024.
 */
ic_status ic_quant_e4m3_rows(const void* x, ic_dtype x_dtype, long rows, int n, uint8_t* codes,
                             float* scales, void* stream);

/*
 * Lightning-indexer scores ("Wie der Indexer funktioniert": a score per
 * previous position, a ReLU gate, then top-k; the weighted head sum is this
 * library's reading of that passage):
 *   I[b, r, s] = sum_h w[b, r, h] * max(0, q[b, r, h, :] . k[b, s, :])
 * for every key s <= pos0 + r (query row r sits at position pos0 + r), and
 * I[b, r, s] = -inf for s > pos0 + r (not a candidate).
 *   q       [batch, rows, H, D]  dt (IC_BF16 / IC_E4M3 codes / IC_F32)
 *   q_scale [batch, rows, H] f32 (IC_E4M3 only; NULL otherwise): q = code * q_scale
 *   k       [batch, Lk, D]       dt
 *   k_scale [batch, Lk] f32      (IC_E4M3 only; NULL otherwise): k = code * k_scale
 *   w       [batch, rows, H] f32 head weights
 *   scores  [batch, rows, ld] f32 output, ld >= Lk; columns [0, Lk) are written
 * IC_BF16 and IC_E4M3 run on the tensor cores and need H = 64, D = 128 (fp32
 * accumulation); IC_F32 runs on the CUDA cores for any H <= 64, D <= 256.
 * pos0 >= 0.  Scores are fp32; the fp8 scales are folded in after the dot products.
 */
ic_status ic_indexer_scores(const void* q, const float* q_scale, const void* k,
                            const float* k_scale, const float* w, ic_dtype dt, int batch, int H,
                            int D, int rows, int Lk, long pos0, float* scores, long ld,
                            void* stream);

/*
 * Exact per-row top-k (routing loop: T <- top-k(I); k = 2048 in the pages).
 * Row r's candidates are columns s < valid(r), where valid(r) = n when
 * pos0 < 0, else min(n, pos0 + r + 1) (causal rows).  Output idx[r, 0..k):
 * the min(k, valid(r)) candidates with the largest scores -- ties go to the
 * lower index and -0 == +0 -- in ascending index order, padded with -1.
 *   scores [rows, ld] f32 (finite on the candidate columns), ld >= n
 *   idx    [rows, k] int32
 * 1 <= k <= 2048.  Bit-exact: the selection is a pure function of the fp32 values.
 */
ic_status ic_topk(const float* scores, long rows, int n, long ld, long pos0, int k, int* idx,
                  void* stream);

/*
 * The indexer and the top-k in one pass, for one query per sequence (the decode
 * shape; routing loop: I <- Indexer(X); T <- top-k(I)).  For sequence b, with
 * the query at position pos0 and the candidates s <= pos0, s < Lk:
 *   idx[b, :] = ic_topk of the scores ic_indexer_scores would write for it
 * -- the same fp32 scores and the same selection rule, so the index sets are
 * identical -- but the scores are never written to memory.  The indexer's
 * epilogue keeps, per group of keys, every key that can still be among the k
 * largest (an exact rising threshold), leaves those candidates in `workspace`,
 * and a second kernel selects the k largest of each sequence.
 *   q [batch, 1, H, D], q_scale [batch, 1, H], k [batch, Lk, D], k_scale [batch, Lk],
 *   w [batch, 1, H]: as ic_indexer_scores with rows = 1; dt = IC_BF16 or IC_E4M3
 *   (H = 64, D = 128);
 *   idx [batch, k_top] int32 out: ascending, -1 padded when pos0 + 1 < k_top;
 *   workspace: device, 16-byte aligned, >= ic_indexer_topk_workspace_size bytes
 *   (IC_ERR_WORKSPACE otherwise); its contents need no initialisation.
 * 1 <= k_top <= 2048.  IC_F32 -> IC_ERR_UNSUPPORTED.
 */
ic_status ic_indexer_topk(const void* q, const float* q_scale, const void* k,
                          const float* k_scale, const float* w, ic_dtype dt, int batch, int H,
                          int D, int Lk, long pos0, int k_top, int* idx, void* workspace,
                          size_t ws_bytes, void* stream);
size_t ic_indexer_topk_workspace_size(int batch, int Lk, long pos0);

/*
 * ic_topk with an arbitrary candidate count per row: row r's candidates are
 * columns s < valid_len[r] (clamped to [0, n]).  Rows of different sequences
 * packed into one call, or rows with their own causal offsets, use this form.
 *   valid_len [rows] int32, device
 * Other arguments, the output and the errors as ic_topk.
 */
ic_status ic_topk_varlen(const float* scores, long rows, int n, long ld, const int* valid_len,
                         int k, int* idx, void* stream);

/*
 * The fp8 latent-KV cache (a serving-side variant of the MLA cache: the same
 * latent rows, about 57% of the bytes to gather).  Row r of kv [rows, ld_kv]
 * bf16 (576 dims: 512 latent + 64 rope) becomes 656 bytes at out + r * ld_out:
 *   bytes   0..511  the 512 latent dims as OCP E4M3 codes, in four groups of 128;
 *                   group g: scale_g = amax_g / 448 (1 if all zero),
 *                   code = E4M3_rne_satfinite(x / scale_g), in fp32 (the same
 *                   arithmetic as ic_quant_e4m3_rows on each 128-dim group)
 *   bytes 512..527  scale_0..scale_3, fp32
 *   bytes 528..655  the 64 rope dims, bf16, unchanged
 * ld_kv >= 576 (elements, a multiple of 8); ld_out >= 656 (bytes, a multiple of
 * 16); both tensors 16-byte aligned.
 */
ic_status ic_pack_kv_e4m3(const void* kv, long rows, long ld_kv, uint8_t* out, long ld_out,
                          void* stream);

/*
 * Sparse attention of each query over its index set (routing loop:
 * X <- SparseAttn(X, T); MLA paragraph).  For query (b, r), head h, with
 * J = { idx[b, r, j] : idx >= 0 } (-1 entries are skipped):
 *   z_j = scale * q[b, r, h, :dk] . kv[b, j, :dk]
 *   out[b, r, h, :] = sum_j softmax(z)_j * V[b, j, :dv]
 *   lse[b, r, h]    = log sum_j exp(z_j)      (natural log; -inf if J is empty)
 * Two forms:
 *   v == NULL  absorbed MLA: V = kv[..., :dv] (the first dv latent dims);
 *              dk = 576, dv = 512, heads = 16, k <= 2048; q and out bf16;
 *              dt = IC_BF16: kv rows are bf16, ld_kv in elements (a multiple of 8);
 *              dt = IC_E4M3: kv rows are fp8 cache rows (ic_pack_kv_e4m3), ld_kv in
 *              bytes (>= 656, a multiple of 16); each gathered row is dequantised
 *              in shared memory (code * its group's scale, rounded to bf16; rope
 *              as stored) before the same bf16 products.
 *   v != NULL  MQA with separate values v [batch, Lkv, dv]; dt = IC_F32,
 *              dk, dv <= 256, heads <= 64; out f32.
 *   q   [batch, rows, heads, dk]; kv [batch, Lkv, ld_kv] (ld_kv >= dk, elements);
 *   idx [batch, rows, k] int32 in [-1, Lkv); out [batch, rows, heads, dv];
 *   lse [batch, rows, heads] f32 or NULL.
 * workspace (device, may be NULL): with IC_BF16 and fewer than 4 queries per SM,
 * the (query, 32-key tile) pairs are cut into one equal contiguous range per SM,
 * and the partial results of each query's pieces go through the workspace (see
 * ic_attn_workspace_size) to a merge kernel; with too little workspace, or a
 * workspace that is not 16-byte aligned, there is no split (one CTA per query),
 * never an error.
 */
ic_status ic_sparse_attn(const void* q, const void* kv, long ld_kv, const void* v, const int* idx,
                         ic_dtype dt, int batch, int rows, int heads, int dk, int dv, int Lkv,
                         int k, float scale, void* out, float* lse, void* workspace,
                         size_t ws_bytes, void* stream);

/* Workspace bytes that let ic_sparse_attn use its preferred split for this shape. */
size_t ic_attn_workspace_size(int batch, int rows, int heads, int dv, int k);

/*
 * ic_sparse_attn_noalloc: the absorbed-MLA form of ic_sparse_attn for callers
 * that cannot allocate device memory -- for example a plugin whose host
 * framework hands it only its input and output buffers and offers no workspace
 * hook, or a process whose memory pool has claimed the whole device up front.
 * The paper has no counterpart; it is a convenience of this library.
 *
 * Same arguments, layouts and results as ic_sparse_attn with v = NULL and a
 * workspace of ic_attn_workspace_size bytes (the same split of the index list
 * is chosen), minus the workspace.  The split partials go to a fixed array of
 * IC_NOALLOC_SCRATCH_BYTES (16.06 MiB) inside this library, which every GPU
 * that loads the library holds until the process exits.  Neither this call
 * nor anything it calls allocates or frees device memory.
 *
 *   batch * rows <= IC_NOALLOC_MAX_QUERIES (64), else IC_ERR_UNSUPPORTED;
 *   v != NULL (the MQA form, which needs no scratch) -> IC_ERR_UNSUPPORTED;
 *   a split that needs more than IC_NOALLOC_SCRATCH_BYTES -> IC_ERR_WORKSPACE
 *     (queries * pieces per query <= SMs + 2 * queries: at most 276 of the 512
 *     slots on a 148-SM B200; only a part with far more SMs could need more);
 *   a failed device query or address lookup -> IC_ERR_CUDA;
 *   other checks and errors as ic_sparse_attn.
 * `out` and `lse` are the caller's, as for ic_sparse_attn.
 *
 * The first call in a CUDA context looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it under the
 * context's id; make that first call before any stream capture.  A call made
 * after a device reset (a new context) looks the address up again.  All calls
 * share the one array: calls that overlap on the GPU (other streams, other host
 * threads) race on it and must be serialised by the caller, e.g. by using a
 * single stream.  Each call overwrites every partial it later reads, so
 * leftovers from an earlier call do not matter.  Runs on the calling thread's
 * current device, which must own `stream`.
 */
#define IC_NOALLOC_MAX_QUERIES 64
#define IC_NOALLOC_SCRATCH_BYTES (64u * 8u * 16u * 514u * 4u)
ic_status ic_sparse_attn_noalloc(const void* q, const void* kv, long ld_kv, const void* v,
                                 const int* idx, ic_dtype dt, int batch, int rows, int heads,
                                 int dk, int dv, int Lkv, int k, float scale, void* out,
                                 float* lse, void* stream);

/*
 * Per-layer inputs of the layer stack.  Every pointer is device memory.
 * F layers need the indexer fields; S layers ignore them (they may be NULL).
 */
typedef struct {
  const void* q_idx;    /* [batch, R, H, D] indexer queries (idx_dtype)          */
  const float* q_scale; /* [batch, R, H] (IC_E4M3 only)                          */
  const void* k_idx;    /* [batch, L, D] indexer keys (idx_dtype)                */
  const float* k_scale; /* [batch, L] (IC_E4M3 only)                             */
  const float* w;       /* [batch, R, H] indexer head weights                    */
  const void* q;        /* [batch, R, heads, dk] attention queries (attn_dtype)  */
  const void* kv;       /* [batch, L, ld_kv] latent (MLA) or keys (MQA)          */
  const void* v;        /* [batch, L, dv] values (MQA only; NULL for MLA)        */
  void* out;            /* [batch, R, heads, dv] attention output                */
  float* lse;           /* [batch, R, heads] or NULL                             */
} ic_layer_io;

/*
 * Shape of a layer stack.
 *   prefill: batch = 1, R = L query rows at positions 0..L-1 (causal);
 *   decode:  batch sequences, R = 1 new token each, at position L-1 of a
 *            context of L tokens (keys 0..L-1).
 */
typedef struct {
  int L;               /* tokens (prefill) / context length (decode)             */
  int batch;           /* 1 for prefill; sequences for decode                    */
  int decode;          /* 0 = prefill, 1 = decode                                */
  int k;               /* top-k (<= 2048)                                        */
  ic_dtype idx_dtype;  /* IC_BF16, IC_E4M3 (H=64, D=128) or IC_F32              */
  int H, D;            /* indexer heads and head dim                             */
  ic_dtype attn_dtype; /* IC_BF16 / IC_E4M3 (absorbed MLA over a bf16 / fp8 cache,
                          ld_kv in elements / bytes) or IC_F32 (MQA)            */
  int heads, dk, dv;   /* attention heads, key dim, value dim                    */
  long ld_kv;          /* row stride of kv in elements                           */
  float scale;         /* softmax scale                                          */
  int flags;           /* IC_STACK_* bits (0 = defaults)                         */
} ic_stack_desc;

/* Decode with a tensor-core indexer: run the indexer and the top-k fused
 * (ic_indexer_topk: the scores never leave the chip; the same index sets)
 * instead of writing batch * L scores to the workspace and running ic_topk.
 * Off by default: on a B200 at 64 sequences x 200000 keys the fused pair takes
 * longer than the unfused one. */
#define IC_STACK_FUSED_TOPK 1

/*
 * The IndexCache layer stack (routing loop of "Einfache Implementierung",
 * without the FFN): for layer l = 1..N,
 *   c_l == 'F': T_cache <- top-k(Indexer_l)   (scores stream through `workspace`
 *               in row blocks; the L x L matrix is never formed)
 *   c_l == 'S': T_cache is reused unchanged   (zero work: the nearest preceding
 *               F layer's index set)
 *   out_l <- SparseAttn_l(T_cache)
 * pattern: host string of 'F'/'S', optionally separated by ',' or ' '; its
 * first layer must be 'F'; its layer count must equal nlayers.
 * layers: host array of nlayers ic_layer_io.  t_cache: device int32
 * [batch * R, k], caller-owned, holds the last F layer's index set on return.
 * workspace: device, at least ic_stack_workspace_size(desc) bytes is
 * recommended; the minimum is one score row block (a smaller workspace means
 * smaller row blocks, IC_ERR_WORKSPACE only below one row).
 */
ic_status ic_layer_stack(const char* pattern, const ic_stack_desc* desc, const ic_layer_io* layers,
                         int nlayers, int* t_cache, void* workspace, size_t ws_bytes,
                         void* stream);

/*
 * The prefill stack for query rows [row0, row0 + rows) of the desc->L-token
 * sequence only, so one long prefill can be shared out by rows (for example
 * over GPUs). Row r of the call sits at position row0 + r and attends causally
 * over keys 0..row0 + r. Per-row results are identical to ic_layer_stack's rows.
 * The row-indexed tensors of `layers` (q_idx, q_scale, w, q, out, lse) and
 * t_cache [rows, k] hold just these rows. k_idx, k_scale and kv hold all L keys.
 * ic_layer_stack is this call with row0 = 0, rows = desc->L.
 * 0 <= row0, row0 + rows <= desc->L, desc->decode = 0.  Other rules, the
 * workspace and the errors are as ic_layer_stack.
 */
ic_status ic_layer_stack_rows(const char* pattern, const ic_stack_desc* desc,
                              const ic_layer_io* layers, int nlayers, long row0, long rows,
                              int* t_cache, void* workspace, size_t ws_bytes, void* stream);

/*
 * The prefill stack over a batch of sequences of different lengths, packed
 * along the row axis: sequence i is rows [cu_seqlens[i], cu_seqlens[i+1]) of
 * every row-indexed tensor of `layers` (q_idx, q_scale, w, q, out, lse), of its
 * keys (k_idx, k_scale, kv, v) and of t_cache [sum L_i, k]. Each sequence runs
 * the whole routing loop on its own keys at positions 0..L_i - 1, as
 * ic_layer_stack would with desc->L = L_i.  cu_seqlens: host int64 [nseq + 1],
 * cu_seqlens[0] = 0, nondecreasing, every L_i <= desc->L (desc->L sizes the
 * workspace: ic_stack_workspace_size(desc) covers any batch).
 * The sequences share their launches: an F layer walks the packed query rows in
 * blocks of as many score rows as the workspace holds (desc->L floats plus one
 * int32 each), each block touching at most 64 sequences, with one indexer, one
 * valid-length and one top-k launch per block (each row scored against its own
 * sequence's keys); every layer's attention runs once per group of up to 64 whole
 * sequences.  Errors as ic_layer_stack.
 */
ic_status ic_layer_stack_varlen(const char* pattern, const ic_stack_desc* desc,
                                const ic_layer_io* layers, int nlayers, const long* cu_seqlens,
                                int nseq, int* t_cache, void* workspace, size_t ws_bytes,
                                void* stream);

/* Decode form of the stack (desc->decode must be 1): same routing per layer,
 * one query per sequence; t_cache is [batch, k].  With IC_STACK_FUSED_TOPK, F
 * layers with a bf16 or e4m3 indexer run it fused with the top-k (see
 * ic_indexer_topk). */
ic_status ic_decode_step(const char* pattern, const ic_stack_desc* desc, const ic_layer_io* layers,
                         int nlayers, int* t_cache, void* workspace, size_t ws_bytes,
                         void* stream);

/* Recommended workspace bytes for ic_layer_stack / ic_decode_step. */
size_t ic_stack_workspace_size(const ic_stack_desc* desc);

#ifdef __cplusplus
}
#endif
#endif /* IC_H_ */
