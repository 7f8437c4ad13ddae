// api.cu -- the C ABI declared in include/ic.h: argument checks, the F/S layer
// stack and the decode step (routing loop of "IndexCache: Wie DeepSeek
// O(NL^2)-Kosten in Sparse Attention um 75% reduziert", section "Einfache
// Implementierung, enorme Effizienzgewinne"), and the device error word.
#include <stdarg.h>
#include <stdio.h>

#include <string>
#include <vector>

#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

static thread_local std::string t_last_error;

// ---------------------------------------------------------------- launch tracing
struct TraceState {
  bool on = false;
  cudaStream_t stream = nullptr;
  std::vector<cudaEvent_t> events;  // events[0] is the start mark
  std::vector<int> kinds;
  std::vector<double> work;
  long launches = 0;
};
static thread_local TraceState t_trace;

void trace_launch(int kind, cudaStream_t stream, double work) {
  TraceState& t = t_trace;
  if (!t.on) return;
  ++t.launches;
  if (t.kinds.size() + 1 >= t.events.size()) return;  // capacity reached: count only
  cudaEvent_t ev = t.events[t.kinds.size() + 1];
  if (cudaEventRecord(ev, stream) != cudaSuccess) return;
  t.kinds.push_back(kind);
  t.work.push_back(work);
}

ic_status fail(ic_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return code;
}

ic_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return IC_OK;
  return fail(IC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

static inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// Pattern grammar: 'F' / 'S', optionally separated by ',' or ' '; first layer F.
static ic_status parse_pattern(const char* pattern, std::vector<char>* kinds) {
  if (!pattern) return fail(IC_ERR_INVALID_ARG, "pattern is NULL");
  kinds->clear();
  for (const char* c = pattern; *c; ++c) {
    if (*c == ',' || *c == ' ') continue;
    if (*c != 'F' && *c != 'S')
      return fail(IC_ERR_INVALID_ARG, "bad character '%c' in layer pattern", *c);
    kinds->push_back(*c);
  }
  if (kinds->empty()) return fail(IC_ERR_INVALID_ARG, "empty layer pattern");
  if ((*kinds)[0] != 'F')
    return fail(IC_ERR_INVALID_ARG, "the first layer must be F (it fills the index cache)");
  return IC_OK;
}

static ic_status check_indexer(const void* q, const float* q_scale, const void* k,
                               const float* k_scale, const float* w, ic_dtype dt, int batch, int H,
                               int D, int rows, int Lk, long pos0, const float* scores, long ld,
                               bool need_scores = true) {
  if (!q || !k || !w || (need_scores && !scores))
    return fail(IC_ERR_INVALID_ARG, "indexer: NULL tensor");
  if (batch < 1 || rows < 0 || Lk < 1 || pos0 < 0 || ld < Lk)
    return fail(IC_ERR_INVALID_ARG, "indexer: bad sizes (batch %d rows %d Lk %d pos0 %ld ld %ld)",
                batch, rows, Lk, pos0, ld);
  if (dt == IC_BF16 || dt == IC_E4M3) {
    if (H != 64 || D != 128)
      return fail(IC_ERR_UNSUPPORTED, "indexer: tensor-core path needs H=64, D=128 (got %d, %d)",
                  H, D);
    if (dt == IC_E4M3 && (!q_scale || !k_scale))
      return fail(IC_ERR_INVALID_ARG, "indexer: e4m3 inputs need q_scale and k_scale");
    if (!aligned(q, 16) || !aligned(k, 16))
      return fail(IC_ERR_INVALID_ARG, "indexer: q and k must be 16-byte aligned");
    if (static_cast<long>(batch) * rows * 64 > 0x7fffffffL || static_cast<long>(batch) * Lk > 0x7fffffffL)
      return fail(IC_ERR_UNSUPPORTED, "indexer: tensor too large for 32-bit TMA coordinates");
  } else if (dt == IC_F32) {
    if (H < 1 || H > 64 || D < 1 || D > 256)
      return fail(IC_ERR_UNSUPPORTED, "indexer: fp32 path needs H <= 64, D <= 256");
  } else {
    return fail(IC_ERR_INVALID_ARG, "indexer: unknown dtype %d", static_cast<int>(dt));
  }
  return IC_OK;
}

static ic_status run_indexer(const void* q, const float* q_scale, const void* k,
                             const float* k_scale, const float* w, ic_dtype dt, int batch, int H,
                             int D, int rows, int Lk, long pos0, float* scores, long ld,
                             bool fill_tail, cudaStream_t stream) {
  if (dt == IC_F32)
    return launch_indexer_f32(static_cast<const float*>(q), static_cast<const float*>(k), w, batch,
                              H, D, rows, Lk, pos0, scores, ld, stream);
  return launch_indexer_tc(dt == IC_E4M3, q, q_scale, k, k_scale, w, batch, rows, Lk, pos0, scores,
                           ld, fill_tail, stream);
}

static ic_status check_attn(const void* q, const void* kv, long ld_kv, const void* v,
                            const int* idx, ic_dtype dt, int batch, int rows, int heads, int dk,
                            int dv, int Lkv, int k, const void* out) {
  if (!q || !kv || !idx || !out) return fail(IC_ERR_INVALID_ARG, "attn: NULL tensor");
  if (batch < 1 || rows < 0 || Lkv < 1 || k < 1 || ld_kv < dk)
    return fail(IC_ERR_INVALID_ARG, "attn: bad sizes");
  if (!v) {
    if ((dt != IC_BF16 && dt != IC_E4M3) || heads != 16 || dk != 576 || dv != 512)
      return fail(IC_ERR_UNSUPPORTED,
                  "attn: absorbed MLA needs a bf16 or e4m3 cache, 16 heads, dk 576, dv 512 "
                  "(got %d, %d, %d, %d)", static_cast<int>(dt), heads, dk, dv);
    if (!aligned(q, 16) || !aligned(kv, 16) ||
        (dt == IC_BF16 ? (ld_kv % 8) != 0 : (ld_kv < KV8_ROW_BYTES || (ld_kv % 16) != 0)))
      return fail(IC_ERR_INVALID_ARG,
                  "attn: q/kv rows must be 16-byte aligned (e4m3 cache: ld_kv >= 656 bytes)");
    if (k > 2048) return fail(IC_ERR_UNSUPPORTED, "attn: absorbed MLA needs k <= 2048");
  } else {
    if (dt != IC_F32 || heads < 1 || heads > 64 || dk < 1 || dk > 256 || dv < 1 || dv > 256)
      return fail(IC_ERR_UNSUPPORTED, "attn: MQA form needs fp32, heads <= 64, dk, dv <= 256");
    if (k > 8192) return fail(IC_ERR_UNSUPPORTED, "attn: MQA form needs k <= 8192");
  }
  return IC_OK;
}

static ic_status run_attn(const void* q, const void* kv, long ld_kv, const void* v,
                          const int* idx, ic_dtype dt, int batch, int rows, int heads, int dk,
                          int dv, int Lkv, int k, float scale, void* out, float* lse, void* ws,
                          size_t ws_bytes, long long valid_entries, cudaStream_t stream) {
  if (!v)
    return launch_attn_mla(q, kv, ld_kv, idx, batch, rows, Lkv, k, scale, out, lse, ws, ws_bytes,
                           valid_entries, stream, dt == IC_E4M3);
  return launch_attn_f32(static_cast<const float*>(q), static_cast<const float*>(kv), ld_kv,
                         static_cast<const float*>(v), idx, batch, rows, heads, dk, dv, Lkv, k,
                         scale, static_cast<float*>(out), lse, stream);
}

static size_t elem_bytes(ic_dtype dt) { return dt == IC_E4M3 ? 1 : (dt == IC_BF16 ? 2 : 4); }

static ic_status check_desc(const ic_stack_desc* d, bool decode) {
  if (!d) return fail(IC_ERR_INVALID_ARG, "stack: desc is NULL");
  if (d->L < 1 || d->k < 1 || d->k > 2048 || d->batch < 1)
    return fail(IC_ERR_INVALID_ARG, "stack: bad sizes (L %d k %d batch %d)", d->L, d->k, d->batch);
  if ((d->decode != 0) != decode)
    return fail(IC_ERR_INVALID_ARG, decode ? "decode step needs desc->decode = 1"
                                           : "layer stack needs desc->decode = 0 (use ic_decode_step)");
  if (!decode && d->batch != 1) return fail(IC_ERR_UNSUPPORTED, "stack: prefill batch must be 1");
  return IC_OK;
}

// Rows per score block for a workspace of ws_bytes: scores [rows, L] fp32.
static long score_rows(size_t ws_bytes, long L, long want) {
  long rb = static_cast<long>(ws_bytes / (static_cast<size_t>(L) * sizeof(float)));
  if (rb > want) rb = want;
  if (rb >= 4 && rb < want) rb &= ~3L;  // keep query blocks of 4 whole
  return rb;
}

// Prefill runs query rows [row0, row0 + rows) of the L-token sequence (keys are
// always 0..L-1); decode runs every sequence's one query (row0 = 0, rows = L unused).
static ic_status run_stack(const char* pattern, const ic_stack_desc* d, const ic_layer_io* layers,
                           int nlayers, int* t_cache, void* workspace, size_t ws_bytes,
                           void* stream_v, bool decode, long row0 = 0, long rows = -1) {
  ic_status st = check_desc(d, decode);
  if (st) return st;
  if (rows < 0) rows = d->L;
  if (!decode && (row0 < 0 || rows < 0 || row0 + rows > d->L))
    return fail(IC_ERR_INVALID_ARG, "stack: rows [%ld, %ld) outside the %d-token sequence", row0,
                row0 + rows, d->L);
  std::vector<char> kinds;
  st = parse_pattern(pattern, &kinds);
  if (st) return st;
  if (static_cast<int>(kinds.size()) != nlayers)
    return fail(IC_ERR_INVALID_ARG, "pattern has %zu layers, nlayers is %d", kinds.size(), nlayers);
  if (!layers || !t_cache) return fail(IC_ERR_INVALID_ARG, "stack: NULL layers or t_cache");
  const int B = d->batch;
  const int R = decode ? 1 : static_cast<int>(rows);  // query rows per sequence
  const long pos0 = decode ? d->L - 1 : row0;
  for (int l = 0; l < nlayers; ++l) {
    const ic_layer_io& io = layers[l];
    if (kinds[l] == 'F') {
      st = check_indexer(io.q_idx, io.q_scale, io.k_idx, io.k_scale, io.w, d->idx_dtype, B, d->H,
                         d->D, R, d->L, pos0, nullptr, d->L, false);
      if (st) return fail(st, "layer %d: %s", l, ic_last_error());
    }
    st = check_attn(io.q, io.kv, d->ld_kv, io.v, t_cache, d->attn_dtype, B, R, d->heads, d->dk,
                    d->dv, d->L, d->k, io.out);
    if (st) return fail(st, "layer %d: %s", l, ic_last_error());
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  const size_t qrow_b = static_cast<size_t>(d->H) * d->D * elem_bytes(d->idx_dtype);
  const size_t krow_b = static_cast<size_t>(d->D) * elem_bytes(d->idx_dtype);

  // decode with a tensor-core indexer: indexer and top-k fused (no score rows)
  const bool fused = decode && d->idx_dtype != IC_F32 && (d->flags & IC_STACK_FUSED_TOPK);
  if (fused) {
    const size_t need = indexer_topk_fused_ws_bytes(B, d->L, d->L - 1);
    if (!workspace || ws_bytes < need)
      return fail(IC_ERR_WORKSPACE, "decode: the fused indexer/top-k needs %zu workspace bytes "
                  "(got %zu)", need, ws_bytes);
  }
  // rows of scores per block: prefill streams query rows, decode streams sequences
  const long units = decode ? B : R;
  const long rb = fused ? units : score_rows(ws_bytes, d->L, units);
  if (!workspace || rb < 1)
    return fail(IC_ERR_WORKSPACE, "stack: workspace of %zu bytes holds no score row of %d floats",
                ws_bytes, d->L);
  float* scores = static_cast<float*>(workspace);

  for (int l = 0; l < nlayers; ++l) {
    const ic_layer_io& io = layers[l];
    if (kinds[l] == 'F' && fused) {
      // T_cache <- top-k(Indexer_l(X)) in one pass over the key cache
      st = launch_indexer_topk_fused(d->idx_dtype == IC_E4M3, io.q_idx, io.q_scale, io.k_idx,
                                     io.k_scale, io.w, B, d->L, d->L - 1, d->k, t_cache,
                                     workspace, ws_bytes, stream);
      if (st) return st;
    } else if (kinds[l] == 'F') {
      // T_cache <- top-k(Indexer_l(X)), one block of score rows at a time
      for (long u0 = 0; u0 < units; u0 += rb) {
        const long nu = (units - u0 < rb) ? units - u0 : rb;
        const uint8_t* qi = static_cast<const uint8_t*>(io.q_idx);
        const float* qs = io.q_scale;
        if (!decode) {
          // local query rows u0 .. u0+nu-1 sit at positions row0 + u0.., keys 0..row0+u0+nu-1
          const long p0 = row0 + u0;
          const int Lk = static_cast<int>(p0 + nu);
          st = run_indexer(qi + u0 * qrow_b, qs ? qs + u0 * d->H : nullptr, io.k_idx, io.k_scale,
                           io.w + u0 * d->H, d->idx_dtype, 1, d->H, d->D, static_cast<int>(nu), Lk,
                           p0, scores, d->L, false, stream);
          if (st) return st;
          st = launch_topk(scores, nu, Lk, d->L, p0, d->k, t_cache + u0 * d->k, stream);
        } else {
          // sequences u0 .. u0+nu-1, one query each at position L-1 over L keys
          const uint8_t* ki = static_cast<const uint8_t*>(io.k_idx);
          st = run_indexer(qi + u0 * qrow_b, qs ? qs + u0 * d->H : nullptr,
                           ki + u0 * static_cast<size_t>(d->L) * krow_b,
                           io.k_scale ? io.k_scale + u0 * d->L : nullptr, io.w + u0 * d->H,
                           d->idx_dtype, static_cast<int>(nu), d->H, d->D, 1, d->L, pos0, scores,
                           d->L, false, stream);
          if (st) return st;
          st = launch_topk(scores, nu, d->L, d->L, -1, d->k, t_cache + u0 * d->k, stream);
        }
        if (st) return st;
      }
    }
    // S layers: T_cache is reused as is (the nearest preceding F layer's set)
    // out_l <- SparseAttn_l(T_cache); the score workspace is free again here
    const long long valid = decode ? static_cast<long long>(B) * (d->k < d->L ? d->k : d->L)
                                   : causal_pairs(R, d->k, row0);
    st = run_attn(io.q, io.kv, d->ld_kv, io.v, t_cache, d->attn_dtype, B, R, d->heads, d->dk,
                  d->dv, d->L, d->k, d->scale, io.out, io.lse, workspace, ws_bytes, valid, stream);
    if (st) return st;
  }
  return IC_OK;
}

// Packed sequences (cu: host [nseq + 1]) of a stack in shared launches.
// F layers walk the packed query rows in blocks that fit the score workspace and
// touch at most IC_MAXSEG sequences: one indexer launch over the block's segments
// (each row against its own sequence's keys), one valid-length fill and one top-k
// launch; attention runs over groups of at most IC_MAXSEG whole sequences.  The
// launch count depends on the rows and the number of groups, not on nseq.
static ic_status run_stack_varlen_shared(const std::vector<char>& kinds, const ic_stack_desc* d,
                                         const ic_layer_io* layers, int nlayers, const long* cu,
                                         int nseq, int* t_cache, void* workspace, size_t ws_bytes,
                                         cudaStream_t stream) {
  const long total = cu[nseq];
  if (total == 0) return IC_OK;
  for (int l = 0; l < nlayers; ++l) {
    const ic_layer_io& io = layers[l];
    if (kinds[l] == 'F') {
      ic_status st = check_indexer(io.q_idx, io.q_scale, io.k_idx, io.k_scale, io.w, d->idx_dtype,
                                   1, d->H, d->D, static_cast<int>(total),
                                   static_cast<int>(total), 0, nullptr, total, false);
      if (st) return fail(st, "layer %d: %s", l, ic_last_error());
    }
    ic_status st = check_attn(io.q, io.kv, d->ld_kv, io.v, t_cache, d->attn_dtype, 1,
                              static_cast<int>(total), d->heads, d->dk, d->dv, d->L, d->k, io.out);
    if (st) return fail(st, "layer %d: %s", l, ic_last_error());
  }
  // score rows of L floats plus one valid length each
  const long ld = d->L;
  long rb = static_cast<long>(ws_bytes / (static_cast<size_t>(ld) * sizeof(float) + sizeof(int)));
  if (rb > total) rb = total;
  if (rb >= 4 && rb < total) rb &= ~3L;
  if (!workspace || rb < 1)
    return fail(IC_ERR_WORKSPACE, "varlen: workspace of %zu bytes holds no score row of %ld floats",
                ws_bytes, ld);
  float* scores = static_cast<float*>(workspace);
  int* valid = reinterpret_cast<int*>(scores + rb * ld);
  const bool kv8 = d->attn_dtype == IC_E4M3;
  const bool f32_idx = d->idx_dtype == IC_F32, f32_attn = d->attn_dtype == IC_F32;
  const size_t qe = f32_attn ? 4 : 2;  // q and out: fp32 (MQA) or bf16 (MLA)
  const size_t arow_b = static_cast<size_t>(d->heads) * d->dk * qe;
  const size_t orow_b = static_cast<size_t>(d->heads) * d->dv * qe;
  const size_t qrow_b = static_cast<size_t>(d->H) * d->D * elem_bytes(d->idx_dtype);
  std::vector<IdxSeg> segs;
  std::vector<AttnSeg> asegs;
  for (int l = 0; l < nlayers; ++l) {
    const ic_layer_io& io = layers[l];
    if (kinds[l] == 'F') {
      int sf = 0;  // first sequence with rows at or after u0
      for (long u0 = 0; u0 < total;) {
        while (sf < nseq && cu[sf + 1] <= u0) ++sf;
        long u1 = u0 + rb < total ? u0 + rb : total;
        const int sl = sf + IC_MAXSEG < nseq ? sf + IC_MAXSEG : nseq;
        if (cu[sl] < u1) u1 = cu[sl];  // at most IC_MAXSEG sequences in the block
        segs.clear();
        for (int sq = sf; sq < sl && cu[sq] < u1; ++sq) {
          const long c0 = cu[sq], c1 = cu[sq + 1];
          const long a0 = c0 > u0 ? c0 : u0, a1 = c1 < u1 ? c1 : u1;
          if (a1 <= a0) continue;
          IdxSeg g;
          g.qrow0 = a0;
          g.krow0 = c0;
          g.orow0 = a0 - u0;
          g.pos0 = a0 - c0;
          g.R = static_cast<int>(a1 - a0);
          g.Lk = static_cast<int>(c1 - c0);
          g.qb0 = 0;
          g.pad = 0;
          segs.push_back(g);
        }
        const long nu = u1 - u0;
        ic_status st =
            f32_idx ? launch_indexer_f32_segs(
                          reinterpret_cast<const float*>(static_cast<const uint8_t*>(io.q_idx) +
                                                         u0 * qrow_b),
                          static_cast<const float*>(io.k_idx), io.w + u0 * d->H, d->H, d->D,
                          segs.data(), static_cast<int>(segs.size()), nu, scores, ld, stream)
                    : launch_indexer_tc_segs(d->idx_dtype == IC_E4M3, io.q_idx, io.q_scale,
                                             io.k_idx, io.k_scale, io.w, segs.data(),
                                             static_cast<int>(segs.size()), total, total, scores,
                                             ld, stream);
        if (st) return st;
        st = launch_fill_valid_len(segs.data(), static_cast<int>(segs.size()), nu, valid, stream);
        if (st) return st;
        st = launch_topk(scores, nu, static_cast<int>(ld), ld, 0, d->k, t_cache + u0 * d->k, stream,
                         valid);
        if (st) return st;
        u0 = u1;
      }
    }
    // attention over groups of whole sequences
    for (int g0 = 0; g0 < nseq; g0 += IC_MAXSEG) {
      const int g1 = g0 + IC_MAXSEG < nseq ? g0 + IC_MAXSEG : nseq;
      const long r0 = cu[g0], nr = cu[g1] - cu[g0];
      if (nr == 0) continue;
      asegs.clear();
      long long valid_entries = 0;
      for (int sq = g0; sq < g1; ++sq) {
        const long n = cu[sq + 1] - cu[sq];
        if (n == 0) continue;
        AttnSeg a;
        a.q0 = cu[sq] - r0;
        a.k0 = cu[sq];
        a.len = static_cast<int>(n);
        a.pad = 0;
        asegs.push_back(a);
        valid_entries += causal_pairs(n, d->k, 0);
      }
      const void* qg = static_cast<const uint8_t*>(io.q) + r0 * arow_b;
      void* og = static_cast<uint8_t*>(io.out) + r0 * orow_b;
      float* lg = io.lse ? io.lse + r0 * d->heads : nullptr;
      ic_status st =
          f32_attn ? launch_attn_f32(static_cast<const float*>(qg), static_cast<const float*>(io.kv),
                                     d->ld_kv, static_cast<const float*>(io.v), t_cache + r0 * d->k,
                                     1, static_cast<int>(nr), d->heads, d->dk, d->dv, d->L, d->k,
                                     d->scale, static_cast<float*>(og), lg, stream, asegs.data(),
                                     static_cast<int>(asegs.size()))
                   : launch_attn_mla(qg, io.kv, d->ld_kv, t_cache + r0 * d->k, 1,
                                     static_cast<int>(nr), d->L, d->k, d->scale, og, lg, workspace,
                                     ws_bytes, valid_entries, stream, kv8, asegs.data(),
                                     static_cast<int>(asegs.size()));
      if (st) return st;
    }
  }
  return IC_OK;
}

}  // namespace ic

using namespace ic;

extern "C" {

const char* ic_last_error(void) { return t_last_error.c_str(); }

int ic_version(void) { return 102; }

ic_status ic_device_status(void* stream) {
  ic_status st = cuda_check(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)),
                            "cudaStreamSynchronize");
  if (st) return st;
  int v = 0;
  st = cuda_check(cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(int)), "read device error word");
  if (st) return st;
  if (v != 0) {
    const int zero = 0;
    st = cuda_check(cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(int)), "clear device error word");
    if (st) return st;
    if (v >= kErrBoundsFirst)
      return fail(IC_ERR_BOUNDS, "device error word %d (a debug-bounds check failed: %s)", v,
                  v == kErrBoundsGather ? "index-list entry outside the cache"
                  : v == kErrBoundsTma  ? "TMA tile coordinate outside the tensor"
                  : v == kErrBoundsTopk ? "top-k output slot outside the row"
                                        : "merge slot or piece count out of range");
    return fail(IC_ERR_TIMEOUT, "device error word %d (a bounded device wait gave up)", v);
  }
  return IC_OK;
}

ic_status ic_trace_begin(void* stream, int capacity) {
  TraceState& t = t_trace;
  if (t.on) return fail(IC_ERR_INVALID_ARG, "trace: already recording on this thread");
  if (capacity < 1) return fail(IC_ERR_INVALID_ARG, "trace: capacity must be >= 1");
  while (static_cast<int>(t.events.size()) < capacity + 1) {
    cudaEvent_t ev;
    ic_status st = cuda_check(cudaEventCreate(&ev), "cudaEventCreate");
    if (st) return st;
    t.events.push_back(ev);
  }
  t.kinds.clear();
  t.work.clear();
  t.launches = 0;
  t.stream = static_cast<cudaStream_t>(stream);
  ic_status st = cuda_check(cudaEventRecord(t.events[0], t.stream), "cudaEventRecord");
  if (st) return st;
  t.on = true;
  return IC_OK;
}

long ic_trace_end(float* ms, int* kinds, double* work, int capacity) {
  TraceState& t = t_trace;
  if (!t.on) return fail(IC_ERR_INVALID_ARG, "trace: not recording");
  t.on = false;
  const int n = static_cast<int>(t.kinds.size());
  if (n > 0) {
    ic_status st = cuda_check(cudaEventSynchronize(t.events[n]), "cudaEventSynchronize");
    if (st) return st;
  }
  for (int i = 0; i < n && i < capacity; ++i) {
    float v = 0.f;
    if (ms) {
      ic_status st = cuda_check(cudaEventElapsedTime(&v, t.events[i], t.events[i + 1]),
                                "cudaEventElapsedTime");
      if (st) return st;
      ms[i] = v;
    }
    if (kinds) kinds[i] = t.kinds[i];
    if (work) work[i] = t.work[i];
  }
  return t.launches;
}

ic_status ic_quant_e4m3_rows(const void* x, ic_dtype x_dtype, long rows, int n, uint8_t* codes,
                             float* scales, void* stream) {
  if (!x || !codes || !scales) return fail(IC_ERR_INVALID_ARG, "quant: NULL tensor");
  if (rows < 0 || n < 8 || n > 1024 || (n % 8) != 0)
    return fail(IC_ERR_INVALID_ARG, "quant: need rows >= 0 and n a multiple of 8 in [8, 1024]");
  if (x_dtype != IC_BF16 && x_dtype != IC_F32)
    return fail(IC_ERR_UNSUPPORTED, "quant: input must be bf16 or fp32");
  return launch_quant_e4m3(x, x_dtype == IC_BF16, rows, n, codes, scales,
                           static_cast<cudaStream_t>(stream));
}

ic_status ic_pack_kv_e4m3(const void* kv, long rows, long ld_kv, uint8_t* out, long ld_out,
                          void* stream) {
  if (!kv || !out) return fail(IC_ERR_INVALID_ARG, "pack_kv: NULL tensor");
  if (rows < 0 || ld_kv < 576 || (ld_kv % 8) != 0 || ld_out < KV8_ROW_BYTES || (ld_out % 16) != 0)
    return fail(IC_ERR_INVALID_ARG,
                "pack_kv: need ld_kv >= 576 (a multiple of 8) and ld_out >= 656 (of 16)");
  if (!aligned(kv, 16) || !aligned(out, 16))
    return fail(IC_ERR_INVALID_ARG, "pack_kv: rows must be 16-byte aligned");
  return launch_pack_kv_e4m3(kv, rows, ld_kv, out, ld_out, static_cast<cudaStream_t>(stream));
}

ic_status ic_indexer_scores(const void* q, const float* q_scale, const void* k,
                            const float* k_scale, const float* w, ic_dtype dt, int batch, int H,
                            int D, int rows, int Lk, long pos0, float* scores, long ld,
                            void* stream) {
  ic_status st =
      check_indexer(q, q_scale, k, k_scale, w, dt, batch, H, D, rows, Lk, pos0, scores, ld);
  if (st) return st;
  return run_indexer(q, q_scale, k, k_scale, w, dt, batch, H, D, rows, Lk, pos0, scores, ld, true,
                     static_cast<cudaStream_t>(stream));
}

ic_status ic_topk(const float* scores, long rows, int n, long ld, long pos0, int k, int* idx,
                  void* stream) {
  if (!scores || !idx) return fail(IC_ERR_INVALID_ARG, "topk: NULL tensor");
  if (rows < 0 || n < 0 || ld < n || k < 1 || k > 2048)
    return fail(IC_ERR_INVALID_ARG, "topk: bad sizes (rows %ld n %d ld %ld k %d)", rows, n, ld, k);
  if (rows > 0x7fffffffL) return fail(IC_ERR_UNSUPPORTED, "topk: too many rows");
  return launch_topk(scores, rows, n, ld, pos0, k, idx, static_cast<cudaStream_t>(stream));
}

ic_status ic_indexer_topk(const void* q, const float* q_scale, const void* k,
                          const float* k_scale, const float* w, ic_dtype dt, int batch, int H,
                          int D, int Lk, long pos0, int k_top, int* idx, void* workspace,
                          size_t ws_bytes, void* stream) {
  if (dt != IC_BF16 && dt != IC_E4M3)
    return fail(IC_ERR_UNSUPPORTED, "indexer_topk: needs the tensor-core indexer (bf16 or e4m3)");
  ic_status st = check_indexer(q, q_scale, k, k_scale, w, dt, batch, H, D, 1, Lk, pos0, nullptr,
                               Lk, false);
  if (st) return st;
  if (!idx) return fail(IC_ERR_INVALID_ARG, "indexer_topk: idx is NULL");
  if (k_top < 1 || k_top > 2048)
    return fail(IC_ERR_INVALID_ARG, "indexer_topk: k must be in [1, 2048] (got %d)", k_top);
  return launch_indexer_topk_fused(dt == IC_E4M3, q, q_scale, k, k_scale, w, batch, Lk, pos0,
                                   k_top, idx, workspace, ws_bytes,
                                   static_cast<cudaStream_t>(stream));
}

size_t ic_indexer_topk_workspace_size(int batch, int Lk, long pos0) {
  if (batch < 1 || Lk < 1 || pos0 < 0) return 0;
  return indexer_topk_fused_ws_bytes(batch, Lk, pos0);
}

ic_status ic_topk_varlen(const float* scores, long rows, int n, long ld, const int* valid_len,
                         int k, int* idx, void* stream) {
  if (!scores || !idx || !valid_len) return fail(IC_ERR_INVALID_ARG, "topk_varlen: NULL tensor");
  if (rows < 0 || n < 0 || ld < n || k < 1 || k > 2048)
    return fail(IC_ERR_INVALID_ARG, "topk_varlen: bad sizes (rows %ld n %d ld %ld k %d)", rows, n,
                ld, k);
  if (rows > 0x7fffffffL) return fail(IC_ERR_UNSUPPORTED, "topk_varlen: too many rows");
  return launch_topk(scores, rows, n, ld, -1, k, idx, static_cast<cudaStream_t>(stream),
                     valid_len);
}

ic_status ic_sparse_attn(const void* q, const void* kv, long ld_kv, const void* v, const int* idx,
                         ic_dtype dt, int batch, int rows, int heads, int dk, int dv, int Lkv,
                         int k, float scale, void* out, float* lse, void* workspace,
                         size_t ws_bytes, void* stream) {
  ic_status st = check_attn(q, kv, ld_kv, v, idx, dt, batch, rows, heads, dk, dv, Lkv, k, out);
  if (st) return st;
  return run_attn(q, kv, ld_kv, v, idx, dt, batch, rows, heads, dk, dv, Lkv, k, scale, out, lse,
                  workspace, ws_bytes, -1, static_cast<cudaStream_t>(stream));
}

size_t ic_attn_workspace_size(int batch, int rows, int heads, int dv, int k) {
  if (heads != 16 || dv != 512 || batch < 1 || rows < 0 || k < 1) return 0;
  return attn_mla_ws_bytes(batch, rows, k);
}

ic_status ic_layer_stack(const char* pattern, const ic_stack_desc* desc, const ic_layer_io* layers,
                         int nlayers, int* t_cache, void* workspace, size_t ws_bytes,
                         void* stream) {
  return run_stack(pattern, desc, layers, nlayers, t_cache, workspace, ws_bytes, stream, false);
}

ic_status ic_layer_stack_rows(const char* pattern, const ic_stack_desc* desc,
                              const ic_layer_io* layers, int nlayers, long row0, long rows,
                              int* t_cache, void* workspace, size_t ws_bytes, void* stream) {
  if (desc && (row0 < 0 || rows < 0 || row0 + rows > desc->L))
    return fail(IC_ERR_INVALID_ARG, "stack: rows [%ld, %ld) outside the %d-token sequence", row0,
                row0 + rows, desc->L);
  return run_stack(pattern, desc, layers, nlayers, t_cache, workspace, ws_bytes, stream, false,
                   row0, rows);
}

ic_status ic_layer_stack_varlen(const char* pattern, const ic_stack_desc* desc,
                                const ic_layer_io* layers, int nlayers, const long* cu_seqlens,
                                int nseq, int* t_cache, void* workspace, size_t ws_bytes,
                                void* stream) {
  if (!desc) return fail(IC_ERR_INVALID_ARG, "stack: desc is NULL");
  if (!cu_seqlens || nseq < 0) return fail(IC_ERR_INVALID_ARG, "varlen: bad cu_seqlens / nseq");
  if (cu_seqlens[0] != 0) return fail(IC_ERR_INVALID_ARG, "varlen: cu_seqlens[0] must be 0");
  for (int i = 0; i < nseq; ++i)
    if (cu_seqlens[i + 1] < cu_seqlens[i] || cu_seqlens[i + 1] - cu_seqlens[i] > desc->L)
      return fail(IC_ERR_INVALID_ARG,
                  "varlen: sequence %d has %ld tokens (must be 0..desc->L = %d)", i,
                  cu_seqlens[i + 1] - cu_seqlens[i], desc->L);
  if (nlayers < 1 || nlayers > 4096 || !layers)
    return fail(IC_ERR_INVALID_ARG, "varlen: bad layers / nlayers");
  ic_status st = check_desc(desc, false);
  if (st) return st;
  std::vector<char> kinds;
  st = parse_pattern(pattern, &kinds);
  if (st) return st;
  if (static_cast<int>(kinds.size()) != nlayers)
    return fail(IC_ERR_INVALID_ARG, "pattern has %zu layers, nlayers is %d", kinds.size(), nlayers);
  if (!t_cache) return fail(IC_ERR_INVALID_ARG, "varlen: NULL t_cache");
  if (cu_seqlens[nseq] * 64 > 0x7fffffffL)
    return fail(IC_ERR_UNSUPPORTED, "varlen: too many rows for 32-bit TMA coordinates");
  return run_stack_varlen_shared(kinds, desc, layers, nlayers, cu_seqlens, nseq, t_cache,
                                 workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

ic_status ic_decode_step(const char* pattern, const ic_stack_desc* desc, const ic_layer_io* layers,
                         int nlayers, int* t_cache, void* workspace, size_t ws_bytes,
                         void* stream) {
  return run_stack(pattern, desc, layers, nlayers, t_cache, workspace, ws_bytes, stream, true);
}

size_t ic_stack_workspace_size(const ic_stack_desc* d) {
  if (!d || d->L < 1 || d->batch < 1) return 0;
  const long units = d->decode ? d->batch : d->L;
  const long want = d->decode ? units : (units < 4096 ? units : 4096);
  size_t s = static_cast<size_t>(want) * d->L * sizeof(float);
  if (d->decode && d->idx_dtype != IC_F32 && (d->flags & IC_STACK_FUSED_TOPK))
    s = indexer_topk_fused_ws_bytes(d->batch, d->L, d->L - 1);
  if (d->decode && d->attn_dtype != IC_F32) {
    const size_t a = attn_mla_ws_bytes(d->batch, 1, d->k);
    if (a > s) s = a;
  }
  return s;
}

}  // extern "C"
