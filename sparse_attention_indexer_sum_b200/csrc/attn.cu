// attn.cu -- sparse attention over the index set (routing loop
// X <- SparseAttn(X, T) of "IndexCache: Wie DeepSeek O(NL^2)-Kosten in Sparse
// Attention um 75% reduziert"; MLA paragraph: one latent row shared by all heads).
//
// Absorbed MLA, bf16: 16 query heads of dim 576 attend over the selected rows
// of the 576-dim latent cache; the value of a row is its first 512 dims.
//
// The work is bound by gathering k latent rows (1152 B each) per query: with
// 16 heads there are only ~30 flops per gathered byte, far below the tensor
// ridge.  So the kernel is built around the gather:
//   * four producer warps issue one TMA bulk copy (cp.async.bulk, 1152 B) per
//     selected row (8 rows of each 32-row tile per warp) straight into a
//     4-stage ring of shared tiles, each stage completing on an mbarrier by
//     transaction count; producer 0 also fetches each item's index list (one
//     bulk copy, one item ahead) and its 16 query rows;
//   * eight consumer warps run S = Q K^T (16 x 32 x 576) and O += P V
//     (16 x 512 x 32) on the warp-level bf16 tensor-core MMA, whose M = 16 is
//     exactly the 16 heads, with an online softmax in base 2.  QK: warp w covers
//     keys 16(w%2)..+16 over dims 144(w/2)..+144 with its quarter of Q in
//     registers; the four partial scores meet in shared memory.  The next tile's
//     QK is issued, then warp w computes the softmax of heads 2w, 2w+1 once
//     (16 lanes per head) and leaves P (bf16) and the rescale factors in shared
//     memory.  PV: warp w owns output dims 64w..+64;
//   * CTAs are persistent (one per SM).  With many queries, they walk the
//     queries round-robin, so neighbouring queries (which share many selected
//     rows) run at the same time and hit in L2.  With few queries (decode), the
//     (query, tile) pairs are cut into one contiguous range per CTA.  Each
//     (query, range) piece leaves an unnormalised partial in the workspace, and
//     attn_combine_kernel merges them.
// Shared rows are padded to 1168 B so that ldmatrix is bank-conflict free.
#include <type_traits>

#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

constexpr int AT_H = 16;
constexpr int AT_DK = 576;
constexpr int AT_DV = 512;
constexpr int AT_BK = 32;                   // keys per tile
constexpr int AT_STAGES = 4;
constexpr int AT_MAXK = 2048;               // longest index list of one item
constexpr int AT_CONSUMERS = 256;           // 8 consumer warps
constexpr int AT_PRODUCERS = 4;             // producer warps; each issues 8 of a tile's 32 rows
constexpr int AT_THREADS = AT_CONSUMERS + 32 * AT_PRODUCERS;
constexpr int AT_ROWB = AT_DK * 2 + 16;     // padded shared row: 1168 B
static_assert(AT_ROWB - KV8_ROW_BYTES == 512, "an fp8 row lands behind its 512 bf16 latent dims");
constexpr uint32_t AT_ROW_BYTES = AT_DK * 2;  // 1152 B gathered per row

constexpr int AT_SROW = 40;  // padded partial-score row (floats): conflict-free 64-bit access
constexpr int AT_PROW = 40;  // padded P row (bf16, 80 B): conflict-free ldmatrix

struct AttnSmem {
  alignas(128) uint8_t kv[AT_STAGES][AT_BK][AT_ROWB];  // 149504 B
  alignas(128) uint8_t q[AT_H][AT_ROWB];               // 18688 B
  alignas(16) float s_part[4][AT_H][AT_SROW];          // partial scores of the 4 dim quarters
  alignas(16) __nv_bfloat16 p[AT_H][AT_PROW];           // softmax numerators of the tile
  float alpha[AT_H];                                   // per-head rescale of the tile
  float fin_m[AT_H], fin_l[AT_H];                      // per-head final max / sum of an item
  alignas(16) int ibuf[2][AT_MAXK];                    // index lists: this item / the next
  unsigned vmask[AT_STAGES];                           // bit j: row j of the stage is valid
  int last[AT_STAGES];
  alignas(8) uint64_t full[AT_STAGES];
  uint64_t empty[AT_STAGES];
  uint64_t qfull, qempty;
  uint64_t ifull[2];
  uint64_t pitem;   // producers meet here at every item start
  uint64_t rawf[AT_STAGES];  // fp8 cache: a stage's raw rows have landed
  int abort;
};

struct AttnArgs {
  const __nv_bfloat16* q;   // [B, R, 16, 576]
  const __nv_bfloat16* kv;  // [B, Lkv, ld_kv]
  long ld_kv;
  const int* idx;           // [B, R, k]
  int B, R, Lkv, k;
  float scale_log2;         // softmax scale * log2(e)
  long items;               // B * R queries
  // Split mode (few queries): the B*R*tq (query, 32-key tile) pairs are cut into
  // gridDim.x equal contiguous ranges, one per CTA; each (query, range) piece
  // leaves a partial result in slot query * maxp + (its CTA - the query's first CTA).
  int split;
  int tq;                   // tiles per query: ceil(k / 32)
  int maxp;                 // partial slots per query
  long tot;                 // items * tq
  int idx_bulk;             // index rows 16-byte aligned: fetch each list with one bulk copy
  __nv_bfloat16* out;       // [B, R, 16, 512]   (not split)
  float* lse;               // [B, R, 16] or null (not split)
  float* part_o;            // [items * maxp, 16, 512] (split)
  float* part_ml;           // [items * maxp, 16, 2]   (split)
  // (the fp8 latent cache instance reads kv as rows of ld_kv bytes, each holding a
  // 656-byte row: 512 e4m3 codes, 4 fp32 group scales, 64 bf16 rope dims; it
  // dequantises them in shared memory to the bf16 row layout the consumers read)
};

// Packed sequences: query row r of the launch belongs to the last segment with
// seg.q0 <= r, whose latent rows start at row seg.k0 and number seg.len.  A kernel
// parameter of its own, so that AttnArgs stays small (the kernel reads it as
// instruction operands; a larger or addressable AttnArgs measured ~1 % slower
// each on the prefill attention).
struct AttnSegs {
  int nseg;
  AttnSeg seg[IC_MAXSEG];
};
struct AttnNoSegs {
  int unused;
};
template <bool SEGS>
using AttnSegParam = typename std::conditional<SEGS, AttnSegs, AttnNoSegs>::type;

// Latent rows of query row qrow: the first row's offset (in rows) and how many.
template <bool SEGS>
__device__ __forceinline__ void attn_kv_range(const AttnArgs& a, const AttnSegParam<SEGS>& sg,
                                              long qrow, long& row0, int& len) {
  if constexpr (!SEGS) {
    row0 = (qrow / a.R) * static_cast<long>(a.Lkv);
    len = a.Lkv;
  } else {
    int lo = 0, hi = sg.nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sg.seg[mid].q0 <= qrow)
        lo = mid;
      else
        hi = mid - 1;
    }
    row0 = sg.seg[lo].k0;
    len = sg.seg[lo].len;
  }
}

// Dequantises the fp8 rows of one tile stage that belong to producer warp pw (rows
// 8pw..8pw+7 with their bit set in `valid`) in place: a raw row (656 bytes at slot
// offset 512) becomes the 576 bf16 values of the row at offset 0, latent code *
// its group's scale rounded to bf16, rope copied.  Lane l owns latent dims
// 16l..16l+15 of every row (and rope bytes 16l..16l+15 for l < 8).  All eight
// rows are loaded before any store, so the overlapping expansion is safe and the
// rows' loads overlap; rows without a copy are left as they are (finite values
// of an earlier tile).
__device__ __forceinline__ void attn_dequant_rows(uint8_t* stage_rows, unsigned valid, int pw) {
  const int lane = threadIdx.x & 31;
  uint8_t* rows = stage_rows + 8 * pw * AT_ROWB;
  const unsigned mine = (valid >> (8 * pw)) & 0xFFu;
  uint4 codes[8], rope[8];
  float sc[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const uint8_t* row = rows + r * AT_ROWB;
    codes[r] = *reinterpret_cast<const uint4*>(row + 512 + 16 * lane);
    sc[r] = *reinterpret_cast<const float*>(row + 1024 + 4 * (lane / 8));
    rope[r] = lane < 8 ? *reinterpret_cast<const uint4*>(row + 1040 + 16 * lane)
                       : make_uint4(0, 0, 0, 0);
  }
  __syncwarp();
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (!((mine >> r) & 1u)) continue;
    uint8_t* row = rows + r * AT_ROWB;
    const __nv_fp8x2_storage_t* cp = reinterpret_cast<const __nv_fp8x2_storage_t*>(&codes[r]);
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // two codes -> two exact halves -> scaled, rounded to bf16
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(cp[i], __NV_E4M3);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
      __nv_bfloat162 v = __floats2bfloat162_rn(f.x * sc[r], f.y * sc[r]);
      o[i] = *reinterpret_cast<uint32_t*>(&v);
    }
    *reinterpret_cast<uint4*>(row + 32 * lane) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(row + 32 * lane + 16) = make_uint4(o[4], o[5], o[6], o[7]);
    if (lane < 8) *reinterpret_cast<uint4*>(row + 1024 + 16 * lane) = rope[r];
  }
  __syncwarp();
}

// CTA holding (query, tile) pair t of the split list: the largest c with
// floor(c * tot / G) <= t.
__host__ __device__ __forceinline__ long attn_cta_of(long t, long tot, long G) {
  return (t * G + G - 1) / tot;
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D (16x8 f32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct AttnItem {
  long qrow;
  int beg, end;  // entries [beg, end) of the query's index list
  long pslot;    // partial slot (split mode)
};
// Number of items of this CTA.
__device__ __forceinline__ long attn_nitems(const AttnArgs& a) {
  if (!a.split)
    return blockIdx.x < a.items ? (a.items - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const long lo = a.tot * blockIdx.x / gridDim.x, hi = a.tot * (blockIdx.x + 1) / gridDim.x;
  return hi > lo ? (hi - 1) / a.tq - lo / a.tq + 1 : 0;
}
// Item j of this CTA.
__device__ __forceinline__ AttnItem attn_item(const AttnArgs& a, long j) {
  AttnItem x;
  if (!a.split) {
    x.qrow = blockIdx.x + j * gridDim.x;
    x.beg = 0;
    x.end = a.k;
    x.pslot = x.qrow;
    return x;
  }
  const long lo = a.tot * blockIdx.x / gridDim.x, hi = a.tot * (blockIdx.x + 1) / gridDim.x;
  x.qrow = lo / a.tq + j;
  const long q0 = x.qrow * a.tq;
  const long t0 = lo > q0 ? lo : q0;
  const long t1 = hi < q0 + a.tq ? hi : q0 + a.tq;
  x.beg = static_cast<int>((t0 - q0) * AT_BK);
  x.end = min(static_cast<int>((t1 - q0) * AT_BK), a.k);
  if (x.end < x.beg) x.end = x.beg;
  x.pslot = x.qrow * a.maxp + (blockIdx.x - attn_cta_of(q0, a.tot, gridDim.x));
  return x;
}

// ---------------------------------------------------------------- producer warp
// Starts loading the index list of item `it` into ibuf[b]: one bulk copy when the
// rows are 16-byte aligned (k % 4 == 0), else plain loads by the warp.
__device__ __forceinline__ void attn_load_indices(AttnSmem& sm, const AttnArgs& a, long it, int b,
                                                  bool bulk) {
  const int lane = threadIdx.x & 31;
  const AttnItem x = attn_item(a, it);
  const int cnt = x.end - x.beg;
  const int* src = a.idx + x.qrow * a.k + x.beg;
  if (bulk) {
    if (lane == 0) {
      const uint32_t bar = smem_u32(&sm.ifull[b]);
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>(cnt) * 4u);
      if (cnt > 0) bulk_g2s(smem_u32(&sm.ibuf[b][0]), src, static_cast<uint32_t>(cnt) * 4u, bar);
    }
  } else {
    for (int j = lane; j < cnt; j += 32) sm.ibuf[b][j] = __ldg(src + j);
    __syncwarp();
  }
}

// Four producer warps walk the same items and tiles in lock step (they wait on the
// same stage barriers); producer pw issues the bulk copies of rows 8pw..8pw+7 of
// every tile -- one warp's bulk copies issue one lane at a time, so spreading a
// tile over four warps quadruples the gather issue rate.  Producer 0 also owns
// the per-item work: the next index list, the queries, the stage flags.
// KV8: fp8 latent rows; SEGS: packed sequences (separate instances, so that the
// bf16 form of one batch compiles without either)
template <bool KV8, bool SEGS>
__device__ __forceinline__ void attn_producer(AttnSmem& sm, const AttnArgs& a,
                                              const AttnSegParam<SEGS>& sg) {
  const int lane = threadIdx.x & 31;
  const int pw = (threadIdx.x - AT_CONSUMERS) >> 5;
  volatile int* abort = &sm.abort;
  const bool bulk = a.idx_bulk != 0;
  int stage = 0;
  uint32_t ph = 0;
  int qloads = 0;
  long issued = 0;
  uint32_t iph[2] = {0u, 0u};
  int ipending[2] = {0, 0};
  const uint32_t kv0 = smem_u32(&sm.kv[0][0][0]);
  const bool mine = (lane >> 3) == pw;  // this lane issues its row's copy
  int ib = 0;
  long nitem = 0;
  const long nj = attn_nitems(a);
  // fp8 cache: the stage, phase and valid rows of the tile whose raw rows are the
  // next to dequantise (one tile behind the copies, so that they overlap)
  int pend_stage = -1;
  uint32_t pend_ph = 0;
  unsigned pend_valid = 0u;
  auto dequant_pending = [&]() -> bool {
    if (pend_stage < 0) return true;
    if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.rawf[pend_stage]), pend_ph, abort,
                                           kErrTimeoutProducer)))
      return false;
    attn_dequant_rows(&sm.kv[pend_stage][0][0], pend_valid, pw);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&sm.full[pend_stage]));
    pend_stage = -1;
    return true;
  };
  if (pw == 0 && nj > 0) {
    attn_load_indices(sm, a, 0, 0, bulk);
    ipending[0] = bulk;
  }
  for (long it = 0; it < nj; ++it, ib ^= 1) {
    const AttnItem x = attn_item(a, it);
    const int cnt = x.end - x.beg;
    long kr0;
    int lkv;
    attn_kv_range<SEGS>(a, sg, x.qrow, kr0, lkv);
    const __nv_bfloat16* kvb = a.kv + kr0 * a.ld_kv;
    const uint8_t* kvb8 = reinterpret_cast<const uint8_t*>(a.kv) + kr0 * a.ld_kv;
    // every producer is done with the previous item (and its index list)
    if (lane == 0) mbar_arrive(smem_u32(&sm.pitem));
    if (!mbar_wait(smem_u32(&sm.pitem), static_cast<uint32_t>(nitem & 1), abort, kErrTimeoutProducer))
      break;
    ++nitem;
    // the next item's list streams in while this one's rows are gathered
    const long nit = it + 1;
    if (pw == 0 && nit < nj) {
      attn_load_indices(sm, a, nit, ib ^ 1, bulk);
      ipending[ib ^ 1] = bulk;
    }
    if (bulk) {
      if (!mbar_wait(smem_u32(&sm.ifull[ib]), iph[ib], abort, kErrTimeoutProducer)) break;
      iph[ib] ^= 1;
      ipending[ib] = 0;
    }
    const int* ilist = sm.ibuf[ib];
    // trailing -1 entries need no tiles: the last valid entry of the list
    int lv = -1;
    for (int j = lane; j < cnt; j += 32) {
      const int s = ilist[j];
      if (s >= 0 && s < lkv) lv = j;
    }
    lv = __reduce_max_sync(0xffffffffu, lv);
    const int ntiles = (lv >= 0) ? lv / AT_BK + 1 : 0;
    if (pw == 0) {
      // the item's queries, once the consumers hold the previous ones in registers
      if (qloads > 0 &&
          !mbar_wait(smem_u32(&sm.qempty), (qloads - 1) & 1, abort, kErrTimeoutProducer))
        break;
      if (lane == 0) mbar_arrive_expect_tx(smem_u32(&sm.qfull), AT_H * AT_ROW_BYTES);
      __syncwarp();
      if (lane < AT_H)
        bulk_g2s(smem_u32(&sm.q[lane][0]), a.q + (x.qrow * AT_H + lane) * AT_DK, AT_ROW_BYTES,
                 smem_u32(&sm.qfull));
      ++qloads;
    }
    const int nt = ntiles > 0 ? ntiles : 1;  // an empty item still ends with one (empty) tile
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      if (!mbar_wait(smem_u32(&sm.empty[stage]), ph ^ 1, abort, kErrTimeoutProducer)) {
        ok = false;
        break;
      }
      const int j = t * AT_BK + lane;
      int s = (t < ntiles && j < cnt) ? ilist[j] : -1;
      if (!in_bounds(s >= -1 && s < lkv, kErrBoundsGather) || s >= lkv) s = -1;
      const unsigned valid = __ballot_sync(0xffffffffu, s >= 0);
      if (pw == 0 && lane == 0) {
        sm.vmask[stage] = valid;
        sm.last[stage] = (t == nt - 1);
      }
      if constexpr (KV8) {
        // the raw fp8 row lands in the slot's last 656 bytes; the warp dequantises
        // its rows of the previous tile while these copies are in flight
        const uint32_t rb = smem_u32(&sm.rawf[stage]);
        if (lane == 0)
          mbar_arrive_expect_tx(rb, __popc(valid & (0xFFu << (8 * pw))) * KV8_ROW_BYTES);
        __syncwarp();
        if (mine && s >= 0)
          bulk_g2s(kv0 + (stage * AT_BK + lane) * AT_ROWB + (AT_ROWB - KV8_ROW_BYTES),
                   kvb8 + static_cast<long>(s) * a.ld_kv, KV8_ROW_BYTES, rb);
        if (!dequant_pending()) {
          ok = false;
          break;
        }
        pend_stage = stage;
        pend_ph = ph;
        pend_valid = valid;
      } else {
        const uint32_t fb = smem_u32(&sm.full[stage]);
        if (lane == 0)
          mbar_arrive_expect_tx(fb, __popc(valid & (0xFFu << (8 * pw))) * AT_ROW_BYTES);
        __syncwarp();
        if (mine && s >= 0)
          bulk_g2s(kv0 + (stage * AT_BK + lane) * AT_ROWB, kvb + static_cast<long>(s) * a.ld_kv,
                   AT_ROW_BYTES, fb);
      }
      ++issued;
      if (++stage == AT_STAGES) {
        stage = 0;
        ph ^= 1;
      }
    }
    if (!ok) break;
  }
  if (KV8 && !*abort) (void)dequant_pending();  // the last tile
  if (*abort) {
    // let every copy still in flight land before the CTA exits
    volatile int never = 0;
    const long n = issued < AT_STAGES ? issued : AT_STAGES;
    for (long j = issued - n; j < issued; ++j)
      (void)mbar_wait(smem_u32(KV8 ? &sm.rawf[j % AT_STAGES] : &sm.full[j % AT_STAGES]),
                      static_cast<uint32_t>((j / AT_STAGES) & 1), &never, kErrTimeoutDrain);
    if (qloads > 0) (void)mbar_wait(smem_u32(&sm.qfull), (qloads - 1) & 1, &never, kErrTimeoutDrain);
    for (int b2 = 0; b2 < 2; ++b2)
      if (ipending[b2]) (void)mbar_wait(smem_u32(&sm.ifull[b2]), iph[b2], &never, kErrTimeoutDrain);
  }
}

// ---------------------------------------------------------------- consumer warps
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Partial scores of this warp: Q[:, dims 144kq..+144] . K[keys 16kh..16kh+15] of the
// tile at kvbase, four accumulator chains (c[0..1]: keys +0..7, c[2..3]: keys +8..15).
__device__ __forceinline__ void attn_qk(uint32_t kvbase, const uint32_t (&qa)[9][4], int kq,
                                        int kh, int lane, float (&c)[4][4]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) c[u][0] = c[u][1] = c[u][2] = c[u][3] = 0.f;
  const int krow = 16 * kh + (lane & 7) + 8 * (lane >> 4);
  const uint32_t rowaddr = kvbase + krow * AT_ROWB;
#pragma unroll
  for (int j = 0; j < 9; ++j) {
    uint32_t b0, b1, b2, b3;
    const int col = kq * 144 + 16 * j + 8 * ((lane >> 3) & 1);
    ldsm_x4(rowaddr + col * 2, b0, b1, b2, b3);
    mma_bf16(c[(j & 1)], qa[j], b0, b1);
    mma_bf16(c[2 + (j & 1)], qa[j], b2, b3);
  }
}

__device__ __forceinline__ void attn_store_partial(float* sp, const float (&c)[4][4], int kh,
                                                   int g, int cq) {
  const int k0 = 16 * kh + 2 * cq;
  *reinterpret_cast<float2*>(sp + g * AT_SROW + k0) =
      make_float2(c[0][0] + c[1][0], c[0][1] + c[1][1]);
  *reinterpret_cast<float2*>(sp + (g + 8) * AT_SROW + k0) =
      make_float2(c[0][2] + c[1][2], c[0][3] + c[1][3]);
  *reinterpret_cast<float2*>(sp + g * AT_SROW + k0 + 8) =
      make_float2(c[2][0] + c[3][0], c[2][1] + c[3][1]);
  *reinterpret_cast<float2*>(sp + (g + 8) * AT_SROW + k0 + 8) =
      make_float2(c[2][2] + c[3][2], c[2][3] + c[3][3]);
}

// O[:, 64w..64w+64) = alpha O + P V for the tile at kvbase (P, alpha from shared).
__device__ __forceinline__ void attn_pv(uint32_t kvbase, uint32_t pbase, float al0, float al1,
                                        int warp, int lane, float (&o)[8][4]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    o[i][0] *= al0;
    o[i][1] *= al0;
    o[i][2] *= al1;
    o[i][3] *= al1;
  }
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    uint32_t pa[4];
    const int pr = (lane & 7) + 8 * ((lane >> 3) & 1);
    ldsm_x4(pbase + (pr * AT_PROW + 16 * ks + 8 * (lane >> 4)) * 2, pa[0], pa[1], pa[2], pa[3]);
    const int vrow = 16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b0, b1, b2, b3;
      const int col = 64 * warp + 16 * np + 8 * (lane >> 4);
      ldsm_x4_t(kvbase + vrow * AT_ROWB + col * 2, b0, b1, b2, b3);
      mma_bf16(o[2 * np], pa, b0, b1);
      mma_bf16(o[2 * np + 1], pa, b2, b3);
    }
  }
}

// Per tile: QK partials -> shared -> barrier -> the next tile's QK is issued, then
// the softmax of heads 2w, 2w+1, done once by warp w (16 lanes per head, 2 keys
// per lane), runs while those MMAs execute -> P, alpha -> barrier -> P V by every
// warp.
__device__ __forceinline__ void attn_consumer(AttnSmem& sm, const AttnArgs& a) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort = &sm.abort;
  const int kq = warp >> 1, kh = warp & 1;  // QK: dim quarter, key half of the tile
  const int g = lane >> 2, cq = lane & 3;
  const int sh = 2 * warp + (lane >> 4);    // softmax: head of this lane
  const int sk = 2 * (lane & 15);           // and its two keys
  int stage = 0;
  uint32_t ph = 0;
  int qwaits = 0;
  int rel = -1;  // stage of the previous tile, released after the next partial barrier
  const long nj = attn_nitems(a);
  for (long it = 0; it < nj; ++it) {
    const AttnItem x = attn_item(a, it);
    if (!mbar_wait(smem_u32(&sm.qfull), qwaits & 1, abort, kErrTimeoutEpilogue)) return;
    ++qwaits;
    uint32_t qa[9][4];
    {
      const uint32_t qbase = smem_u32(&sm.q[0][0]);
      const int r = (lane & 7) + 8 * ((lane >> 3) & 1);
      const int cofs = 8 * (lane >> 4);
#pragma unroll
      for (int j = 0; j < 9; ++j) {
        const int col = kq * 144 + 16 * j + cofs;
        ldsm_x4(qbase + r * AT_ROWB + col * 2, qa[j][0], qa[j][1], qa[j][2], qa[j][3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&sm.qempty));
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;  // softmax state of head sh (its 16 lanes agree)

    if (!mbar_wait(smem_u32(&sm.full[stage]), ph, abort, kErrTimeoutEpilogue)) return;
    int cur = stage;
    int cur_last = sm.last[stage];
    unsigned cur_vm = sm.vmask[stage];
    {
      float c[4][4];
      attn_qk(smem_u32(&sm.kv[stage][0][0]), qa, kq, kh, lane, c);
      attn_store_partial(&sm.s_part[kq][0][0], c, kh, g, cq);
    }
    if (++stage == AT_STAGES) {
      stage = 0;
      ph ^= 1;
    }
    for (;;) {
      named_bar_sync(1, AT_CONSUMERS);  // B1: partials of cur complete, P V of prev done
      if (tid == 0 && rel >= 0) mbar_arrive(smem_u32(&sm.empty[rel]));
      // ---- the next tile's QK goes out first: its MMAs run under this tile's softmax
      const bool more = !cur_last;
      float c[4][4];
      int nxt = -1, nxt_last = 1;
      unsigned nxt_vm = 0u;
      if (more) {
        if (!mbar_wait(smem_u32(&sm.full[stage]), ph, abort, kErrTimeoutEpilogue)) return;
        nxt = stage;
        nxt_last = sm.last[stage];
        nxt_vm = sm.vmask[stage];
        attn_qk(smem_u32(&sm.kv[stage][0][0]), qa, kq, kh, lane, c);
        if (++stage == AT_STAGES) {
          stage = 0;
          ph ^= 1;
        }
      }
      // ---- softmax of head sh over keys sk, sk+1 (done once)
      {
        float2 z = make_float2(0.f, 0.f);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const float2 u = *reinterpret_cast<const float2*>(&sm.s_part[qq][sh][sk]);
          z.x += u.x;
          z.y += u.y;
        }
        const float z0 = ((cur_vm >> sk) & 1) ? z.x * a.scale_log2 : -INFINITY;
        const float z1 = ((cur_vm >> (sk + 1)) & 1) ? z.y * a.scale_log2 : -INFINITY;
        float t = fmaxf(z0, z1);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, off));
        const float n = fmaxf(m_run, t);
        const float al = (n == -INFINITY) ? 1.f : fast_exp2(m_run - n);
        const float bse = (n == -INFINITY) ? 0.f : n;
        const float e0 = fast_exp2(z0 - bse), e1 = fast_exp2(z1 - bse);
        float rs = e0 + e1;
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
        l_run = l_run * al + rs;
        m_run = n;
        *reinterpret_cast<uint32_t*>(&sm.p[sh][sk]) = pack_bf16(e0, e1);
        if ((lane & 15) == 0) sm.alpha[sh] = al;
      }
      named_bar_sync(1, AT_CONSUMERS);  // B2: P, alpha complete
      attn_pv(smem_u32(&sm.kv[cur][0][0]), smem_u32(&sm.p[0][0]), sm.alpha[g], sm.alpha[g + 8],
              warp, lane, o);
      rel = cur;
      if (!more) break;
      attn_store_partial(&sm.s_part[kq][0][0], c, kh, g, cq);
      cur = nxt;
      cur_last = nxt_last;
      cur_vm = nxt_vm;
    }

    // ---- item epilogue: head h's final max and sum live in warp h/2
    named_bar_sync(1, AT_CONSUMERS);  // every warp's P V of the item is done
    if ((lane & 15) == 0) {
      sm.fin_m[sh] = m_run;
      sm.fin_l[sh] = l_run;
    }
    named_bar_sync(1, AT_CONSUMERS);
    const float M0 = sm.fin_m[g], M1 = sm.fin_m[g + 8];
    const float L0 = sm.fin_l[g], L1 = sm.fin_l[g + 8];
    if (!a.split) {
      const float inv0 = L0 > 0.f ? 1.f / L0 : 0.f, inv1 = L1 > 0.f ? 1.f / L1 : 0.f;
      __nv_bfloat16* ob = a.out + x.qrow * (AT_H * AT_DV);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int d = 64 * warp + 8 * i + 2 * cq;
        *reinterpret_cast<uint32_t*>(ob + g * AT_DV + d) = pack_bf16(o[i][0] * inv0, o[i][1] * inv0);
        *reinterpret_cast<uint32_t*>(ob + (g + 8) * AT_DV + d) =
            pack_bf16(o[i][2] * inv1, o[i][3] * inv1);
      }
      if (a.lse && warp == 0 && cq == 0) {
        a.lse[x.qrow * AT_H + g] = L0 > 0.f ? (M0 + log2f(L0)) * 0.69314718055994531f : -INFINITY;
        a.lse[x.qrow * AT_H + g + 8] =
            L1 > 0.f ? (M1 + log2f(L1)) * 0.69314718055994531f : -INFINITY;
      }
    } else {
      const long ps = x.pslot;
      float* po = a.part_o + ps * (AT_H * AT_DV);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int d = 64 * warp + 8 * i + 2 * cq;
        *reinterpret_cast<float2*>(po + g * AT_DV + d) = make_float2(o[i][0], o[i][1]);
        *reinterpret_cast<float2*>(po + (g + 8) * AT_DV + d) = make_float2(o[i][2], o[i][3]);
      }
      if (warp == 0 && cq == 0) {
        a.part_ml[(ps * AT_H + g) * 2] = M0;
        a.part_ml[(ps * AT_H + g) * 2 + 1] = L0;
        a.part_ml[(ps * AT_H + g + 8) * 2] = M1;
        a.part_ml[(ps * AT_H + g + 8) * 2 + 1] = L1;
      }
    }
  }
}

template <bool KV8, bool SEGS>
__global__ void __launch_bounds__(AT_THREADS, 1)
    attn_mla_kernel(const AttnArgs a, const __grid_constant__ AttnSegParam<SEGS> sg) {
  extern __shared__ uint8_t at_smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(
      (reinterpret_cast<uintptr_t>(at_smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  if (threadIdx.x == 0) {
    for (int s = 0; s < AT_STAGES; ++s) {
      mbar_init(smem_u32(&sm.full[s]), AT_PRODUCERS);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.qfull), 1);
    mbar_init(smem_u32(&sm.qempty), AT_CONSUMERS / 32);
    mbar_init(smem_u32(&sm.ifull[0]), 1);
    mbar_init(smem_u32(&sm.ifull[1]), 1);
    mbar_init(smem_u32(&sm.pitem), AT_PRODUCERS);
    if (KV8)
      for (int st = 0; st < AT_STAGES; ++st) mbar_init(smem_u32(&sm.rawf[st]), AT_PRODUCERS);
    sm.abort = 0;
    fence_barrier_init();
  }
  // rows a tile never receives (index < 0) keep whatever the buffer held; start from
  // zeros so that those stale rows are always finite (their softmax weight is 0)
  uint4* z = reinterpret_cast<uint4*>(&sm.kv[0][0][0]);
  for (int i = threadIdx.x; i < static_cast<int>(sizeof(sm.kv) / 16); i += blockDim.x)
    z[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  __syncthreads();
  grid_dep_wait();  // set-up above touches no global memory
  if (threadIdx.x >= AT_CONSUMERS)
    attn_producer<KV8, SEGS>(sm, a, sg);
  else
    attn_consumer(sm, a);
  __syncthreads();
}

// Merges the partial results of one query (its pieces in split mode): per head,
// M = max m_i, L = sum l_i 2^(m_i - M), O = sum O_i 2^(m_i - M) / L.  Each warp
// reads the pieces' (m, l) in parallel (lane i: pieces i and i + 32) and reduces
// them with shuffles; every thread accumulates its output dims over the pieces.
__global__ void attn_combine_kernel(const float* part_o, const float* part_ml, int maxp, long tot,
                                    int tq, int G, __nv_bfloat16* out, float* lse) {
  grid_dep_wait();
  const long qrow = blockIdx.x;
  const int h = blockIdx.y;
  const long c0 = attn_cta_of(qrow * tq, tot, G);
  int np = static_cast<int>(attn_cta_of((qrow + 1) * tq - 1, tot, G) - c0 + 1);  // <= 64
  if (!in_bounds(np <= 64, kErrBoundsMerge)) np = 64;
  const long s0 = qrow * maxp;
  // Each thread owns 4 adjacent output dims.  The first CMB_PRE pieces' partial
  // outputs are loaded before the weights are known, so their latency overlaps
  // the (m, l) reduction; later pieces (rare) are loaded as they are used.
  constexpr int CMB_PRE = 8;
  const float* po = part_o + (s0 * AT_H + h) * AT_DV;
  const long pstride = static_cast<long>(AT_H) * AT_DV;
  const int d = 4 * threadIdx.x;
  float4 pv[CMB_PRE];
#pragma unroll
  for (int i = 0; i < CMB_PRE; ++i)
    if (i < np) pv[i] = *reinterpret_cast<const float4*>(po + i * pstride + d);
  // Every warp reduces the pieces' (m, l) itself (lane i: pieces i and i + 32), so
  // no warp waits for another; the values are the same in every warp.
  const int lane = threadIdx.x & 31;
  float w0, w1, il;
  {
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    if (lane < np) {
      m0 = part_ml[((s0 + lane) * AT_H + h) * 2];
      l0 = part_ml[((s0 + lane) * AT_H + h) * 2 + 1];
    }
    if (lane + 32 < np) {
      m1 = part_ml[((s0 + lane + 32) * AT_H + h) * 2];
      l1 = part_ml[((s0 + lane + 32) * AT_H + h) * 2 + 1];
    }
    float M = fmaxf(m0, m1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    w0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - M);
    w1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M);
    float L = l0 * w0 + l1 * w1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    il = L > 0.f ? 1.f / L : 0.f;
    if (threadIdx.x == 0 && lse)
      lse[qrow * AT_H + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
  // weight of piece i (held by lane i % 32)
  auto wt = [&](int i) { return __shfl_sync(0xffffffffu, i < 32 ? w0 : w1, i & 31); };
  // even pieces accumulate into a0, odd ones into a1
  float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
  auto madd = [](float4& acc, float w, const float4& u) {
    acc.x += w * u.x;
    acc.y += w * u.y;
    acc.z += w * u.z;
    acc.w += w * u.w;
  };
#pragma unroll
  for (int i = 0; i < CMB_PRE; ++i)
    if (i < np) madd((i & 1) ? a1 : a0, wt(i), pv[i]);
  for (int i = CMB_PRE; i < np; ++i)
    madd((i & 1) ? a1 : a0, wt(i), *reinterpret_cast<const float4*>(po + i * pstride + d));
  uint32_t* o = reinterpret_cast<uint32_t*>(out + (qrow * AT_H + h) * AT_DV + d);
  o[0] = pack_bf16((a0.x + a1.x) * il, (a0.y + a1.y) * il);
  o[1] = pack_bf16((a0.z + a1.z) * il, (a0.w + a1.w) * il);
}

// Split plan for few queries: G CTAs over the items*tq (query, tile) pairs, each
// query cut into at most 64 pieces (G <= 63 * items keeps a range >= tq / 63 tiles).
struct SplitPlan {
  bool split;
  int G, tq, maxp;
  long tot;
};
static SplitPlan split_plan(long items, int k) {
  SplitPlan p{false, 0, 0, 0, 0};
  const long nsm = num_sms();
  if (items <= 0 || items >= 4 * nsm) return p;  // enough queries for every SM
  p.tq = (k + AT_BK - 1) / AT_BK;
  p.tot = items * p.tq;
  long G = nsm;
  if (G > p.tot) G = p.tot;
  if (G > 63 * items) G = 63 * items;
  p.G = static_cast<int>(G);
  int mx = 1;
  for (long q = 0; q < items; ++q) {
    const long np = attn_cta_of((q + 1) * p.tq - 1, p.tot, G) - attn_cta_of(q * p.tq, p.tot, G) + 1;
    if (np > mx) mx = static_cast<int>(np);
  }
  p.maxp = mx;
  p.split = p.G > 1 || items > 1;
  return p;
}

size_t attn_mla_ws_bytes(int batch, int rows, int k) {
  const long items = static_cast<long>(batch) * rows;
  const SplitPlan p = split_plan(items, k);
  if (!p.split) return 0;
  return static_cast<size_t>(items) * p.maxp * AT_H * (AT_DV + 2) * sizeof(float);
}

template <bool KV8, bool SEGS>
static ic_status launch_attn_inst(const AttnArgs& a, const AttnSegParam<SEGS>& sg, long grid,
                                  cudaStream_t stream) {
  const int smem = static_cast<int>(sizeof(AttnSmem)) + 128;
  ic_status st = cuda_check(cudaFuncSetAttribute(attn_mla_kernel<KV8, SEGS>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                            "cudaFuncSetAttribute(attn)");
  if (st) return st;
  return cuda_check(launch_dep(attn_mla_kernel<KV8, SEGS>, dim3(static_cast<unsigned>(grid)),
                               dim3(AT_THREADS), smem, stream, 1, a, sg),
                    "attn_mla_kernel launch");
}

ic_status launch_attn_mla(const void* q, const void* kv, long ld_kv, const int* idx, int batch,
                          int rows, int Lkv, int k, float scale, void* out, float* lse, void* ws,
                          size_t ws_bytes, long long valid_entries, cudaStream_t stream,
                          bool kv8, const AttnSeg* segs, int nseg) {
  const long items = static_cast<long>(batch) * rows;
  if (nseg < 0 || nseg > IC_MAXSEG || (nseg > 0 && (batch != 1 || !segs)))
    return fail(IC_ERR_INVALID_ARG, "attn: bad segment list (%d)", nseg);
  if (items == 0) return IC_OK;
  SplitPlan p = split_plan(items, k);
  const size_t need = static_cast<size_t>(items) * p.maxp * AT_H * (AT_DV + 2) * sizeof(float);
  // no room, or a workspace the merge's 16-byte loads cannot use: one CTA per query
  if (p.split && (ws == nullptr || need > ws_bytes || reinterpret_cast<uintptr_t>(ws) % 16 != 0))
    p.split = false;
  AttnArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kv = static_cast<const __nv_bfloat16*>(kv);  // fp8 cache: rows of ld_kv bytes
  a.ld_kv = ld_kv;
  a.idx = idx;
  a.B = batch;
  a.R = rows;
  a.Lkv = Lkv;
  a.k = k;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.items = items;
  a.split = p.split ? 1 : 0;
  a.tq = p.tq;
  a.maxp = p.maxp;
  a.tot = p.tot;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.idx_bulk = (k % 4 == 0) && (reinterpret_cast<uintptr_t>(idx) % 16 == 0);
  a.part_o = p.split ? static_cast<float*>(ws) : nullptr;
  a.part_ml = p.split ? static_cast<float*>(ws) + items * p.maxp * AT_H * AT_DV : nullptr;
  const long grid = p.split ? p.G : (items < num_sms() ? items : num_sms());
  ic_status st;
  if (nseg > 0) {
    AttnSegs sg;
    sg.nseg = nseg;
    for (int j = 0; j < nseg; ++j) sg.seg[j] = segs[j];
    st = kv8 ? launch_attn_inst<true, true>(a, sg, grid, stream)
             : launch_attn_inst<false, true>(a, sg, grid, stream);
  } else {
    const AttnNoSegs sg{0};
    st = kv8 ? launch_attn_inst<true, false>(a, sg, grid, stream)
             : launch_attn_inst<false, false>(a, sg, grid, stream);
  }
  if (st) return st;
  // algorithmic bytes: each selected latent row gathered once, q read once, out written once
  const double ve = valid_entries >= 0 ? static_cast<double>(valid_entries)
                                       : static_cast<double>(items) * k;
  const double io = static_cast<double>(items) * AT_H * (AT_DK + AT_DV) * 2.0;
  trace_launch(kv8 ? kKindAttnMlaKv8 : kKindAttnMla, stream,
               ve * (kv8 ? KV8_ROW_BYTES : AT_DK * 2.0) + io + 4.0 * static_cast<double>(items) * k);
  if (!p.split) return IC_OK;
  static_assert(AT_DV == 4 * 128, "combine: 128 threads x 4 dims");
  st = cuda_check(launch_dep(attn_combine_kernel, dim3(static_cast<unsigned>(items), AT_H), dim3(128),
                             0, stream, 1, a.part_o, a.part_ml, p.maxp, p.tot, p.tq, p.G, a.out, lse),
                  "attn_combine_kernel launch");
  if (!st) {
    // pieces actually written: every (query, CTA) overlap
    const double pieces = static_cast<double>(p.G) + static_cast<double>(items) - 1.0;
    trace_launch(kKindAttnCombine, stream,
                 pieces * AT_H * (AT_DV + 2) * 4.0 + static_cast<double>(items) * AT_H * AT_DV * 2.0);
  }
  return st;
}

// ------------------------------------------------------------------ fp32 (MQA) form
// One CTA per query row, CUDA cores: small shapes only (the fp32 workload has
// 4 heads of dim 64 over k = 64 keys).
template <bool SEGS>
__global__ void attn_f32_kernel(const float* q, const float* kv, long ld_kv, const float* v,
                                const int* idx, int R, int heads, int dk, int dv, int Lkv_, int k,
                                float scale, float* out, float* lse,
                                const __grid_constant__ AttnSegParam<SEGS> sg) {
  extern __shared__ float f32_smem[];
  float* qs = f32_smem;        // [dk]
  float* z = f32_smem + dk;    // [k]
  __shared__ float red[32];
  const long qrow = blockIdx.x;
  long r0;
  int Lkv;
  if constexpr (SEGS) {
    int lo = 0, hi = sg.nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sg.seg[mid].q0 <= qrow)
        lo = mid;
      else
        hi = mid - 1;
    }
    r0 = sg.seg[lo].k0;
    Lkv = sg.seg[lo].len;
  } else {
    r0 = (qrow / R) * static_cast<long>(Lkv_);
    Lkv = Lkv_;
  }
  const int* irow = idx + qrow * k;
  const float* kvb = kv + r0 * ld_kv;
  const float* vb = v + r0 * dv;
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int h = 0; h < heads; ++h) {
    const float* qh = q + (qrow * heads + h) * dk;
    for (int d = tid; d < dk; d += nt) qs[d] = qh[d];
    __syncthreads();
    float lmax = -INFINITY;
    for (int j = tid; j < k; j += nt) {
      const int s = irow[j];
      float zz = -INFINITY;
      if (s >= 0 && s < Lkv) {
        const float* kr = kvb + static_cast<long>(s) * ld_kv;
        float acc = 0.f;
        for (int d = 0; d < dk; ++d) acc = fmaf(qs[d], kr[d], acc);
        zz = acc * scale;
      }
      z[j] = zz;
      lmax = fmaxf(lmax, zz);
    }
    for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    if ((tid & 31) == 0) red[tid >> 5] = lmax;
    __syncthreads();
    float M = -INFINITY;
    for (int i = 0; i < (nt + 31) / 32; ++i) M = fmaxf(M, red[i]);
    __syncthreads();
    float lsum = 0.f;
    for (int j = tid; j < k; j += nt) {
      const float e = (M == -INFINITY) ? 0.f : expf(z[j] - M);
      z[j] = e;
      lsum += e;
    }
    for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    if ((tid & 31) == 0) red[tid >> 5] = lsum;
    __syncthreads();
    float L = 0.f;
    for (int i = 0; i < (nt + 31) / 32; ++i) L += red[i];
    const float inv = L > 0.f ? 1.f / L : 0.f;
    for (int d = tid; d < dv; d += nt) {
      float acc = 0.f;
      for (int j = 0; j < k; ++j) {
        const int s = irow[j];
        if (s >= 0 && s < Lkv) acc = fmaf(z[j], vb[static_cast<long>(s) * dv + d], acc);
      }
      out[(qrow * heads + h) * dv + d] = acc * inv;
    }
    if (lse && tid == 0) lse[qrow * heads + h] = L > 0.f ? M + logf(L) : -INFINITY;
    __syncthreads();
  }
}

ic_status launch_attn_f32(const float* q, const float* kv, long ld_kv, const float* v,
                          const int* idx, int batch, int rows, int heads, int dk, int dv, int Lkv,
                          int k, float scale, float* out, float* lse, cudaStream_t stream,
                          const AttnSeg* segs, int nseg) {
  const long items = static_cast<long>(batch) * rows;
  if (items == 0) return IC_OK;
  if (nseg < 0 || nseg > IC_MAXSEG || (nseg > 0 && (batch != 1 || !segs)))
    return fail(IC_ERR_INVALID_ARG, "attn: bad segment list (%d)", nseg);
  const int smem = (dk + k) * static_cast<int>(sizeof(float));
  ic_status st;
  if (nseg > 0) {
    AttnSegs sg;
    sg.nseg = nseg;
    for (int j = 0; j < nseg; ++j) sg.seg[j] = segs[j];
    st = cuda_check(cudaFuncSetAttribute(attn_f32_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                    "cudaFuncSetAttribute(attn_f32)");
    if (st) return st;
    attn_f32_kernel<true><<<static_cast<unsigned>(items), 128, smem, stream>>>(
        q, kv, ld_kv, v, idx, rows, heads, dk, dv, Lkv, k, scale, out, lse, sg);
  } else {
    st = cuda_check(cudaFuncSetAttribute(attn_f32_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                    "cudaFuncSetAttribute(attn_f32)");
    if (st) return st;
    attn_f32_kernel<false><<<static_cast<unsigned>(items), 128, smem, stream>>>(
        q, kv, ld_kv, v, idx, rows, heads, dk, dv, Lkv, k, scale, out, lse, AttnNoSegs{0});
  }
  st = cuda_check(cudaGetLastError(), "attn_f32_kernel launch");
  if (!st)
    trace_launch(kKindAttnF32, stream,
                 4.0 * static_cast<double>(items) * (k * (dk + dv) + heads * (dk + dv) + k));
  return st;
}

}  // namespace ic
