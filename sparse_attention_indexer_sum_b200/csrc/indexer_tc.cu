// indexer_tc.cu -- lightning-indexer scores on the sm_100a tensor cores.
//
// Computes I[b, r, s] = sum_h w[b,r,h] * max(0, q[b,r,h,:] . k[b,s,:]) for the
// causal keys s <= pos0 + r ("IndexCache: Wie DeepSeek O(NL^2)-Kosten in Sparse
// Attention um 75% reduziert", section "Wie der Indexer funktioniert": score,
// ReLU gate, then top-k; the head-weighted sum is this library's reading).
//
// Mapping.  The contraction runs transposed: the MMA's M dimension is 128 KEYS
// (operand A = a tile of k), its N dimension is TPM query tokens x 64 heads
// (operand B = the resident block of q), K = the 128-dim head dimension.  The
// fp32 accumulator D[key, (token, head)] lives in TMEM with one key per lane,
// so the epilogue thread that owns a key reads the 64 head values of a token
// from its own lane and reduces ReLU * w over heads entirely in registers:
// no cross-lane reduction, and the L x L score matrix is produced one
// 128-key x TPM-token tile at a time, never formed as a whole.
//
// Pipeline (one persistent CTA per SM, warp-specialised):
//   warp 0      TMA producer: q block (once per query block) + a ring of key tiles
//   warp 1      MMA issuer: one thread issues tcgen05.mma into a ring of TMEM
//               accumulators, commits to mbarriers (one-token blocks: warps 1
//               and 2, alternating key tiles)
//   the rest    epilogue: tcgen05.ld -> ReLU -> w-weighted head sum -> causal
//               mask -> fp32 score stores (coalesced, one key per lane)
// The work is the list of (query block, key tile) pairs of the causal
// triangle; CTA c takes the c-th equal share of that list, so every SM gets
// the same number of MMA tiles whatever the triangle's shape.
//
// fp8 variant: q, k are e4m3 codes with per-(token, head) and per-token fp32
// scales; the MMA runs kind::f8f6f4 and the scales are folded into the
// epilogue: I = k_scale[s] * sum_h (w * q_scale)[h] * ReLU(q8 . k8).
#include <cudaTypedefs.h>

#include <mutex>
#include <vector>

#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

struct IdxTcArgs {
  const float* w;        // [B, R, 64]
  const float* q_scale;  // [B, R, 64] (fp8) or null
  const float* k_scale;  // [B, Lk] (fp8) or null
  float* scores;         // [B, R, ld]
  long ld;
  int B, R, Lk;
  long pos0;
  int qb_per_batch;      // ceil(R / TPM)
  int nqb;               // B * qb_per_batch
  long total_tiles;
  // Fused top-k (one query per sequence): every (row, CTA piece) leaves its
  // candidates in a slot of `cslots`; topk_merge_kernel selects.
  uint8_t* cslots;
  int maxp;              // CTA pieces per row
  int topk;              // k of the selection
  // Segments (packed sequences of different lengths; 0 = the uniform batch above).
  // Segment j holds seg[j].R query rows at positions seg[j].pos0.. over seg[j].Lk
  // keys: its query rows are rows qrow0.. of q / w / q_scale, its keys rows krow0..
  // of k / k_scale, its score rows rows orow0.. of scores; its query blocks are
  // qb0 .. qb0 + ceil(R / TPM) - 1.  Used by the multi-token instances only.
  int nseg;
  IdxSeg seg[IC_MAXSEG];
};

// Fused top-k slot: a 64-byte header {int count; int pad; uint64 tau; uint64 max}
// and then `count` selection keys (select_key) of one row's keys in one CTA:
// every key of that share with selection key >= tau; when tau is not 0, at least
// k of them; max is the largest.
constexpr int FUSED_CB = 8192;                         // candidate buffer of a CTA
constexpr size_t FUSED_SLOT_BYTES = 64 + 8 * FUSED_CB;
constexpr int FUSED_SELW = 4;                          // selector warps
constexpr int FUSED_XINTS = 104;                       // selector scratch ints

template <bool FP8, int TPM, bool FUSED = false>
struct IdxCfg {
  static constexpr int H = 64, D = 128;
  static constexpr int BM = 128;                   // keys per tile (MMA M)
  static constexpr int N = 64 * TPM;               // MMA N: TPM tokens x 64 heads
  static constexpr int EB = FP8 ? 1 : 2;           // bytes per element
  static constexpr int ROWB = D * EB;              // bytes per 128-dim row
  static constexpr int KBLK = ROWB / 128;          // 128-byte swizzle blocks per row
  static constexpr int ELEMS_128B = 128 / EB;      // elements per 128-byte block
  static constexpr int KSTEPS = FP8 ? 4 : 8;       // MMAs per tile (K = 32 / 16 each)
  static constexpr int A_BYTES = BM * ROWB;        // one key tile
  static constexpr int Q_BYTES = N * ROWB;         // the query block
  // the fused top-k's staging ring and candidate buffer take the shared memory
  // of some key ring stages
  static constexpr int STAGES = FP8 ? (FUSED ? 6 : 8) : 4;
  static constexpr int NACC = (TPM == 4) ? 2 : 6;  // TMEM accumulators in the ring
  static constexpr int TMEM_COLS = (NACC * N <= 256) ? 256 : 512;
  // epilogue warps per TMEM lane quadrant: with fp8 keys the tiles come twice as
  // fast and four warps per quadrant (one token each) hide more of the TMEM round
  // trips than two (measured 5% faster on long e4m3 rows, 6% slower with bf16)
  static constexpr int EPG = (TPM == 4) ? (FP8 ? 4 : 2) : 1;
  // Epilogue warp sets: set j takes the accumulator slots a with a % NSETS == j, so
  // each set sees every use of its slots in order.  One-token blocks (decode) have
  // little epilogue work per tile; several sets overlap consecutive tiles.
  // (the fused instance keeps two sets: with its selector warps, three sets would
  // cap every thread at 96 registers and spill; two measured 4 % faster)
  static constexpr int NSETS = (TPM == 4) ? 1 : (FUSED ? 2 : 3);
  static constexpr int SETW = 4 * EPG;             // warps per set
  static constexpr int NEPI = SETW * NSETS;
  static constexpr int TOK_PER_EW = TPM / EPG;     // tokens per epilogue warp
  // MMA-issuing warps: tile i is issued by warp 1 + i % MMAW.  With N = 64
  // (one-token blocks) a tile's four or eight MMAs are short, and one thread's
  // issue loop (waits, MMAs, commits) sets the pace; two threads alternate
  // tiles.  With N = 256 the tensor pipe itself is the limit.
  static constexpr int MMAW = (TPM == 1) ? 2 : 1;
  // Each MMA warp must wait on every phase of the full barriers of the stages it
  // reads: with STAGES a multiple of MMAW, all uses of a stage fall to the same
  // warp.  Otherwise a warp waits on parity p two phases apart while the other
  // warp's phase in between may not have completed yet, and the parity test
  // passes on the older phase (the ring would run ahead of its data).
  static_assert(STAGES % MMAW == 0, "every use of a ring stage falls to one MMA warp");
  static_assert(NACC % MMAW == 0, "every use of an accumulator falls to one MMA warp");
  static constexpr int EPI_W0 = 1 + MMAW;  // first epilogue warp
  // fused top-k: selector warps after the epilogue warps consume the tiles'
  // candidate keys from a staging ring of NSTG tiles (a multiple of NSETS, so that
  // every use of a staging slot falls to the same epilogue set)
  static constexpr int NSEL = FUSED ? FUSED_SELW : 0;
  static constexpr int SEL_W0 = EPI_W0 + NEPI;
  static constexpr int NSTG = FUSED ? (FP8 ? 24 : 12) : 0;
  static constexpr int THREADS = 32 * (EPI_W0 + NEPI + NSEL);
  // TMEM columns an epilogue thread loads at a time: 16, so that the head
  // weights of both its tokens fit in registers beside them
  static constexpr int EPI_COLS = 16;  // matches tmem_ld16
  static constexpr int OFF_A = 0;
  static constexpr int OFF_Q = STAGES * A_BYTES;
  static constexpr int OFF_W = OFF_Q + Q_BYTES;
  static constexpr int W_FLOATS = NEPI * TOK_PER_EW * 64;
  static constexpr int OFF_BAR = OFF_W + W_FLOATS * 4;
  static constexpr int NBAR = 2 * STAGES + 2 * NACC + 3 + 2 * NSTG + (FUSED ? 2 : 0);
  // fused top-k: the staging ring (per tile, each epilogue warp's candidate
  // selection keys, packed, and their count), the candidate buffer of FUSED_CB
  // selection keys, a 256-bin radix histogram and FUSED_XINTS ints of scratch
  static constexpr int CB = FUSED ? FUSED_CB : 0;
  static constexpr int OFF_STG = (OFF_BAR + NBAR * 8 + 15) / 16 * 16;
  static constexpr int OFF_SCNT = OFF_STG + NSTG * BM * 8;
  static constexpr int OFF_CBUF = OFF_SCNT + NSTG * 16;
  static constexpr int OFF_CHIST = OFF_CBUF + CB * 8;
  static constexpr int OFF_CX = OFF_CHIST + (FUSED ? 256 * 4 : 0);
  static constexpr int OFF_MISC = OFF_CX + (FUSED ? FUSED_XINTS * 4 : 0);
  static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;  // + alignment slack
  static_assert(!FUSED || (TPM == 1 && NSTG % NSETS == 0 && SETW == 4),
                "the fused top-k runs in the one-token instance");
  static_assert(A_BYTES % 1024 == 0 && Q_BYTES % 1024 == 0, "swizzle atoms need 1 KB alignment");
  static_assert(N <= 256 && N % 16 == 0, "MMA N");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(NACC * N <= TMEM_COLS, "TMEM");
  static_assert(NACC % NSETS == 0, "each epilogue set owns whole accumulator slots");
};

// Where query block qb lies: its first query row's index in its segment (ql *
// TPM), the segment's rows, positions and keys, and the row offsets of its query,
// key and score rows.
struct QbInfo {
  long qrow0, krow0, orow0, pos0;
  int R, Lk, ql;
};
template <int TPM, bool SEGS>
__host__ __device__ __forceinline__ QbInfo qb_info(const IdxTcArgs& a, int qb) {
  QbInfo x;
  if (SEGS) {
    int lo = 0, hi = a.nseg - 1;  // the last segment with qb0 <= qb
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.seg[mid].qb0 <= qb)
        lo = mid;
      else
        hi = mid - 1;
    }
    const IdxSeg& g = a.seg[lo];
    x.ql = qb - g.qb0;
    x.qrow0 = g.qrow0;
    x.krow0 = g.krow0;
    x.orow0 = g.orow0;
    x.pos0 = g.pos0;
    x.R = g.R;
    x.Lk = g.Lk;
  } else {
    const int b = qb / a.qb_per_batch;
    x.ql = qb - b * a.qb_per_batch;
    x.qrow0 = static_cast<long>(b) * a.R;
    x.orow0 = x.qrow0;
    x.krow0 = static_cast<long>(b) * a.Lk;
    x.pos0 = a.pos0;
    x.R = a.R;
    x.Lk = a.Lk;
  }
  return x;
}

template <int TPM, bool SEGS>
__host__ __device__ __forceinline__ int qb_tiles(const IdxTcArgs& a, int qb) {
  const QbInfo x = qb_info<TPM, SEGS>(a, qb);
  const int r_last = min(x.ql * TPM + TPM, x.R) - 1;
  long keys = x.pos0 + r_last + 1;
  if (keys > x.Lk) keys = x.Lk;
  return static_cast<int>((keys + 127) / 128);
}

template <int TPM, bool SEGS>
struct WorkIt {
  int qb, kt, nt;
  __device__ __forceinline__ void advance(const IdxTcArgs& a) {
    if (++kt >= nt) {
      kt = 0;
      ++qb;
      nt = (qb < a.nqb) ? qb_tiles<TPM, SEGS>(a, qb) : 0;
    }
  }
};

// Drain wait used only after an abort: bounded by time alone.
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
  volatile int never = 0;
  (void)mbar_wait(bar, parity, &never, kErrTimeoutDrain);
}

// ------------------------------------------------------------------ fused top-k
// Each epilogue warp leaves, per tile, the selection keys of its 32 keys that may
// be candidates -- packed in index order -- and their count in a staging ring; one
// streaming selector warp walks the tiles in order and appends them to a
// shared-memory buffer for the row it is working on, keeping index order.  The
// buffer has a rising threshold tau: it holds every key of the CTA's share of the
// row seen so far whose selection key is >= tau (and possibly some below).  When
// it fills up, the streaming warp and three helper warps find by a radix descent a
// new tau with at least k and at most `target` buffered keys >= tau, and compact
// the buffer to those, keeping their order.  A key below tau has at least k larger
// keys in the same share of the row, so it cannot be among the row's top k.  The
// streaming warp publishes tau's score key, tagged with the row, and the epilogue
// stages no key whose score key is below it (a stale value only lets more keys
// through).  At the end of the row (or of the CTA's work) the buffer goes to the
// row's slot in global memory.  Selection runs beside the tensor-core pipeline;
// the staging ring absorbs short delays, but a compaction outlasts it and holds
// the epilogue (and so the tensor pipe) until it ends.
//
// The four selector warps meet on an mbarrier (one arrival per warp) that each
// waits on by polling, bounded in time and by the CTA's abort flag; a warp whose
// wait gave up returns false and the selectors leave.
struct CandSet {
  uint64_t* buf;   // [FUSED_CB]
  uint32_t* hist;  // [256]
  int* x;          // [FUSED_XINTS]: 0..7 warp sums and 8..15 the chosen bin (by
                   // round parity), 16..79 per-round counts of a compaction (by
                   // round parity, 8 x 4 each), 96.. the streamer's request (op,
                   // count, target, -, tau and the buffer's largest key as uint64)
  uint32_t bar;    // group barrier (mbarrier, 4 arrivals: lane 0 of each selector warp)
  uint32_t phase;  // its phase parity, the same in every selector thread
  volatile int* abort;
  // Bounded: false if the CTA aborted (the group's results are void then).
  __device__ __forceinline__ bool sync() {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = __all_sync(0xffffffffu, mbar_wait_poll(bar, phase, abort, kErrTimeoutEpilogue));
    phase ^= 1u;
    return ok;
  }
};

// The new threshold and the compaction.  Every selector thread calls it with the
// same cnt, tau and hi (kept in registers, identical in every thread) and t = its
// index (0..127).  hi is the largest buffered key; the buffer holds at least k
// keys >= tau when tau != 0, so the k-th largest lies in [tau, hi] and the radix
// rounds start below the bits those two share, with 8-bit digits.  The survivors
// move down in place, 1024 entries per round in their original order (a round's
// reads precede its writes, which land below the next round's reads).
struct CompactResult {
  uint64_t tau;
  int cnt;
  uint32_t phase;  // the group barrier's parity afterwards
  bool ok;
};
__device__ __noinline__ CompactResult cand_compact(CandSet cs, const int cnt, uint64_t tau,
                                                   uint64_t hi, int k, int target, int t) {
  const int lane = t & 31, wid = t >> 5;
  CompactResult fail{tau, cnt, 0u, false};
  if (!cs.sync()) return fail;  // the streamer's keys are in the buffer
  int pbits = (tau >= hi) ? 63 : __clzll(static_cast<long long>(tau ^ hi));
  uint64_t prefix = pbits == 0 ? 0ull : (tau >> (64 - pbits));
  int need = k, above = 0;
  uint64_t tnew;
  for (int round = 0;; ++round) {
    const int bits = (64 - pbits) < 8 ? 64 - pbits : 8;
    const int shift = 64 - pbits - bits;
    const uint64_t dmask = (1ull << bits) - 1ull;
    cs.hist[t] = 0u;
    cs.hist[t + 128] = 0u;
    if (!cs.sync()) return fail;
    for (int base = 0; base < cnt; base += 1024) {
      uint64_t c[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = base + 128 * j + t;
        c[j] = i < cnt ? cs.buf[i] : 0ull;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = base + 128 * j + t;
        if (i < cnt && (pbits == 0 || (c[j] >> (64 - pbits)) == prefix))
          atomicAdd(&cs.hist[static_cast<int>((c[j] >> shift) & dmask)], 1u);
      }
    }
    if (!cs.sync()) return fail;
    // thread t owns bins 2t and 2t + 1; count the keys in higher bins
    const int h1 = static_cast<int>(cs.hist[2 * t + 1]), h0 = static_cast<int>(cs.hist[2 * t]);
    const int v = h0 + h1;
    int incl = v;  // sum over lanes >= this lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    if (lane == 0) cs.x[4 * (round & 1) + wid] = incl;
    if (!cs.sync()) return fail;
    int higher = 0;
    for (int w = wid + 1; w < 4; ++w) higher += cs.x[4 * (round & 1) + w];
    const int gt1 = higher + incl - v, gt0 = gt1 + h1;
    int* xb = cs.x + 8 + 4 * (round & 1);  // the chosen bin, by round parity
    if (gt1 < need && need <= gt1 + h1) {
      xb[0] = 2 * t + 1;
      xb[1] = gt1;
      xb[2] = h1;
    }
    if (gt0 < need && need <= gt0 + h0) {
      xb[0] = 2 * t;
      xb[1] = gt0;
      xb[2] = h0;
    }
    if (!cs.sync()) return fail;
    const uint64_t pre = (prefix << bits) | static_cast<uint64_t>(xb[0] & 255);
    const int gt = xb[1], inb = xb[2];
    pbits += bits;
    if (above + gt + inb <= target || pbits == 64) {  // keys >= the bin's lower edge
      tnew = pbits == 64 ? pre : pre << (64 - pbits);
      break;
    }
    above += gt;
    need -= gt;
    prefix = pre;
  }
  // entry base + 128 j + t is thread t's j-th of the round; a survivor's place
  // counts the survivors of the earlier (j, warp) groups, in that order
  int wpos = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int base = 0, par = 0; base < cnt; base += 1024, par ^= 1) {
    uint64_t c[8];
    unsigned m[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = base + 128 * j + t;
      c[j] = i < cnt ? cs.buf[i] : 0ull;
      m[j] = __ballot_sync(0xffffffffu, i < cnt && c[j] >= tnew);
    }
    int* rc = cs.x + 16 + 32 * par;
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < 8; ++j) rc[4 * j + wid] = __popc(m[j]);
    }
    if (!cs.sync()) return fail;
    int acc = 0;
    int off[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int4 n = *reinterpret_cast<const int4*>(rc + 4 * j);
      const int nw[4] = {n.x, n.y, n.z, n.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        if (w == wid) off[j] = acc;
        acc += nw[w];
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if ((m[j] >> lane) & 1u) {
        const int d = wpos + off[j] + __popc(m[j] & lt);
        if (d < FUSED_CB) cs.buf[d] = c[j];
      }
    }
    wpos += acc;
  }
  CompactResult r{tnew > tau ? tnew : tau, wpos < FUSED_CB ? wpos : FUSED_CB, 0u, false};
  r.ok = cs.sync();
  r.phase = cs.phase;
  return r;
}

template <bool FP8, int TPM, bool FUSED, bool SEGS>
__global__ void __launch_bounds__(IdxCfg<FP8, TPM, FUSED>::THREADS, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ IdxTcArgs a) {
  using C = IdxCfg<FP8, TPM, FUSED>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto accfull_bar = [&](int i) { return bar0 + 8u * (2 * C::STAGES + i); };
  auto accempty_bar = [&](int i) { return bar0 + 8u * (2 * C::STAGES + C::NACC + i); };
  const uint32_t qfull_bar = bar0 + 8u * (2 * C::STAGES + 2 * C::NACC);
  const uint32_t qempty_bar = qfull_bar + 8;
  const uint32_t mmadone_bar = qfull_bar + 16;
  // fused top-k: staging slot s holds a tile's scores (full: 4 epilogue warps
  // arrive; empty: the selector warps arrive)
  auto stgfull_bar = [&](int s) { return mmadone_bar + 8u * (1 + s); };
  auto stgempty_bar = [&](int s) { return mmadone_bar + 8u * (1 + C::NSTG + s); };
  // the streaming selector's requests to its helpers, and the selector group barrier
  const uint32_t selreq_bar = mmadone_bar + 8u * (1 + 2 * C::NSTG);
  const uint32_t selgrp_bar = selreq_bar + 8;

  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* start = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
  // fused: the streaming selector's threshold, (row + 1) << 32 | tau's score key
  volatile uint64_t* tau_pub = reinterpret_cast<volatile uint64_t*>(smem + C::OFF_MISC + 16);
  float* w_smem = reinterpret_cast<float*>(smem + C::OFF_W);
  const uint32_t a_base = smem_u32(smem + C::OFF_A);
  const uint32_t q_base = smem_u32(smem + C::OFF_Q);

  const long g0 = a.total_tiles * blockIdx.x / gridDim.x;
  const long g1 = a.total_tiles * (blockIdx.x + 1) / gridDim.x;
  const long nitems = g1 - g0;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < C::STAGES; ++s) {
        mbar_init(full_bar(s), 1);
        mbar_init(empty_bar(s), 1);
      }
      for (int i = 0; i < C::NACC; ++i) {
        mbar_init(accfull_bar(i), 1);
        mbar_init(accempty_bar(i), C::SETW);
      }
      mbar_init(qfull_bar, 1);
      mbar_init(qempty_bar, C::MMAW);
      mbar_init(mmadone_bar, C::MMAW);
      if constexpr (FUSED) {
        for (int j = 0; j < C::NSTG; ++j) {
          mbar_init(stgfull_bar(j), C::SETW);
          mbar_init(stgempty_bar(j), 1);
        }
        mbar_init(selreq_bar, 1);
        mbar_init(selgrp_bar, C::NSEL);
        for (int j = 0; j < FUSED_XINTS; ++j) reinterpret_cast<int*>(smem + C::OFF_CX)[j] = 0;
        *tau_pub = 0ull;
      }
      *abort_flag = 0;
      fence_barrier_init();
      fence_proxy_async_smem();
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmQ);
    }
    // Locate tile g0 in the (query block, key tile) list: warp-parallel prefix scan.
    long cum = 0;
    for (int base = 0; base < a.nqb; base += 32) {
      const int qb = base + lane;
      const long t = (qb < a.nqb) ? qb_tiles<TPM, SEGS>(a, qb) : 0;
      long incl = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const long tot = __shfl_sync(0xffffffffu, incl, 31);
      if (cum + tot > g0) {
        const unsigned m = __ballot_sync(0xffffffffu, cum + incl > g0);
        const int l = __ffs(m) - 1;
        const long incl_l = __shfl_sync(0xffffffffu, incl, l);
        const long t_l = __shfl_sync(0xffffffffu, t, l);
        if (lane == 0) {
          start[0] = base + l;
          start[1] = static_cast<int>(g0 - (cum + incl_l - t_l));
        }
        break;
      }
      cum += tot;
    }
  } else if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();  // set-up above touches no global memory

  if (nitems > 0) {
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        WorkIt<TPM, SEGS> it{start[0], start[1], qb_tiles<TPM, SEGS>(a, start[0])};
        int stage = 0;
        uint32_t ph = 0;
        int qloads = 0, cur_qb = -1;
        long issued = 0;
        for (long i = 0; i < nitems; ++i) {
          if (it.qb != cur_qb) {
            if (qloads > 0 &&
                !mbar_wait(qempty_bar, (qloads - 1) & 1, abort_flag, kErrTimeoutProducer))
              break;
            const QbInfo x = qb_info<TPM, SEGS>(a, it.qb);
            const int qrow = static_cast<int>((x.qrow0 + x.ql * TPM) * 64);
            (void)in_bounds(qrow >= 0 && x.ql * TPM < x.R, kErrBoundsTma);  // loads stay legal
            mbar_arrive_expect_tx(qfull_bar, C::Q_BYTES);
#pragma unroll
            for (int kb = 0; kb < C::KBLK; ++kb)
              tma_load_2d(q_base + kb * (C::N * 128), &tmQ, kb * C::ELEMS_128B, qrow, qfull_bar);
            ++qloads;
            cur_qb = it.qb;
          }
          if (!mbar_wait(empty_bar(stage), ph ^ 1, abort_flag, kErrTimeoutProducer)) break;
          const QbInfo kx = qb_info<TPM, SEGS>(a, it.qb);
          const int krow = static_cast<int>(kx.krow0 + it.kt * C::BM);
          (void)in_bounds(krow >= 0 && it.kt * C::BM < kx.Lk, kErrBoundsTma);
          mbar_arrive_expect_tx(full_bar(stage), C::A_BYTES);
#pragma unroll
          for (int kb = 0; kb < C::KBLK; ++kb)
            tma_load_2d(a_base + stage * C::A_BYTES + kb * (C::BM * 128), &tmK,
                        kb * C::ELEMS_128B, krow, full_bar(stage));
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            ph ^= 1;
          }
          it.advance(a);
        }
        if (*abort_flag) {
          // let every copy this thread started land before the CTA's smem goes away
          long n = issued < C::STAGES ? issued : C::STAGES;
          for (long j = issued - n; j < issued; ++j)
            mbar_wait_drain(full_bar(static_cast<int>(j % C::STAGES)),
                            static_cast<uint32_t>((j / C::STAGES) & 1));
          if (qloads > 0) mbar_wait_drain(qfull_bar, (qloads - 1) & 1);
        }
      }
    } else if (warp < C::EPI_W0) {
      // ------------------------------------------------------------ MMA issuer(s)
      if (lane == 0) {
        const int mw = warp - 1;
        constexpr uint32_t fmt = FP8 ? 0u : 1u;  // e4m3 : bf16
        constexpr uint32_t idesc = idesc_f32acc(fmt, fmt, C::BM, C::N);
        // Descriptors, built once: one per K step of the resident query block,
        // and the key ring's base (a K step or stage offset adds its address >> 4
        // to the start-address field, which cannot carry out: every shared
        // address is below 256 KB).
        uint64_t bdesc[C::KSTEPS];
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk)
          bdesc[kk] = sdesc_k_sw128(q_base + (kk / 4) * (C::N * 128) + (kk % 4) * 32);
        const uint64_t adesc0 = sdesc_k_sw128(a_base);
        WorkIt<TPM, SEGS> it{start[0], start[1], qb_tiles<TPM, SEGS>(a, start[0])};
        int stage = 0, acc = 0;
        uint32_t ph = 0, aph = 0;
        int qwaits = 0, cur_qb = -1;
        for (long i = 0; i < nitems; ++i) {
          if (it.qb != cur_qb) {
            if (!mbar_wait(qfull_bar, qwaits & 1, abort_flag, kErrTimeoutMma)) break;
            ++qwaits;
            cur_qb = it.qb;
          }
          if (C::MMAW == 1 || i % C::MMAW == mw) {
            if (!mbar_wait(accempty_bar(acc), aph ^ 1, abort_flag, kErrTimeoutMma)) break;
            if (!mbar_wait(full_bar(stage), ph, abort_flag, kErrTimeoutMma)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::N);
            const uint64_t a_st = adesc0 + static_cast<uint64_t>(stage * (C::A_BYTES >> 4));
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS; ++kk) {
              const uint64_t adesc = a_st + (((kk / 4) * (C::BM * 128) + (kk % 4) * 32) >> 4);
              if constexpr (FP8)
                tc_mma_f8(d_tmem, adesc, bdesc[kk], idesc, kk > 0 ? 1u : 0u);
              else
                tc_mma_f16(d_tmem, adesc, bdesc[kk], idesc, kk > 0 ? 1u : 0u);
            }
            tc_commit(empty_bar(stage));
            tc_commit(accfull_bar(acc));
          }
          WorkIt<TPM, SEGS> nx = it;
          nx.advance(a);
          if (i + 1 == nitems || nx.qb != it.qb) tc_commit(qempty_bar);
          it = nx;
          if (++stage == C::STAGES) {
            stage = 0;
            ph ^= 1;
          }
          if (++acc == C::NACC) {
            acc = 0;
            aph ^= 1;
          }
        }
        // every MMA this thread issued has completed before TMEM is released
        tc_commit(mmadone_bar);
        mbar_wait_drain(mmadone_bar, 0);
      }
    } else if (warp < C::SEL_W0) {
      // ------------------------------------------------------------ epilogue
      const int e = warp - C::EPI_W0;
      const int qd = warp & 3;     // TMEM lane quadrant this warp may access
      const int set = e / C::SETW;  // accumulator slots a with a % NSETS == set
      const int member = (e % C::SETW) / 4;  // which tokens of the block this warp reduces
      float* wsl = w_smem + e * C::TOK_PER_EW * 64;
      WorkIt<TPM, SEGS> it{start[0], start[1], qb_tiles<TPM, SEGS>(a, start[0])};
      int acc = 0;
      uint32_t aph = 0;
      int cur_qb = -1;
      // head weights of this warp's tokens: the warp's shared copy (wsl), written
      // when a query block starts; a warp with several tokens keeps them in registers
      // (wr), a one-token warp reads them with one broadcast load per 4 heads
      constexpr bool WREG = C::TOK_PER_EW > 1;
      float wr[WREG ? C::TOK_PER_EW : 1][64];
#pragma unroll
      for (int t = 0; t < (WREG ? C::TOK_PER_EW : 1); ++t)
#pragma unroll
        for (int h = 0; h < 64; ++h) wr[t][h] = 0.f;
      uint64_t* stg = reinterpret_cast<uint64_t*>(smem + C::OFF_STG);  // fused: staged keys
      int* scnt = reinterpret_cast<int*>(smem + C::OFF_SCNT);             // and counts
      for (long i = 0; i < nitems; ++i) {
        if (C::NSETS > 1 && acc % C::NSETS != set) {  // another set's slot
          if (++acc == C::NACC) {
            acc = 0;
            aph ^= 1;
          }
          it.advance(a);
          continue;
        }
        const QbInfo qi = qb_info<TPM, SEGS>(a, it.qb);
        const int r0 = qi.ql * TPM + member * C::TOK_PER_EW;
        if (it.qb != cur_qb) {
          __syncwarp();
          for (int x = lane; x < C::TOK_PER_EW * 64; x += 32) {
            const int r = r0 + x / 64;
            float v = 0.f;
            if (r < qi.R) {
              const long o = (qi.qrow0 + r) * 64 + (x % 64);
              v = a.w[o];
              if constexpr (FP8) v *= a.q_scale[o];
            }
            wsl[x] = v;
          }
          __syncwarp();
          if constexpr (WREG) {
#pragma unroll
            for (int t = 0; t < C::TOK_PER_EW; ++t)
#pragma unroll
              for (int h = 0; h < 64; ++h) wr[t][h] = wsl[t * 64 + h];
          }
          cur_qb = it.qb;
        }
        // this lane's key; its fp8 scale is fetched before the wait so the load's
        // latency hides behind it
        const int s = it.kt * C::BM + qd * 32 + lane;
        const bool key_ok = s < qi.Lk;
        float ks = 1.f;
        if constexpr (FP8) ks = key_ok ? a.k_scale[qi.krow0 + s] : 0.f;
        // every lane leaves together, so the warp never splits before tcgen05.ld
        const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(accfull_bar(acc), aph, abort_flag,
                                                              kErrTimeoutEpilogue));
        if (!acc_ok) break;
        float res[C::TOK_PER_EW];
        tc_fence_after();
        // sum_h w_h relu(x_h) of each token, heads h = j mod 4 into s_j in head order
        auto head_sum = [&](const float* v, int tk) {
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
          for (int h = 0; h < 64; h += 4) {
            const float4 wv = *reinterpret_cast<const float4*>(wsl + tk * 64 + h);
            s0 = fmaf(wv.x, fmaxf(v[h + 0], 0.f), s0);
            s1 = fmaf(wv.y, fmaxf(v[h + 1], 0.f), s1);
            s2 = fmaf(wv.z, fmaxf(v[h + 2], 0.f), s2);
            s3 = fmaf(wv.w, fmaxf(v[h + 3], 0.f), s3);
          }
          return (s0 + s1) + (s2 + s3);
        };
        auto tok_addr = [&](int tk) {
          return tmem_base + (static_cast<uint32_t>(qd * 32) << 16) +
                 static_cast<uint32_t>(acc * C::N + (member * C::TOK_PER_EW + tk) * 64);
        };
        if constexpr (WREG) {
          // 16 columns per TMEM round trip, weights in registers
#pragma unroll
          for (int tk = 0; tk < C::TOK_PER_EW; ++tk) {
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
            for (int part = 0; part < 4; ++part) {
              float v[16];
              tmem_ld16(tok_addr(tk) + 16 * part, v);
              tmem_ld_wait();
#pragma unroll
              for (int h4 = 0; h4 < 4; ++h4) {  // chains (s0, s1) and (s2, s3) in pairs
                const int h = 16 * part + 4 * h4;
                const float2 p01 = ffma2(make_float2(wr[tk][h], wr[tk][h + 1]),
                                         make_float2(fmaxf(v[4 * h4 + 0], 0.f), fmaxf(v[4 * h4 + 1], 0.f)),
                                         make_float2(s0, s1));
                const float2 p23 = ffma2(make_float2(wr[tk][h + 2], wr[tk][h + 3]),
                                         make_float2(fmaxf(v[4 * h4 + 2], 0.f), fmaxf(v[4 * h4 + 3], 0.f)),
                                         make_float2(s2, s3));
                s0 = p01.x;
                s1 = p01.y;
                s2 = p23.x;
                s3 = p23.y;
              }
            }
            res[tk] = (s0 + s1) + (s2 + s3);
          }
        } else if constexpr (!FUSED && TPM == 1) {
          // one token: its 64 columns are loaded before one wait, a single TMEM
          // round trip per tile
          float v[64];
#pragma unroll
          for (int part = 0; part < 4; ++part)
            tmem_ld16(tok_addr(0) + 16 * part, *reinterpret_cast<float(*)[16]>(&v[16 * part]));
          tmem_ld_wait();
          res[0] = head_sum(v, 0);
        } else if constexpr (!FUSED) {
          // one token of a multi-token block (fewer registers per warp): 32 columns
          // per round trip
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float v[32];
            tmem_ld16(tok_addr(0) + 32 * half, *reinterpret_cast<float(*)[16]>(&v[0]));
            tmem_ld16(tok_addr(0) + 32 * half + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
            tmem_ld_wait();
#pragma unroll
            for (int h = 0; h < 32; h += 4) {  // chains (s0, s1) and (s2, s3) in pairs
              const float4 wv = *reinterpret_cast<const float4*>(wsl + 32 * half + h);
              const float2 p01 =
                  ffma2(make_float2(wv.x, wv.y),
                        make_float2(fmaxf(v[h + 0], 0.f), fmaxf(v[h + 1], 0.f)), make_float2(s0, s1));
              const float2 p23 =
                  ffma2(make_float2(wv.z, wv.w),
                        make_float2(fmaxf(v[h + 2], 0.f), fmaxf(v[h + 3], 0.f)), make_float2(s2, s3));
              s0 = p01.x;
              s1 = p01.y;
              s2 = p23.x;
              s3 = p23.y;
            }
          }
          res[0] = (s0 + s1) + (s2 + s3);
        } else {
          // 16 columns at a time, leaving the registers to the selection
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
          for (int part = 0; part < 4; ++part) {
            float v[16];
            tmem_ld16(tok_addr(0) + 16 * part, v);
            tmem_ld_wait();
#pragma unroll
            for (int h4 = 0; h4 < 4; ++h4) {
              const int h = 16 * part + 4 * h4;
              const float4 wv = *reinterpret_cast<const float4*>(wsl + h);
              s0 = fmaf(wv.x, fmaxf(v[4 * h4 + 0], 0.f), s0);
              s1 = fmaf(wv.y, fmaxf(v[4 * h4 + 1], 0.f), s1);
              s2 = fmaf(wv.z, fmaxf(v[4 * h4 + 2], 0.f), s2);
              s3 = fmaf(wv.w, fmaxf(v[4 * h4 + 3], 0.f), s3);
            }
          }
          res[0] = (s0 + s1) + (s2 + s3);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(accempty_bar(acc));
        if constexpr (FUSED) {
          // the selection keys of the keys in range whose score (the same fp32
          // value the unfused store writes) reaches the row's published threshold go,
          // packed in index order, to staging slot i % NSTG, which only this set uses
          const uint64_t ck = select_key(res[0] * ks, static_cast<uint32_t>(s));
          const uint64_t pub = *tau_pub;
          const uint32_t tf =
              (static_cast<uint32_t>(pub >> 32) == static_cast<uint32_t>(it.qb) + 1u)
                  ? static_cast<uint32_t>(pub)
                  : 0u;
          const bool cand = key_ok && s <= qi.pos0 && static_cast<uint32_t>(ck >> 32) >= tf;
          const unsigned cm = __ballot_sync(0xffffffffu, cand);
          const int sl = static_cast<int>(i % C::NSTG);
          const uint32_t use = static_cast<uint32_t>(i / C::NSTG);
          if (!__all_sync(0xffffffffu, mbar_wait(stgempty_bar(sl), (use & 1u) ^ 1u, abort_flag,
                                                 kErrTimeoutEpilogue)))
            break;
          if (cand) stg[sl * C::BM + qd * 32 + __popc(cm & ((1u << lane) - 1u))] = ck;
          if (lane == 0) scnt[sl * 4 + qd] = __popc(cm);
          __syncwarp();
          if (lane == 0) mbar_arrive(stgfull_bar(sl));
        } else if (key_ok) {
#pragma unroll
          for (int tk = 0; tk < C::TOK_PER_EW; ++tk) {
            const int r = r0 + tk;
            if (r < qi.R) {
              const long pos = qi.pos0 + r;
              a.scores[(qi.orow0 + r) * a.ld + s] =
                  (s <= pos) ? res[tk] * ks : -INFINITY;
            }
          }
        }
        if (++acc == C::NACC) {
          acc = 0;
          aph ^= 1;
        }
        it.advance(a);
      }
    } else {
      // ------------------------------------------------------------ selectors (fused)
      // The first selector warp streams: it takes every tile's candidate keys from
      // the staging ring and appends them to the buffer in index order.  The other three wait until it asks them to compact
      // the buffer with it (or to leave).
      if constexpr (FUSED) {
        const int wid = warp - C::SEL_W0, t = wid * 32 + lane;
        CandSet cs{reinterpret_cast<uint64_t*>(smem + C::OFF_CBUF),
                   reinterpret_cast<uint32_t*>(smem + C::OFF_CHIST),
                   reinterpret_cast<int*>(smem + C::OFF_CX), selgrp_bar, 0u, abort_flag};
        int* req = cs.x + 96;  // op (1 compact, 2 leave), count, target; tau, hi at req + 4, + 6
        if (wid == 0) {
          const uint64_t* stg = reinterpret_cast<const uint64_t*>(smem + C::OFF_STG);
          const int* scnt = reinterpret_cast<const int*>(smem + C::OFF_SCNT);
          uint64_t* const cbuf = reinterpret_cast<uint64_t*>(smem + C::OFF_CBUF);
          WorkIt<TPM, SEGS> it{start[0], start[1], qb_tiles<TPM, SEGS>(a, start[0])};
          int ccnt = 0, crow = -1;
          uint64_t ctau = 0, kmx = 0;  // kmx: this lane's largest appended key
          long crow_first = 0;         // first CTA of the current row
          int sl = 0;                  // staging slot of tile i, and its use parity
          uint32_t sph = 0;
          // (the loop state stays in registers: no helper takes its address)
          for (long i = 0;; ++i) {
            // before tile i: the buffer goes to the row's slot when the row (or the
            // work) ends, first compacted to at most k + 256 keys if it holds more
            // than 2k; otherwise it is compacted to 3/8 of its size when the next
            // tile might not fit
            const bool row_end = crow >= 0 && (i == nitems || it.qb != crow);
            int target = 0;
            if (row_end && ccnt > 2 * a.topk) target = a.topk + 256;
            if (!row_end && ccnt > FUSED_CB - C::BM) target = 3 * FUSED_CB / 8;
            if (target > 0) {  // with the helpers
              uint64_t hi = kmx;
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) {
                const uint64_t y = __shfl_xor_sync(0xffffffffu, hi, o);
                hi = y > hi ? y : hi;
              }
              if (lane == 0) {
                req[0] = 1;
                req[1] = ccnt;
                req[2] = target;
                *reinterpret_cast<uint64_t*>(req + 4) = ctau;
                *reinterpret_cast<uint64_t*>(req + 6) = hi;
              }
              __syncwarp();
              if (lane == 0) mbar_arrive(selreq_bar);
              const CompactResult r = cand_compact(cs, ccnt, ctau, hi, a.topk, target, t);
              if (!r.ok) break;
              ccnt = r.cnt;
              ctau = r.tau;
              cs.phase = r.phase;
              if (lane == 0)
                *tau_pub = (static_cast<uint64_t>(static_cast<uint32_t>(crow) + 1u) << 32) |
                           (ctau >> 32);
            }
            if (row_end) {  // header: count, tau, largest key
              const long piece = static_cast<long>(blockIdx.x) - crow_first;
              uint8_t* slot = a.cslots + (static_cast<long>(crow) * a.maxp + piece) *
                                             static_cast<long>(FUSED_SLOT_BYTES);
              uint64_t* dst = reinterpret_cast<uint64_t*>(slot + 64);
              for (int j = lane; j < ccnt; j += 32) dst[j] = cbuf[j];
              uint64_t mx = kmx;
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) {
                const uint64_t y = __shfl_xor_sync(0xffffffffu, mx, o);
                mx = y > mx ? y : mx;
              }
              if (lane == 0) {
                *reinterpret_cast<int*>(slot) = ccnt;
                *reinterpret_cast<uint64_t*>(slot + 8) = ctau;
                *reinterpret_cast<uint64_t*>(slot + 16) = mx;
              }
              __syncwarp();
              ccnt = 0;
              ctau = 0;
              kmx = 0;
            }
            if (i == nitems) break;
            if (it.qb != crow) {
              crow = it.qb;
              crow_first = ((g0 + i - it.kt) * gridDim.x + gridDim.x - 1) / a.total_tiles;
            }
            if (!__all_sync(0xffffffffu, mbar_wait_poll(stgfull_bar(sl), sph, abort_flag,
                                                        kErrTimeoutEpilogue)))
              break;
            const int4 n4 = *reinterpret_cast<const int4*>(scnt + sl * 4);
            const int nq[4] = {n4.x, n4.y, n4.z, n4.w};
            uint64_t kv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) kv[q] = lane < nq[q] ? stg[sl * C::BM + q * 32 + lane] : 0ull;
            __syncwarp();
            if (lane == 0) mbar_arrive(stgempty_bar(sl));
            if (++sl == C::NSTG) {
              sl = 0;
              sph ^= 1u;
            }
            // warp q's keys follow warp q - 1's: the tile's candidates in index order
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (lane < nq[q]) {
                cbuf[ccnt + lane] = kv[q];
                kmx = kv[q] > kmx ? kv[q] : kmx;
              }
              ccnt += nq[q];
            }
            it.advance(a);
          }
          // the helpers leave
          __syncwarp();
          if (lane == 0) {
            req[0] = 2;
            mbar_arrive(selreq_bar);
          }
        } else {
          uint32_t rph = 0;
          for (;;) {
            // wait for a request: bounded by a long limit (the streamer always ends
            // with one), or the CTA's abort
            bool got = mbar_test(selreq_bar, rph);
            const uint64_t t0 = globaltimer();
            while (!got) {
              __nanosleep(64);
              if (*abort_flag) break;
              if (globaltimer() - t0 > 30ull * IC_WAIT_NS) {
                *abort_flag = 1;
                record_error(kErrTimeoutEpilogue);
                break;
              }
              got = mbar_test(selreq_bar, rph);
            }
            if (!__all_sync(0xffffffffu, got)) break;
            rph ^= 1u;
            if (req[0] != 1) break;
            const CompactResult r =
                cand_compact(cs, req[1], *reinterpret_cast<const uint64_t*>(req + 4),
                             *reinterpret_cast<const uint64_t*>(req + 6), a.topk, req[2], t);
            if (!r.ok) break;
            cs.phase = r.phase;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Writes -inf on the masked keys [pos0 + r + 1, Lk) of every row (the tensor-core
// kernel only visits key tiles up to its query block's diagonal).  One CTA per row.
__global__ void fill_masked_kernel(float* scores, long ld, int R, int Lk, long pos0) {
  grid_dep_wait();
  const long row = blockIdx.x;  // b * R + r
  const long r = row % R;
  for (long s = pos0 + r + 1 + threadIdx.x; s < Lk; s += blockDim.x) scores[row * ld + s] = -INFINITY;
}

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

static ic_status make_map(CUtensorMap* m, const void* base, bool fp8, uint64_t rows,
                          uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return fail(IC_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const uint32_t eb = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128ull * eb};
  cuuint32_t box[2] = {128u / eb, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(IC_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return IC_OK;
}

long long causal_pairs(long R, long Lk, long pos0) {
  long long n = 0;
  const long r_full = Lk - pos0 - 1;  // rows from here on see all Lk keys
  const long r_tri = r_full < 0 ? 0 : (r_full < R ? r_full : R);
  n += static_cast<long long>(r_tri) * (pos0 + 1) +
       static_cast<long long>(r_tri) * (r_tri - 1) / 2;  // sum_{r < r_tri} (pos0 + r + 1)
  n += static_cast<long long>(R - r_tri) * Lk;
  return n;
}

template <bool FP8, int TPM, bool FUSED = false>
static ic_status launch_tpl(const void* q, const float* q_scale, const void* k,
                            const float* k_scale, const float* w, int batch, int rows, int Lk,
                            long pos0, float* scores, long ld, cudaStream_t stream,
                            uint8_t* cslots = nullptr, int maxp = 0, int topk = 0) {
  using C = IdxCfg<FP8, TPM, FUSED>;
  IdxTcArgs a;
  a.w = w;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.scores = scores;
  a.ld = ld;
  a.B = batch;
  a.R = rows;
  a.Lk = Lk;
  a.pos0 = pos0;
  a.qb_per_batch = (rows + TPM - 1) / TPM;
  a.nqb = batch * a.qb_per_batch;
  a.cslots = cslots;
  a.maxp = maxp;
  a.topk = topk;
  a.nseg = 0;
  long total = 0;
  for (int qb = 0; qb < a.qb_per_batch; ++qb) total += qb_tiles<TPM, false>(a, qb);
  total *= batch;  // every batch has the same triangle
  a.total_tiles = total;
  if (total == 0) return IC_OK;

  CUtensorMap tmK, tmQ;
  ic_status st = make_map(&tmK, k, FP8, static_cast<uint64_t>(batch) * Lk, C::BM);
  if (st) return st;
  st = make_map(&tmQ, q, FP8, static_cast<uint64_t>(batch) * rows * 64, C::N);
  if (st) return st;

  st = cuda_check(cudaFuncSetAttribute(indexer_tc_kernel<FP8, TPM, FUSED, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES),
                  "cudaFuncSetAttribute(indexer)");
  if (st) return st;
  const long grid = total < num_sms() ? total : num_sms();
  st = cuda_check(launch_dep(indexer_tc_kernel<FP8, TPM, FUSED, false>, dim3(static_cast<unsigned>(grid)),
                             dim3(C::THREADS), C::SMEM_BYTES, stream, 1, tmK, tmQ, a),
                  "indexer_tc_kernel launch");
  if (st) return st;
  const int kind = FUSED ? (FP8 ? kKindIndexerTopkE4m3 : kKindIndexerTopkBf16)
                         : (FP8 ? kKindIndexerE4m3 : kKindIndexerBf16);
  trace_launch(kind, stream,
               2.0 * 64 * 128 * static_cast<double>(causal_pairs(rows, Lk, pos0)) * batch);
  return IC_OK;
}

// The multi-token instance over packed segments (see IdxTcArgs): one launch for
// every segment; q_rows and k_rows are the rows of the packed query and key tensors.
template <bool FP8>
static ic_status launch_segs(const void* q, const float* q_scale, const void* k,
                             const float* k_scale, const float* w, const IdxSeg* segs, int nseg,
                             long q_rows, long k_rows, float* scores, long ld,
                             cudaStream_t stream) {
  constexpr int TPM = 4;
  using C = IdxCfg<FP8, TPM, false>;
  IdxTcArgs a;
  a.w = w;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.scores = scores;
  a.ld = ld;
  a.B = 1;
  a.R = 0;
  a.Lk = 0;
  a.pos0 = 0;
  a.qb_per_batch = 1;
  a.cslots = nullptr;
  a.maxp = 0;
  a.topk = 0;
  a.nseg = nseg;
  int nqb = 0;
  double flop = 0.0;
  for (int j = 0; j < nseg; ++j) {
    a.seg[j] = segs[j];
    a.seg[j].qb0 = nqb;
    nqb += (segs[j].R + TPM - 1) / TPM;
    flop += 2.0 * 64 * 128 * static_cast<double>(causal_pairs(segs[j].R, segs[j].Lk, segs[j].pos0));
  }
  a.nqb = nqb;
  long total = 0;
  for (int qb = 0; qb < nqb; ++qb) total += qb_tiles<TPM, true>(a, qb);
  a.total_tiles = total;
  if (total == 0) return IC_OK;

  CUtensorMap tmK, tmQ;
  ic_status st = make_map(&tmK, k, FP8, static_cast<uint64_t>(k_rows), C::BM);
  if (st) return st;
  st = make_map(&tmQ, q, FP8, static_cast<uint64_t>(q_rows) * 64, C::N);
  if (st) return st;
  st = cuda_check(cudaFuncSetAttribute(indexer_tc_kernel<FP8, TPM, false, true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES),
                  "cudaFuncSetAttribute(indexer)");
  if (st) return st;
  const long grid = total < num_sms() ? total : num_sms();
  st = cuda_check(launch_dep(indexer_tc_kernel<FP8, TPM, false, true>, dim3(static_cast<unsigned>(grid)),
                             dim3(C::THREADS), C::SMEM_BYTES, stream, 1, tmK, tmQ, a),
                  "indexer_tc_kernel launch");
  if (st) return st;
  trace_launch(FP8 ? kKindIndexerE4m3 : kKindIndexerBf16, stream, flop);
  return IC_OK;
}

ic_status launch_indexer_tc_segs(bool fp8, const void* q, const float* q_scale, const void* k,
                                 const float* k_scale, const float* w, const IdxSeg* segs,
                                 int nseg, long q_rows, long k_rows, float* scores, long ld,
                                 cudaStream_t stream) {
  if (nseg < 1 || nseg > IC_MAXSEG) return fail(IC_ERR_INVALID_ARG, "indexer: %d segments", nseg);
  return fp8 ? launch_segs<true>(q, q_scale, k, k_scale, w, segs, nseg, q_rows, k_rows, scores, ld,
                                 stream)
             : launch_segs<false>(q, q_scale, k, k_scale, w, segs, nseg, q_rows, k_rows, scores,
                                  ld, stream);
}

// Plan of the fused indexer -> top-k for `batch` sequences of one query each at
// position pos0 over Lk keys: nt key tiles per row, total = batch * nt tiles cut
// into G equal contiguous CTA shares (as the kernel cuts them), and the most CTA
// pieces any row is split into.
struct FusedPlan {
  long nt, total;
  int G, maxp;
};
static FusedPlan fused_plan(int batch, int Lk, long pos0) {
  FusedPlan p{0, 0, 0, 0};
  const long keys = pos0 + 1 < Lk ? pos0 + 1 : Lk;
  p.nt = (keys + 127) / 128;
  p.total = static_cast<long>(batch) * p.nt;
  if (p.total == 0) return p;
  const long sms = num_sms();
  p.G = static_cast<int>(p.total < sms ? p.total : sms);
  auto cta_of = [&](long t) { return (t * p.G + p.G - 1) / p.total; };
  for (long b = 0; b < batch; ++b) {
    const long np = cta_of(b * p.nt + p.nt - 1) - cta_of(b * p.nt) + 1;
    if (np > p.maxp) p.maxp = static_cast<int>(np);
  }
  return p;
}

size_t indexer_topk_fused_ws_bytes(int batch, int Lk, long pos0) {
  const FusedPlan p = fused_plan(batch, Lk, pos0);
  return static_cast<size_t>(batch) * p.maxp * FUSED_SLOT_BYTES;
}

ic_status launch_indexer_topk_fused(bool fp8, const void* q, const float* q_scale, const void* k,
                                    const float* k_scale, const float* w, int batch, int Lk,
                                    long pos0, int topk, int* idx, void* ws, size_t ws_bytes,
                                    cudaStream_t stream) {
  const FusedPlan p = fused_plan(batch, Lk, pos0);
  const long nv = pos0 + 1 < Lk ? pos0 + 1 : Lk;
  uint8_t* slots = static_cast<uint8_t*>(ws);
  if (nv > topk) {  // otherwise every candidate is selected: the merge alone writes T
    const size_t need = static_cast<size_t>(batch) * p.maxp * FUSED_SLOT_BYTES;
    if (!ws || ws_bytes < need || reinterpret_cast<uintptr_t>(ws) % 16 != 0)
      return fail(IC_ERR_WORKSPACE,
                  "indexer_topk: needs a 16-byte aligned workspace of %zu bytes (got %zu)", need,
                  ws_bytes);
    ic_status st = fp8 ? launch_tpl<true, 1, true>(q, q_scale, k, k_scale, w, batch, 1, Lk, pos0,
                                                   nullptr, Lk, stream, slots, p.maxp, topk)
                       : launch_tpl<false, 1, true>(q, q_scale, k, k_scale, w, batch, 1, Lk,
                                                    pos0, nullptr, Lk, stream, slots, p.maxp, topk);
    if (st) return st;
  }
  return launch_topk_merge(slots, batch, p.nt, p.total, p.G, p.maxp, FUSED_SLOT_BYTES,
                           FUSED_CB, static_cast<int>(nv), topk, idx, stream);
}

ic_status launch_indexer_tc(bool fp8, const void* q, const float* q_scale, const void* k,
                            const float* k_scale, const float* w, int batch, int rows, int Lk,
                            long pos0, float* scores, long ld, bool fill_tail,
                            cudaStream_t stream) {
  ic_status st;
  const bool small = rows < 4;
  if (fp8)
    st = small ? launch_tpl<true, 1>(q, q_scale, k, k_scale, w, batch, rows, Lk, pos0, scores, ld,
                                     stream)
               : launch_tpl<true, 4>(q, q_scale, k, k_scale, w, batch, rows, Lk, pos0, scores, ld,
                                     stream);
  else
    st = small ? launch_tpl<false, 1>(q, q_scale, k, k_scale, w, batch, rows, Lk, pos0, scores,
                                      ld, stream)
               : launch_tpl<false, 4>(q, q_scale, k, k_scale, w, batch, rows, Lk, pos0, scores,
                                      ld, stream);
  if (st || !fill_tail) return st;
  if (pos0 + 1 < Lk) {  // some row has masked keys
    st = cuda_check(launch_dep(fill_masked_kernel, dim3(static_cast<unsigned>(static_cast<long>(batch) * rows)),
                               dim3(256), 0, stream, 1, scores, ld, rows, Lk, pos0),
                    "fill_masked_kernel launch");
    if (!st)
      trace_launch(kKindFillMasked, stream,
                   4.0 * (static_cast<double>(rows) * Lk - causal_pairs(rows, Lk, pos0)) * batch);
  }
  return st;
}

}  // namespace ic
