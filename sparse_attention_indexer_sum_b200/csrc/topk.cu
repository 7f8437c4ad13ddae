// topk.cu -- exact per-row top-k over fp32 scores (routing loop T <- top-k(I) of
// "IndexCache: Wie DeepSeek O(NL^2)-Kosten in Sparse Attention um 75% reduziert";
// k = 2048 in its intro).  Ties go to the lower index, -0 == +0, output in
// ascending index order padded with -1.
//
// One CTA (512 threads) per row.  Scores are mapped to order-preserving 32-bit
// keys.  Common path: a threshold estimated from a 2% sample, one streaming pass
// that collects every key above it (unordered, warp-aggregated shared atomics),
// the exact k-th key among those candidates by radix selection, ties at it broken
// toward the lower index, and the selection written in ascending order from a
// shared-memory bitmap.  When the sample misjudges (or the row is heavily tied
// or very long), the exact path below runs instead:
//   1. histogram of the top 12 key bits over the row (shared-memory atomics,
//      128-bit loads); the bin holding the k-th largest is located with one
//      block scan.  If that bin holds more than CAP keys (heavily tied data),
//      further 12/8-bit histogram passes over the row narrow the prefix.
//   2. one ordered pass over the row (ballot-free block scans over 4-element
//      chunks) compacts, in index order, the keys strictly above the prefix
//      (selected for sure) and the keys equal to it (candidates) into shared
//      memory.
//   3. the candidates are resolved in shared memory by more radix digits, the
//      last tie broken by index order, and the two ascending index lists are
//      merged into the output row.
// In the common case each score is read twice from global memory (L2).
#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

constexpr int TK_THREADS = 512;
constexpr int TK_NW = TK_THREADS / 32;
constexpr int TK_NBINS = 4096;  // 12-bit digits
constexpr int TK_CAP = 6144;    // candidates kept in shared memory
constexpr int TK_SAMPLE = 4096; // keys sampled to estimate the threshold
constexpr int TK_EPT = 16;      // contiguous scores per thread per step of the ordered pass
constexpr int TK_CHUNK = TK_THREADS * TK_EPT;
constexpr int TK_MAXK = 2048;

constexpr int TK_BM_WORDS = 8192;  // selection bitmap: rows of up to 262144 scores
constexpr int TK_MAXTIE = 512;     // ties at the k-th key resolved in shared memory

struct TopkSmem {
  int hist[TK_NBINS];
  uint32_t cand_key[TK_CAP];
  int cand_idx[TK_CAP];
  union {
    struct {
      int gt_idx[TK_MAXK];
      int sel_idx[TK_MAXK];
    } ex;                            // exact path
    uint32_t bitmap[TK_BM_WORDS];    // fast path: selected indices
  } u;
  int scan_tmp[TK_NW];
  int bcast[4];
  int counter, ties;
};

// Exclusive block-wide prefix sum of v; *total receives the sum over the block.
__device__ __forceinline__ int block_excl_scan(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) tmp[w] = incl;
  __syncthreads();
  if (w == 0) {
    int t = (lane < TK_NW) ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < TK_NW) tmp[lane] = t;
  }
  __syncthreads();
  const int res = (w > 0 ? tmp[w - 1] : 0) + incl - v;
  *total = tmp[TK_NW - 1];
  __syncthreads();
  return res;
}

// Finds the bin B (of nbins) with count(bins > B) < need <= count(bins >= B).
// Writes B to sm.bcast[0] and count(bins > B) to sm.bcast[1].
// (If no bin qualifies -- inconsistent counts -- bin 0 and 0 are reported.)
template <typename Smem>
__device__ __forceinline__ void find_bin(Smem& sm, int nbins, int need) {
  if (threadIdx.x == 0) {
    sm.bcast[0] = 0;
    sm.bcast[1] = 0;
  }
  const int per = nbins / TK_THREADS;  // 8 (4096 bins) or 0 (256 bins)
  int local = 0;
  int b_lo = 0, b_hi = 0;
  if (per > 0) {
    b_lo = threadIdx.x * per;
    b_hi = b_lo + per;
  } else if (threadIdx.x < nbins) {
    b_lo = threadIdx.x;
    b_hi = b_lo + 1;
  }
  for (int b = b_lo; b < b_hi; ++b) local += sm.hist[b];
  int total;
  const int before = block_excl_scan(local, sm.scan_tmp, &total);
  int above = total - before - local;  // keys in bins owned by later threads
  for (int b = b_hi - 1; b >= b_lo; --b) {
    const int c = sm.hist[b];
    if (above < need && above + c >= need) {
      sm.bcast[0] = b;
      sm.bcast[1] = above;
    }
    above += c;
  }
  __syncthreads();
}

// Keys of scores [i0, i0 + 16) (0 past nv): four 128-bit loads when aligned and in range.
__device__ __forceinline__ void load_keys16(const float* __restrict__ x, int nv, bool vec, int i0,
                                            uint32_t (&k)[TK_EPT]) {
  if (vec && i0 + TK_EPT - 1 < nv) {
#pragma unroll
    for (int v = 0; v < TK_EPT / 4; ++v) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(x + i0 + 4 * v));
      k[4 * v + 0] = score_key(f.x);
      k[4 * v + 1] = score_key(f.y);
      k[4 * v + 2] = score_key(f.z);
      k[4 * v + 3] = score_key(f.w);
    }
  } else {
#pragma unroll
    for (int e = 0; e < TK_EPT; ++e) k[e] = (i0 + e < nv) ? score_key(__ldg(x + i0 + e)) : 0u;
  }
}

template <typename F>
__device__ __forceinline__ void for_row(const float* x, int nv, bool vec, F&& f) {
#pragma unroll 4
  for (int i0 = 4 * threadIdx.x; i0 < nv; i0 += 4 * TK_THREADS) {
    if (vec && i0 + 3 < nv) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(x + i0));
      f(i0, v.x);
      f(i0 + 1, v.y);
      f(i0 + 2, v.z);
      f(i0 + 3, v.w);
    } else {
      for (int e = 0; e < 4 && i0 + e < nv; ++e) f(i0 + e, __ldg(x + i0 + e));
    }
  }
}

// Exact radix selection over the whole row: 12-bit histogram passes narrow the
// bin of the k-th key (more passes only for heavily tied rows), one ordered pass
// compacts the keys above it and its candidates, the candidates are resolved in
// shared memory and the two ascending lists are merged into `out`.
__device__ __noinline__ void topk_exact(TopkSmem& sm, const float* __restrict__ x, int nv,
                                        bool vec, int k, int* __restrict__ out) {
  // ---------------------------------------------------------------- 1. radix passes
  uint32_t prefix = 0;
  int pbits = 0;
  int k_rem = k;
  int cand = 0;
  for (int level = 0; level < 3; ++level) {
    const int bits = (level < 2) ? 12 : 8;
    const int shift = 32 - pbits - bits;
    const int nb = 1 << bits;
    for (int b = threadIdx.x; b < nb; b += TK_THREADS) sm.hist[b] = 0;
    __syncthreads();
    const uint32_t mask = static_cast<uint32_t>(nb - 1);
    if (level == 0) {
      for_row(x, nv, vec, [&](int, float v) {
        atomicAdd(&sm.hist[score_key(v) >> shift], 1);
      });
    } else {
      const int hs = shift + bits;  // = 32 - pbits, in [8, 20]
      for_row(x, nv, vec, [&](int, float v) {
        const uint32_t key = score_key(v);
        if ((key >> hs) == prefix) atomicAdd(&sm.hist[(key >> shift) & mask], 1);
      });
    }
    __syncthreads();
    find_bin(sm, nb, k_rem);
    const int B = sm.bcast[0];
    const int above = sm.bcast[1];
    cand = sm.hist[B];
    prefix = (prefix << bits) | static_cast<uint32_t>(B);
    pbits += bits;
    k_rem -= above;
    __syncthreads();
    if (cand <= TK_CAP) break;
  }

  // ---------------------------------------------------------------- 2. ordered compaction
  const int hs = 32 - pbits;  // 20, 8 or 0
  int g_run = 0, c_run = 0;
  for (int c0 = 0; c0 < nv; c0 += 4 * TK_THREADS) {
    const int i0 = c0 + 4 * threadIdx.x;
    uint32_t keys[4];
    int cls[4];  // 2 = above the prefix, 1 = candidate, 0 = neither
    int ng = 0, nc = 0;
    if (vec && i0 + 3 < nv) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(x + i0));
      keys[0] = score_key(v.x);
      keys[1] = score_key(v.y);
      keys[2] = score_key(v.z);
      keys[3] = score_key(v.w);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) keys[e] = (i0 + e < nv) ? score_key(__ldg(x + i0 + e)) : 0u;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      cls[e] = 0;
      if (i0 + e < nv) {
        const uint32_t kp = (hs >= 32) ? 0u : (keys[e] >> hs);
        if (kp > prefix) {
          cls[e] = 2;
          ++ng;
        } else if (kp == prefix) {
          cls[e] = 1;
          ++nc;
        }
      }
    }
    int tot;
    const int ex = block_excl_scan(ng | (nc << 16), sm.scan_tmp, &tot);
    int gp = g_run + (ex & 0xFFFF), cp = c_run + (ex >> 16);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (cls[e] == 2) {
        if (gp < TK_MAXK) sm.u.ex.gt_idx[gp] = i0 + e;
        ++gp;
      } else if (cls[e] == 1) {
        const int lim = (pbits == 32) ? k_rem : TK_CAP;
        if (cp < lim) {
          sm.cand_key[cp] = keys[e];
          sm.cand_idx[cp] = i0 + e;
        }
        ++cp;
      }
    }
    g_run += tot & 0xFFFF;
    c_run += tot >> 16;
  }
  __syncthreads();
  const int G = g_run;
  if (G + k_rem != k || G >= TK_MAXK) {
    // cannot happen for finite inputs; leave a recognisable row rather than garbage
    if (threadIdx.x == 0) record_error(kErrTopkOverflow);
    for (int j = threadIdx.x; j < k; j += TK_THREADS) out[j] = -1;
    return;
  }

  // ---------------------------------------------------------------- 3. resolve candidates
  int S;
  if (pbits == 32) {
    // every candidate carries the same key: the first k_rem in index order win
    for (int j = threadIdx.x; j < k_rem; j += TK_THREADS) sm.u.ex.sel_idx[j] = sm.cand_idx[j];
    S = k_rem;
  } else {
    const int C = c_run;  // <= TK_CAP here
    while (pbits < 32) {
      const int bits = (32 - pbits) >= 12 ? 12 : (32 - pbits);
      const int shift = 32 - pbits - bits;
      const int nb = 1 << bits;
      const uint32_t mask = static_cast<uint32_t>(nb - 1);
      const int hsh = shift + bits;
      for (int b = threadIdx.x; b < nb; b += TK_THREADS) sm.hist[b] = 0;
      __syncthreads();
      for (int j = threadIdx.x; j < C; j += TK_THREADS) {
        const uint32_t key = sm.cand_key[j];
        if ((key >> hsh) == prefix) atomicAdd(&sm.hist[(key >> shift) & mask], 1);
      }
      __syncthreads();
      find_bin(sm, nb, k_rem);
      const int B = sm.bcast[0];
      k_rem -= sm.bcast[1];
      prefix = (prefix << bits) | static_cast<uint32_t>(B);
      pbits += bits;
      __syncthreads();
    }
    // prefix is now the exact k-th key T; take every key > T and the first k_rem keys == T
    const uint32_t T = prefix;
    const int take_eq = k_rem;
    int gt_run = 0, eq_run = 0;
    for (int c0 = 0; c0 < C; c0 += TK_THREADS) {
      const int j = c0 + threadIdx.x;
      uint32_t key = 0;
      int isgt = 0, iseq = 0;
      if (j < C) {
        key = sm.cand_key[j];
        isgt = key > T;
        iseq = key == T;
      }
      int tot;
      const int ex = block_excl_scan(isgt | (iseq << 16), sm.scan_tmp, &tot);
      const int gt_before = gt_run + (ex & 0xFFFF);
      const int eq_rank = eq_run + (ex >> 16);
      const int pos = gt_before + (eq_rank < take_eq ? eq_rank : take_eq);
      if (isgt || (iseq && eq_rank < take_eq)) sm.u.ex.sel_idx[pos] = sm.cand_idx[j];
      gt_run += tot & 0xFFFF;
      eq_run += tot >> 16;
    }
    S = k - G;
  }
  __syncthreads();

  // ---------------------------------------------------------------- merge two ascending lists
  for (int p = threadIdx.x; p < G; p += TK_THREADS) {
    const int v = sm.u.ex.gt_idx[p];
    int lo = 0, hi = S;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sm.u.ex.sel_idx[mid] < v) lo = mid + 1; else hi = mid;
    }
    if (in_bounds(p + lo < k, kErrBoundsTopk)) out[p + lo] = v;
  }
  for (int p = threadIdx.x; p < S; p += TK_THREADS) {
    const int v = sm.u.ex.sel_idx[p];
    int lo = 0, hi = G;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sm.u.ex.gt_idx[mid] < v) lo = mid + 1; else hi = mid;
    }
    if (in_bounds(p + lo < k, kErrBoundsTopk)) out[p + lo] = v;
  }
}

// The j-th largest of `count` keys held in shared memory (count >= j >= 1), by
// 12-bit histogram rounds over the keys (the last round takes the bits left).
// With bits = 24 it stops after two rounds and returns the lowest key of the j-th
// key's 24-bit bin (a lower bound: at least j keys are >= it).  common_bits > 0
// says every key shares its top common_bits bits with `common`: the rounds start
// below them.
__device__ uint32_t select_kth_smem(TopkSmem& sm, const uint32_t* keys, int count, int j,
                                    int bits_total = 32, int common_bits = 0,
                                    uint32_t common = 0u) {
  int pbits = common_bits < bits_total ? common_bits : bits_total;
  uint32_t prefix = pbits > 0 ? common >> (32 - pbits) : 0u;
  int need = j;
  while (pbits < bits_total) {
    const int bits = (32 - pbits) >= 12 ? 12 : (32 - pbits);
    const int shift = 32 - pbits - bits;
    const int nb = 1 << bits;
    const uint32_t mask = static_cast<uint32_t>(nb - 1);
    for (int b = threadIdx.x; b < nb; b += TK_THREADS) sm.hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < count; i += TK_THREADS) {
      const uint32_t key = keys[i];
      if (pbits == 0 || (key >> (shift + bits)) == prefix)
        atomicAdd(&sm.hist[(key >> shift) & mask], 1);
    }
    __syncthreads();
    find_bin(sm, nb, need);
    need -= sm.bcast[1];
    prefix = (prefix << bits) | static_cast<uint32_t>(sm.bcast[0]);
    pbits += bits;
    __syncthreads();
  }
  return pbits >= 32 ? prefix : (prefix << (32 - pbits));
}

__device__ __forceinline__ void mark_selected(TopkSmem& sm, int i) {
  atomicOr(&sm.u.bitmap[i >> 5], 1u << (i & 31));
}

// Every key >= tau among scores [lo, hi) into the candidate list, unordered (one
// shared atomic per warp and step, no block barriers); the count goes to
// sm.counter, which may exceed TK_CAP (entries past it are dropped).  lo is a
// multiple of TK_EPT.
__device__ __forceinline__ void collect_candidates(TopkSmem& sm, const float* __restrict__ x,
                                                   int lo, int hi, bool vec, uint32_t tau) {
  const int tid = threadIdx.x, lane = tid & 31;
  {
    uint32_t cur[TK_EPT], nxt[TK_EPT];
    load_keys16(x, hi, vec, lo + TK_EPT * tid, cur);
    for (int c0 = lo; c0 < hi; c0 += TK_CHUNK) {
      const int i0 = c0 + TK_EPT * tid;
      if (c0 + TK_CHUNK < hi) load_keys16(x, hi, vec, i0 + TK_CHUNK, nxt);
      int hits = 0;
#pragma unroll
      for (int e = 0; e < TK_EPT; ++e) hits += (i0 + e < hi && cur[e] >= tau) ? 1 : 0;
      int incl = hits;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int wtot = __shfl_sync(0xffffffffu, incl, 31);
      if (wtot) {
        int base = 0;
        if (lane == 31) base = atomicAdd(&sm.counter, wtot);
        base = __shfl_sync(0xffffffffu, base, 31);
        int pos = base + incl - hits;
        if (hits) {
#pragma unroll
          for (int e = 0; e < TK_EPT; ++e) {
            if (i0 + e < hi && cur[e] >= tau) {
              if (pos < TK_CAP) {
                sm.cand_key[pos] = cur[e];
                sm.cand_idx[pos] = i0 + e;
              }
              ++pos;
            }
          }
        }
      }
#pragma unroll
      for (int e = 0; e < TK_EPT; ++e) cur[e] = nxt[e];
    }
  }
}

__global__ void __launch_bounds__(TK_THREADS) topk_kernel(const float* __restrict__ scores, long ld,
                                                          int n, long pos0,
                                                          const int* __restrict__ valid_len,
                                                          int k, int* __restrict__ idx) {
  extern __shared__ uint8_t tk_smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(tk_smem_raw);
  const int tid = threadIdx.x;
  grid_dep_wait();
  // A row is split over the S CTAs of a cluster (S = 1 without clusters): each
  // collects the candidates of its part, CTA 0 merges them and selects.
  const uint32_t S = cluster_nctarank(), crank = cluster_ctarank();
  const long row = blockIdx.x / S;
  long nvl = valid_len ? static_cast<long>(__ldg(valid_len + row)) : (pos0 < 0) ? n : pos0 + row + 1;
  if (nvl > n) nvl = n;
  if (nvl < 0) nvl = 0;
  const int nv = static_cast<int>(nvl);
  int* out = idx + row * k;
  if (nv <= k) {
    if (crank == 0)
      for (int j = tid; j < k; j += TK_THREADS) out[j] = (j < nv) ? j : -1;
    return;
  }
  const float* x = scores + row * ld;
  const bool vec = ((ld & 3) == 0) && ((reinterpret_cast<uintptr_t>(scores) & 15) == 0);
  if (nv > TK_BM_WORDS * 32) {  // longer than the selection bitmap: exact multi-pass path
    if (crank == 0) topk_exact(sm, x, nv, vec, k, out);
    return;
  }
  const int nwords = (nv + 31) >> 5;
  for (int w = tid; w < nwords; w += TK_THREADS) sm.u.bitmap[w] = 0u;
  if (tid == 0) {
    sm.counter = 0;
    sm.ties = 0;
  }

  // ---- 1. threshold from a sample: the whole row when it is short, else 32 evenly
  //         spread runs of 128 contiguous scores (2% of a 200K row).  tau is a lower
  //         bound of the sample's j-th key, aimed at ~1.6 k keys >= tau in the row.
  uint32_t* samp = sm.cand_key;
  int m, j;
  if (nv <= TK_SAMPLE) {
    m = nv;
    for (int i = tid; i < nv; i += TK_THREADS) samp[i] = score_key(__ldg(x + i));
    j = k;  // at least k keys are >= the k-th key
  } else {
    m = TK_SAMPLE;
    const int run = TK_SAMPLE / 32;  // 128
    // every thread's loads go out before any is used
    constexpr int SPT = TK_SAMPLE / TK_THREADS;
    static_assert(TK_SAMPLE % TK_THREADS == 0, "whole sample loads per thread");
    float sv[SPT];
#pragma unroll
    for (int u = 0; u < SPT; ++u) {
      const int i = tid + u * TK_THREADS;
      const int b = i / run, o = i % run;
      const int start = static_cast<int>((static_cast<long>(b) * (nv - run)) / 31) & ~3;
      sv[u] = __ldg(x + start + o);
    }
#pragma unroll
    for (int u = 0; u < SPT; ++u) samp[tid + u * TK_THREADS] = score_key(sv[u]);
    const long jj = (static_cast<long>(k) * 16 * m + 10L * nv - 1) / (10L * nv);
    j = static_cast<int>(jj < 1 ? 1 : (jj > m ? m : jj));
  }
  __syncthreads();
  const uint32_t tau = select_kth_smem(sm, samp, m, j, 24);

  // ---- 2. one streaming pass over this CTA's part of the row: every key >= tau into
  //         the candidate list (unordered; one shared atomic per warp and step)
  const int seg = ((nv + S - 1) / S + TK_EPT - 1) / TK_EPT * TK_EPT;
  const int lo = min(nv, static_cast<int>(crank) * seg), hi = min(nv, lo + seg);
  collect_candidates(sm, x, lo, hi, vec, tau);
  __syncthreads();
  if (S > 1) {
    // ---- 2b. the leader appends the other CTAs' candidates (distributed shared memory)
    cluster_sync_all();  // every CTA's list is complete
    if (crank == 0) {
      const int own = sm.counter;
      int total = own;
      bool over = own > TK_CAP;
      for (uint32_t p = 1; p < S; ++p) {
        const int cnt = static_cast<int>(ld_cluster_u32(mapa_shared(smem_u32(&sm.counter), p)));
        over = over || cnt > TK_CAP;
        const int take = (!over && total + cnt <= TK_CAP) ? cnt : 0;
        const uint32_t rk = mapa_shared(smem_u32(sm.cand_key), p);
        const uint32_t ri = mapa_shared(smem_u32(sm.cand_idx), p);
        for (int c = tid; c < take; c += TK_THREADS) {
          sm.cand_key[total + c] = ld_cluster_u32(rk + 4u * c);
          sm.cand_idx[total + c] = static_cast<int>(ld_cluster_u32(ri + 4u * c));
        }
        total += cnt;
      }
      __syncthreads();
      if (tid == 0) sm.counter = over ? TK_CAP + 1 : total;
    }
    cluster_sync_all();  // the leader is done reading the others' lists
    if (crank != 0) return;
    __syncthreads();
  }
  const int C = sm.counter;
  if (C < k || C > TK_CAP) {
    // the sample misjudged the threshold (or the row is heavily tied): exact path
    topk_exact(sm, x, nv, vec, k, out);
    return;
  }

  // ---- 3. the exact k-th key T among the candidates
  // every candidate lies in [tau, max]: their common leading bits need no round
  uint32_t kmax = 0u;
  for (int i = tid; i < C; i += TK_THREADS) kmax = max(kmax, sm.cand_key[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  if ((tid & 31) == 0) sm.scan_tmp[tid >> 5] = static_cast<int>(kmax);
  __syncthreads();
  kmax = 0u;
#pragma unroll
  for (int w = 0; w < TK_NW; ++w) kmax = max(kmax, static_cast<uint32_t>(sm.scan_tmp[w]));
  __syncthreads();
  const int cbits = __clz(static_cast<int>(tau ^ kmax));  // 32 when tau == kmax
  const uint32_t T = select_kth_smem(sm, sm.cand_key, C, k, 32, cbits, tau);
  int gt_total, eq_total;
  {
    int lg = 0, le = 0;
    for (int i = tid; i < C; i += TK_THREADS) {
      const uint32_t key = sm.cand_key[i];
      lg += key > T ? 1 : 0;
      le += key == T ? 1 : 0;
    }
    int tot;
    block_excl_scan(lg | (le << 16), sm.scan_tmp, &tot);
    gt_total = tot & 0xFFFF;
    eq_total = tot >> 16;
  }
  const int take_eq = k - gt_total;  // >= 1
  if (eq_total > take_eq && eq_total > TK_MAXTIE) {
    topk_exact(sm, x, nv, vec, k, out);  // many ties at the k-th key: exact path
    return;
  }

  // ---- 4. mark the selection: keys > T, and the take_eq lowest indices among ties
  const bool all_ties = (eq_total == take_eq);
  for (int i = tid; i < C; i += TK_THREADS) {
    const uint32_t key = sm.cand_key[i];
    if (key > T || (all_ties && key == T)) {
      mark_selected(sm, sm.cand_idx[i]);
    } else if (key == T) {
      sm.hist[atomicAdd(&sm.ties, 1)] = sm.cand_idx[i];
    }
  }
  __syncthreads();
  if (!all_ties) {
    const int nt = sm.ties;
    for (int a = tid; a < nt; a += TK_THREADS) {
      const int v = sm.hist[a];
      int rank = 0;
      for (int b = 0; b < nt; ++b) rank += sm.hist[b] < v ? 1 : 0;
      if (rank < take_eq) mark_selected(sm, v);
    }
    __syncthreads();
  }

  // ---- 5. ascending output: contiguous bitmap words per thread, one block scan
  {
    const int wpt = (nwords + TK_THREADS - 1) / TK_THREADS;
    const int w0 = tid * wpt;
    const int w1 = min(nwords, w0 + wpt);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(sm.u.bitmap[w]);
    int tot;
    int pos = block_excl_scan(cnt, sm.scan_tmp, &tot);
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = sm.u.bitmap[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        if (in_bounds(pos < k, kErrBoundsTopk)) out[pos] = (w << 5) + b;
        ++pos;
        bits &= bits - 1;
      }
    }
  }
}

// ------------------------------------------------------------------ fused top-k merge
// The second half of the fused indexer -> top-k (indexer_tc.cu, one query per
// sequence): every (row, CTA piece) left a slot holding, in ascending index
// order, every key of its share of the row whose selection key (score key << 32
// | ~index) is >= the slot's tau, and, when tau != 0, at least k of them; the
// pieces of a row follow one another in index order.  So the row's k largest
// selection keys are all in the slots and all >= the largest tau.  One CTA per
// row gathers the slot keys >= that tau into shared memory (narrowing the bound
// by radix digits over the slots if too many pass), finds the exact k-th largest
// selection key by 12-bit radix rounds, and writes the indices of the slot keys
// >= it in slot order, which is ascending.  Selection keys are unique within a
// row, so exactly k keys are >= the k-th: ties need no separate handling.
constexpr int TM_CAP = 8192;  // selection keys gathered into shared memory

struct MergeSmem {
  uint64_t cand[TM_CAP];
  int hist[TK_NBINS];
  int scnt[512];        // keys per slot (clamped)
  int soff[513];        // prefix of scnt
  int scan_tmp[TK_NW];
  int bcast[4];
  int counter;
  unsigned long long tau, kmax;
};

// One radix round over keys offered by `each` (which calls its argument with
// (ok, key) for every key, in warp-uniform rounds): counts the keys >= lo whose
// top pbits bits equal prefix into sm.hist by their next `bits` bits, one shared
// atomic per distinct bin per warp.
template <typename Each>
__device__ __forceinline__ void merge_hist(MergeSmem& sm, Each&& each, uint64_t lo,
                                           uint64_t prefix, int pbits, int bits) {
  const int lane = threadIdx.x & 31;
  const int shift = 64 - pbits - bits;
  const uint64_t mask = (1ull << bits) - 1ull;
  for (int b = threadIdx.x; b < (1 << bits); b += TK_THREADS) sm.hist[b] = 0;
  __syncthreads();
  each([&](bool ok, uint64_t c) {
    int bin = -1;
    if (ok && c >= lo && (pbits == 0 || (c >> (64 - pbits)) == prefix))
      bin = static_cast<int>((c >> shift) & mask);
    const unsigned peers = __match_any_sync(0xffffffffu, bin);
    if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bin], __popc(peers));
  });
  __syncthreads();
}

// Calls f(ok, key) for every key of the row's slots, 8 loads in flight per thread.
// The loop runs the same number of rounds in every thread (f may use warp votes):
// past the last key, f gets ok = false.
template <typename F>
__device__ __forceinline__ void for_slot_keys(const MergeSmem& sm, const uint8_t* base, int nslot,
                                              long slot_bytes, F&& f) {
  const int tot = sm.soff[nslot];
  for (int f0 = 0; f0 < tot; f0 += 8 * TK_THREADS) {
    uint64_t c[8];
    bool ok[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int fi = f0 + u * TK_THREADS + static_cast<int>(threadIdx.x);
      ok[u] = fi < tot;
      c[u] = 0;
      if (ok[u]) {
        int j = 0;  // slot of flat index fi (few slots: linear search)
        while (sm.soff[j + 1] <= fi) ++j;
        c[u] = __ldg(reinterpret_cast<const unsigned long long*>(base + j * slot_bytes + 64) +
                     (fi - sm.soff[j]));
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) f(ok[u], c[u]);
  }
}

__global__ void __launch_bounds__(TK_THREADS) topk_merge_kernel(
    const uint8_t* __restrict__ slots, long nt, long total, int G, int maxp,
    long slot_bytes, int cb, int nv, int k, int* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t tm_smem_raw[];
  MergeSmem& sm = *reinterpret_cast<MergeSmem*>(tm_smem_raw);
  const int tid = threadIdx.x, lane = tid & 31;
  grid_dep_wait();
  const long row = blockIdx.x;
  int* out = idx + row * k;
  if (nv <= k) {  // every candidate is selected
    for (int j = tid; j < k; j += TK_THREADS) out[j] = (j < nv) ? j : -1;
    return;
  }
  const long first = (row * nt * G + G - 1) / total;
  const long last = ((row * nt + nt - 1) * G + G - 1) / total;
  int nslot = static_cast<int>(last - first + 1);
  if (nslot > 512) nslot = 512;  // cannot happen for a plan of <= 170 pieces per row
  const uint8_t* base = slots + row * static_cast<long>(maxp) * slot_bytes;
  if (tid == 0) {
    sm.tau = 0ull;
    sm.kmax = 0ull;
  }
  for (int j = tid; j < nslot; j += TK_THREADS) {
    int c = *reinterpret_cast<const int*>(base + j * slot_bytes);
    sm.scnt[j] = c < 0 ? 0 : (c > cb ? cb : c);
  }
  __syncthreads();
  for (int j = tid; j < nslot; j += TK_THREADS) {
    atomicMax(&sm.tau, *reinterpret_cast<const unsigned long long*>(base + j * slot_bytes + 8));
    if (sm.scnt[j] > 0)
      atomicMax(&sm.kmax, *reinterpret_cast<const unsigned long long*>(base + j * slot_bytes + 16));
  }
  if (tid == 0) {
    int acc = 0;
    for (int j = 0; j < nslot; ++j) {
      sm.soff[j] = acc;
      acc += sm.scnt[j];
    }
    sm.soff[nslot] = acc;
  }
  __syncthreads();
  uint64_t tau = sm.tau;

  // gather every slot key >= tau (the count may pass TM_CAP: then nothing is usable)
  auto gather = [&](uint64_t t) {
    if (tid == 0) sm.counter = 0;
    __syncthreads();
    for_slot_keys(sm, base, nslot, slot_bytes, [&](bool ok, uint64_t c) {
      const bool take = ok && c >= t;
      const unsigned m = __ballot_sync(0xffffffffu, take);
      if (m) {
        int p = 0;
        if (lane == 0) p = atomicAdd(&sm.counter, __popc(m));
        p = __shfl_sync(0xffffffffu, p, 0) + __popc(m & ((1u << lane) - 1u));
        if (take && p < TM_CAP) sm.cand[p] = c;
      }
    });
    __syncthreads();
    return sm.counter;
  };
  // Each slot's tau bounds only its own share, so many more than k keys of the row
  // pass the largest tau (about 17 k at the decode shape).  If the slots hold more
  // keys than fit, first narrow the bound by 12-bit digits over the slot keys >= tau
  // until the keys >= the k-th key's bin fit (usually one round), then gather.
  // every candidate lies in [tau, kmax]: the leading bits these share need no round
  const uint64_t kmax = sm.kmax;
  auto common = [&](uint64_t lo, int& pbits, uint64_t& prefix) {
    pbits = (lo >= kmax) ? 63 : __clzll(static_cast<long long>(lo ^ kmax));
    prefix = pbits == 0 ? 0ull : (lo >> (64 - pbits));
  };
  auto slot_each = [&](auto&& f) { for_slot_keys(sm, base, nslot, slot_bytes, f); };
  int C = 0;
  if (sm.soff[nslot] <= TM_CAP) {
    C = gather(tau);
  } else {
    uint64_t prefix;
    int pbits, need = k, above = 0;
    common(tau, pbits, prefix);
    for (;;) {
      const int bits = (64 - pbits) >= 12 ? 12 : 64 - pbits;
      merge_hist(sm, slot_each, tau, prefix, pbits, bits);
      find_bin(sm, 1 << bits, need);
      const int B = min(max(sm.bcast[0], 0), (1 << bits) - 1), gt = sm.bcast[1];
      const int inb = sm.hist[B];
      prefix = (prefix << bits) | static_cast<uint64_t>(B);
      pbits += bits;
      __syncthreads();
      if (above + gt + inb <= TM_CAP || pbits == 64) {
        const uint64_t edge = pbits == 64 ? prefix : prefix << (64 - pbits);
        if (edge > tau) tau = edge;
        break;
      }
      above += gt;
      need -= gt;
    }
    C = gather(tau);
    if (C > TM_CAP) {  // cannot happen: the descent stops once the keys >= tau fit
      if (tid == 0) record_error(kErrTopkOverflow);
      C = TM_CAP;
    }
  }

  // the exact k-th largest selection key T among the gathered keys (all in [tau, kmax])
  auto cand_each = [&](auto&& f) {
    for (int i0 = 0; i0 < C; i0 += TK_THREADS) {
      const int i = i0 + tid;
      f(i < C, i < C ? sm.cand[i] : 0ull);
    }
  };
  uint64_t prefix;
  int pbits, need = k;
  common(tau, pbits, prefix);
  uint64_t T;
  for (;;) {
    const int bits = (64 - pbits) >= 12 ? 12 : 64 - pbits;
    merge_hist(sm, cand_each, 0ull, prefix, pbits, bits);
    find_bin(sm, 1 << bits, need);
    const int B = min(max(sm.bcast[0], 0), (1 << bits) - 1), gt = sm.bcast[1];
    const int inb = sm.hist[B];
    prefix = (prefix << bits) | static_cast<uint64_t>(B);
    pbits += bits;
    __syncthreads();
    if (gt + inb == need || pbits == 64) {  // every key of bin B is selected
      T = pbits == 64 ? prefix : prefix << (64 - pbits);
      break;
    }
    need -= gt;
  }

  // the k keys >= T in slot order (ascending index): each round takes 8 x 512
  // slot keys, key f0 + 512 u + thread; a key's place counts the selected keys of
  // the earlier (u, warp) groups (scanned by warp 0) and of the lower lanes
  const int tot = sm.soff[nslot];
  const int warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  int wbase = 0;
  for (int f0 = 0; f0 < tot; f0 += 8 * TK_THREADS) {
    uint64_t c[8];
    unsigned m[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int fi = f0 + u * TK_THREADS + tid;
      c[u] = 0;
      if (fi < tot) {
        int j = 0;
        while (sm.soff[j + 1] <= fi) ++j;
        c[u] = __ldg(reinterpret_cast<const unsigned long long*>(base + j * slot_bytes + 64) +
                     (fi - sm.soff[j]));
      }
      m[u] = __ballot_sync(0xffffffffu, fi < tot && c[u] >= T);
    }
    if (lane == 0) {
#pragma unroll
      for (int u = 0; u < 8; ++u) sm.hist[u * TK_NW + warp] = __popc(m[u]);
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the 8 x TK_NW group counts, 4 per lane
      static_assert(8 * TK_NW == 128, "four group counts per lane");
      const int4 v = *reinterpret_cast<const int4*>(sm.hist + 4 * lane);
      const int sum = v.x + v.y + v.z + v.w;
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int ex = incl - sum;
      *reinterpret_cast<int4*>(sm.hist + 4 * lane) =
          make_int4(ex, ex + v.x, ex + v.x + v.y, ex + v.x + v.y + v.z);
      if (lane == 31) sm.counter = incl;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if ((m[u] >> lane) & 1u) {
        const int p = wbase + sm.hist[u * TK_NW + warp] + __popc(m[u] & lt);
        if (in_bounds(p < k, kErrBoundsMerge) && p < k)
          out[p] = static_cast<int>(~static_cast<uint32_t>(c[u]));
      }
    }
    wbase += sm.counter;
    __syncthreads();
  }
  if (wbase != k && tid == 0) record_error(kErrTopkOverflow);  // cannot happen
  for (int j = wbase + tid; j < k; j += TK_THREADS) out[j] = -1;
}

ic_status launch_topk_merge(const uint8_t* slots, long rows, long nt, long total, int G, int maxp,
                            size_t slot_bytes, int cb, int nv, int k, int* idx,
                            cudaStream_t stream) {
  if (rows == 0) return IC_OK;
  const int smem = static_cast<int>(sizeof(MergeSmem));
  ic_status st = cuda_check(
      cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
      "cudaFuncSetAttribute(topk_merge)");
  if (st) return st;
  st = cuda_check(launch_dep(topk_merge_kernel, dim3(static_cast<unsigned>(rows)),
                             dim3(TK_THREADS), smem, stream, 1, slots, nt, total, G, maxp,
                             static_cast<long>(slot_bytes), cb, nv, k, idx),
                  "topk_merge_kernel launch");
  if (st) return st;
  // algorithmic bytes: the index rows written (the candidates it reads depend on the data)
  trace_launch(kKindTopkMerge, stream, 4.0 * static_cast<double>(rows) * k);
  return IC_OK;
}

ic_status launch_topk(const float* scores, long rows, int n, long ld, long pos0, int k, int* idx,
                      cudaStream_t stream, const int* valid_len) {
  if (rows == 0) return IC_OK;
  const int smem = static_cast<int>(sizeof(TopkSmem));
  ic_status st = cuda_check(
      cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
      "cudaFuncSetAttribute(topk)");
  if (st) return st;
  // Few long rows (decode): split each row over a cluster of S CTAs, at most one
  // CTA per SM (64 rows of 200000 scores: S = 2 took 0.040 ms, S = 4 with two CTAs
  // per SM 0.044 ms, S = 8 0.071 ms).
  int S = 1;
  if (n >= 32768 && n <= TK_BM_WORDS * 32) {
    const long sms = num_sms();
    while (S < 8 && rows * 2 * S <= sms) S *= 2;
  }
  st = cuda_check(launch_dep(topk_kernel, dim3(static_cast<unsigned>(rows * S)), dim3(TK_THREADS),
                             smem, stream, static_cast<unsigned>(S), scores, ld, n, pos0,
                             valid_len, k, idx),
                  "topk_kernel launch");
  if (st) return st;
  // algorithmic bytes: every candidate score read once, the index rows written once
  // (with per-row lengths from the device the host counts every row as n long)
  const double cand = (pos0 < 0 || valid_len) ? static_cast<double>(rows) * n
                                              : static_cast<double>(causal_pairs(rows, n, pos0));
  trace_launch(kKindTopk, stream, 4.0 * cand + 4.0 * static_cast<double>(rows) * k);
  return IC_OK;
}

}  // namespace ic
