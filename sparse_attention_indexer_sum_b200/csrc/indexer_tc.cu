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
};

template <bool FP8, int TPM>
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
  static constexpr int STAGES = FP8 ? 8 : 4;
  static constexpr int NACC = (TPM == 4) ? 2 : 6;  // TMEM accumulators in the ring
  static constexpr int TMEM_COLS = (NACC * N <= 256) ? 256 : 512;
  static constexpr int EPG = (TPM == 4) ? 2 : 1;   // epilogue warps per TMEM lane quadrant
  // Epilogue warp sets: set j takes the accumulator slots a with a % NSETS == j, so
  // each set sees every use of its slots in order.  One-token blocks (decode) have
  // little epilogue work per tile; several sets overlap consecutive tiles.
  static constexpr int NSETS = (TPM == 4) ? 1 : 3;
  static constexpr int SETW = 4 * EPG;             // warps per set
  static constexpr int NEPI = SETW * NSETS;
  static constexpr int TOK_PER_EW = TPM / EPG;     // tokens per epilogue warp
  // MMA-issuing warps: tile i is issued by warp 1 + i % MMAW.  With N = 64
  // (one-token blocks) a tile's four or eight MMAs are short, and one thread's
  // issue loop (waits, MMAs, commits) sets the pace; two threads alternate
  // tiles.  With N = 256 the tensor pipe itself is the limit.
  static constexpr int MMAW = (TPM == 1) ? 2 : 1;
  static constexpr int EPI_W0 = 1 + MMAW;  // first epilogue warp
  static constexpr int THREADS = 32 * (EPI_W0 + NEPI);
  // TMEM columns an epilogue thread loads at a time: 16, so that the head
  // weights of both its tokens fit in registers beside them
  static constexpr int EPI_COLS = 16;  // matches tmem_ld16
  static constexpr int OFF_A = 0;
  static constexpr int OFF_Q = STAGES * A_BYTES;
  static constexpr int OFF_W = OFF_Q + Q_BYTES;
  static constexpr int W_FLOATS = NEPI * TOK_PER_EW * 64;
  static constexpr int OFF_BAR = OFF_W + W_FLOATS * 4;
  static constexpr int NBAR = 2 * STAGES + 2 * NACC + 3;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;  // + alignment slack
  static_assert(A_BYTES % 1024 == 0 && Q_BYTES % 1024 == 0, "swizzle atoms need 1 KB alignment");
  static_assert(N <= 256 && N % 16 == 0, "MMA N");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(NACC * N <= TMEM_COLS, "TMEM");
  static_assert(NACC % NSETS == 0, "each epilogue set owns whole accumulator slots");
};

template <int TPM>
__host__ __device__ __forceinline__ int qb_tiles(const IdxTcArgs& a, int qb) {
  int ql = qb % a.qb_per_batch;
  int r_last = min(ql * TPM + TPM, a.R) - 1;
  long keys = a.pos0 + r_last + 1;
  if (keys > a.Lk) keys = a.Lk;
  return static_cast<int>((keys + 127) / 128);
}

template <int TPM>
struct WorkIt {
  int qb, kt, nt;
  __device__ __forceinline__ void advance(const IdxTcArgs& a) {
    if (++kt >= nt) {
      kt = 0;
      ++qb;
      nt = (qb < a.nqb) ? qb_tiles<TPM>(a, qb) : 0;
    }
  }
};

// Drain wait used only after an abort: bounded by time alone.
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
  volatile int never = 0;
  (void)mbar_wait(bar, parity, &never, kErrTimeoutDrain);
}

template <bool FP8, int TPM>
__global__ void __launch_bounds__(IdxCfg<FP8, TPM>::THREADS, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmQ, const IdxTcArgs a) {
  using C = IdxCfg<FP8, TPM>;
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

  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* start = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
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
      const long t = (qb < a.nqb) ? qb_tiles<TPM>(a, qb) : 0;
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
        WorkIt<TPM> it{start[0], start[1], qb_tiles<TPM>(a, start[0])};
        int stage = 0;
        uint32_t ph = 0;
        int qloads = 0, cur_qb = -1;
        long issued = 0;
        for (long i = 0; i < nitems; ++i) {
          if (it.qb != cur_qb) {
            if (qloads > 0 &&
                !mbar_wait(qempty_bar, (qloads - 1) & 1, abort_flag, kErrTimeoutProducer))
              break;
            const int b = it.qb / a.qb_per_batch, ql = it.qb % a.qb_per_batch;
            const int qrow = (b * a.R + ql * TPM) * 64;
            mbar_arrive_expect_tx(qfull_bar, C::Q_BYTES);
#pragma unroll
            for (int kb = 0; kb < C::KBLK; ++kb)
              tma_load_2d(q_base + kb * (C::N * 128), &tmQ, kb * C::ELEMS_128B, qrow, qfull_bar);
            ++qloads;
            cur_qb = it.qb;
          }
          if (!mbar_wait(empty_bar(stage), ph ^ 1, abort_flag, kErrTimeoutProducer)) break;
          const int b = it.qb / a.qb_per_batch;
          const int krow = b * a.Lk + it.kt * C::BM;
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
        WorkIt<TPM> it{start[0], start[1], qb_tiles<TPM>(a, start[0])};
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
          WorkIt<TPM> nx = it;
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
    } else {
      // ------------------------------------------------------------ epilogue
      const int e = warp - C::EPI_W0;
      const int qd = warp & 3;     // TMEM lane quadrant this warp may access
      const int set = e / C::SETW;  // accumulator slots a with a % NSETS == set
      const int member = (e % C::SETW) / 4;  // which tokens of the block this warp reduces
      float* wsl = w_smem + e * C::TOK_PER_EW * 64;
      WorkIt<TPM> it{start[0], start[1], qb_tiles<TPM>(a, start[0])};
      int acc = 0;
      uint32_t aph = 0;
      int cur_qb = -1;
      // head weights of this warp's tokens, kept in registers while the query
      // block lasts (the values are then read from TMEM 16 columns at a time)
      float wr[C::TOK_PER_EW][64];
#pragma unroll
      for (int t = 0; t < C::TOK_PER_EW; ++t)
#pragma unroll
        for (int h = 0; h < 64; ++h) wr[t][h] = 0.f;
      for (long i = 0; i < nitems; ++i) {
        if (C::NSETS > 1 && acc % C::NSETS != set) {  // another set's slot
          if (++acc == C::NACC) {
            acc = 0;
            aph ^= 1;
          }
          it.advance(a);
          continue;
        }
        const int b = it.qb / a.qb_per_batch, ql = it.qb % a.qb_per_batch;
        const int r0 = ql * TPM + member * C::TOK_PER_EW;
        if (it.qb != cur_qb) {
          __syncwarp();
          for (int x = lane; x < C::TOK_PER_EW * 64; x += 32) {
            const int r = r0 + x / 64;
            float v = 0.f;
            if (r < a.R) {
              const long o = (static_cast<long>(b) * a.R + r) * 64 + (x % 64);
              v = a.w[o];
              if constexpr (FP8) v *= a.q_scale[o];
            }
            wsl[x] = v;
          }
          __syncwarp();
#pragma unroll
          for (int t = 0; t < C::TOK_PER_EW; ++t)
#pragma unroll
            for (int h = 0; h < 64; ++h) wr[t][h] = wsl[t * 64 + h];
          cur_qb = it.qb;
        }
        // this lane's key; its fp8 scale is fetched before the wait so the load's
        // latency hides behind it
        const int s = it.kt * C::BM + qd * 32 + lane;
        const bool key_ok = s < a.Lk && b < a.B;
        float ks = 1.f;
        if constexpr (FP8) ks = key_ok ? a.k_scale[static_cast<long>(b) * a.Lk + s] : 0.f;
        if (!mbar_wait(accfull_bar(acc), aph, abort_flag, kErrTimeoutEpilogue)) break;
        tc_fence_after();
        float res[C::TOK_PER_EW];
#pragma unroll
        for (int tk = 0; tk < C::TOK_PER_EW; ++tk) {
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) +
                                 static_cast<uint32_t>(acc * C::N + (member * C::TOK_PER_EW + tk) * 64);
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
          for (int part = 0; part < 64 / C::EPI_COLS; ++part) {  // heads in chunks of EPI_COLS
            float v[C::EPI_COLS];
            tmem_ld16(taddr + C::EPI_COLS * part, v);
            tmem_ld_wait();
#pragma unroll
            for (int h4 = 0; h4 < C::EPI_COLS / 4; ++h4) {
              const int h = C::EPI_COLS * part + 4 * h4;
              const float4 wv = make_float4(wr[tk][h], wr[tk][h + 1], wr[tk][h + 2], wr[tk][h + 3]);
              s0 = fmaf(wv.x, fmaxf(v[4 * h4 + 0], 0.f), s0);
              s1 = fmaf(wv.y, fmaxf(v[4 * h4 + 1], 0.f), s1);
              s2 = fmaf(wv.z, fmaxf(v[4 * h4 + 2], 0.f), s2);
              s3 = fmaf(wv.w, fmaxf(v[4 * h4 + 3], 0.f), s3);
            }
          }
          res[tk] = (s0 + s1) + (s2 + s3);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(accempty_bar(acc));
        if (key_ok) {
#pragma unroll
          for (int tk = 0; tk < C::TOK_PER_EW; ++tk) {
            const int r = r0 + tk;
            if (r < a.R) {
              const long pos = a.pos0 + r;
              a.scores[(static_cast<long>(b) * a.R + r) * a.ld + s] =
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

template <bool FP8, int TPM>
static ic_status launch_tpl(const void* q, const float* q_scale, const void* k,
                            const float* k_scale, const float* w, int batch, int rows, int Lk,
                            long pos0, float* scores, long ld, cudaStream_t stream) {
  using C = IdxCfg<FP8, TPM>;
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
  long total = 0;
  for (int qb = 0; qb < a.qb_per_batch; ++qb) total += qb_tiles<TPM>(a, qb);
  total *= batch;  // every batch has the same triangle
  a.total_tiles = total;
  if (total == 0) return IC_OK;

  CUtensorMap tmK, tmQ;
  ic_status st = make_map(&tmK, k, FP8, static_cast<uint64_t>(batch) * Lk, C::BM);
  if (st) return st;
  st = make_map(&tmQ, q, FP8, static_cast<uint64_t>(batch) * rows * 64, C::N);
  if (st) return st;

  st = cuda_check(cudaFuncSetAttribute(indexer_tc_kernel<FP8, TPM>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES),
                  "cudaFuncSetAttribute(indexer)");
  if (st) return st;
  const long grid = total < num_sms() ? total : num_sms();
  st = cuda_check(launch_dep(indexer_tc_kernel<FP8, TPM>, dim3(static_cast<unsigned>(grid)),
                             dim3(C::THREADS), C::SMEM_BYTES, stream, 1, tmK, tmQ, a),
                  "indexer_tc_kernel launch");
  if (st) return st;
  trace_launch(FP8 ? kKindIndexerE4m3 : kKindIndexerBf16, stream,
               2.0 * 64 * 128 * static_cast<double>(causal_pairs(rows, Lk, pos0)) * batch);
  return IC_OK;
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
