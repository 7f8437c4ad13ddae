// attn.cu -- sparse attention over the index set (routing loop
// X <- SparseAttn(X, T) of "IndexCache: Wie DeepSeek O(NL^2)-Kosten in Sparse
// Attention um 75% reduziert"; MLA paragraph: one latent row shared by all heads).
//
// Absorbed MLA, bf16: 16 query heads of dim 576 attend over the selected rows
// of the 576-dim latent cache; the value of a row is its first 512 dims.
//
// The work is bound by gathering k latent rows (1152 B each) per query: with
// 16 heads there are only ~30 flops per gathered byte, far below the tensor
// ridge.  So the kernel is built around the gather: 16-byte cp.async row copies
// into a double-buffered shared tile of 32 rows (padded rows: conflict-free
// ldmatrix), and the two small contractions per tile -- S = Q K^T (16 x 32 x 576)
// and O += P V (16 x 512 x 32) -- on the warp-level bf16 tensor-core MMA, whose
// M = 16 matches the 16 heads exactly.  Softmax is online (running max / sum
// per head, base 2).
//
// CTA = 8 warps, one (query, split) item.  QK: warp w covers keys 8(w%4)..+8
// over dims 288(w/4)..+288 with its slice of Q held in registers; the two
// half-dim partial scores meet in shared memory.  PV: warp w owns output dims
// 64w..+64.  Decode-sized batches split each index list over several CTAs;
// their unnormalised partial outputs are merged by attn_combine_kernel.
#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

constexpr int AT_H = 16;
constexpr int AT_DK = 576;
constexpr int AT_DV = 512;
constexpr int AT_BK = 32;                   // keys per tile
constexpr int AT_THREADS = 256;
constexpr int AT_ROWB = AT_DK * 2 + 16;     // padded shared row: 1168 B
constexpr int AT_CHUNKS = AT_DK * 2 / 16;   // 72 16-byte chunks per row
constexpr int AT_PROWB = 80;                // padded P row (32 bf16 + 16 B)

struct AttnSmem {
  alignas(16) uint8_t kv[2][AT_BK][AT_ROWB];  // 74752 B
  alignas(16) uint8_t q[AT_H][AT_ROWB];       // 18688 B
  alignas(16) float s_part[2][AT_H][AT_BK];   // 4096 B
  alignas(16) uint8_t p[AT_H][AT_PROWB];      // 1280 B
  int idx[2][AT_BK];
  float m[AT_H], l[AT_H], alpha[AT_H];
  int last_valid;
};

struct AttnArgs {
  const __nv_bfloat16* q;   // [B, R, 16, 576]
  const __nv_bfloat16* kv;  // [B, Lkv, ld_kv]
  long ld_kv;
  const int* idx;           // [B, R, k]
  int B, R, Lkv, k;
  float scale_log2;         // softmax scale * log2(e)
  int nsplit, chunk;        // index list split into nsplit chunks of `chunk` entries
  __nv_bfloat16* out;       // [B, R, 16, 512]   (nsplit == 1)
  float* lse;               // [B, R, 16] or null (nsplit == 1)
  float* part_o;            // [B*R*nsplit, 16, 512] (nsplit > 1)
  float* part_ml;           // [B*R*nsplit, 16, 2]   (nsplit > 1)
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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

// Issue the copies of tile t (index-list entries j0 .. j0+31, clipped at `end`)
// into buffer `buf`; rows whose index is < 0 (or past the end) become zeros.
__device__ __forceinline__ void gather_tile(AttnSmem& sm, const AttnArgs& a, const int* irow,
                                            const __nv_bfloat16* kvb, int j0, int end, int buf) {
  for (int c = threadIdx.x; c < AT_BK * AT_CHUNKS; c += AT_THREADS) {
    const int row = c / AT_CHUNKS, ch = c % AT_CHUNKS;
    const int j = j0 + row;
    int s = (j < end) ? __ldg(irow + j) : -1;
    if (s >= a.Lkv) s = -1;
    uint8_t* dst = &sm.kv[buf][row][ch * 16];
    if (s >= 0)
      cp_async16(smem_u32(dst), reinterpret_cast<const uint8_t*>(kvb + static_cast<long>(s) * a.ld_kv) + ch * 16);
    else
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    if (ch == 0) sm.idx[buf][row] = s;
  }
}

__global__ void __launch_bounds__(AT_THREADS, 2) attn_mla_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t at_smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(at_smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long item = blockIdx.x;  // (b * R + r) * nsplit + sp
  const long qrow = item / a.nsplit;
  const int sp = static_cast<int>(item % a.nsplit);
  const long b = qrow / a.R;
  const int* irow = a.idx + qrow * a.k;
  const __nv_bfloat16* kvb = a.kv + b * static_cast<long>(a.Lkv) * a.ld_kv;
  const int beg = sp * a.chunk;
  int end = beg + a.chunk;
  if (end > a.k) end = a.k;

  // q rows of this query -> shared (async), trim trailing -1 entries of the list
  const __nv_bfloat16* qg = a.q + qrow * (AT_H * AT_DK);
  for (int c = tid; c < AT_H * AT_CHUNKS; c += AT_THREADS) {
    const int h = c / AT_CHUNKS, ch = c % AT_CHUNKS;
    cp_async16(smem_u32(&sm.q[h][ch * 16]), reinterpret_cast<const uint8_t*>(qg + h * AT_DK) + ch * 16);
  }
  if (tid == 0) sm.last_valid = beg - 1;
  if (tid < AT_H) {
    sm.m[tid] = -INFINITY;
    sm.l[tid] = 0.f;
  }
  __syncthreads();
  {
    int lv = beg - 1;
    for (int j = beg + tid; j < end; j += AT_THREADS)
      if (__ldg(irow + j) >= 0) lv = j;
    atomicMax(&sm.last_valid, lv);
  }
  __syncthreads();
  end = sm.last_valid + 1;
  const int ntiles = (end > beg) ? (end - beg + AT_BK - 1) / AT_BK : 0;

  if (ntiles > 0) gather_tile(sm, a, irow, kvb, beg, end, 0);
  cp_async_commit();  // group: q + tile 0
  cp_async_wait<0>();
  __syncthreads();

  // this warp's slice of Q as A fragments: 18 k-steps of 16 dims
  const int kh = warp >> 2, kg = warp & 3;
  uint32_t qa[18][4];
  {
    const uint32_t qbase = smem_u32(&sm.q[0][0]);
    const int r = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int cofs = 8 * (lane >> 4);
#pragma unroll
    for (int j = 0; j < 18; ++j) {
      const int col = kh * 288 + 16 * j + cofs;
      ldsm_x4(qbase + r * AT_ROWB + col * 2, qa[j][0], qa[j][1], qa[j][2], qa[j][3]);
    }
  }
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  const int g = lane >> 2, cq = lane & 3;
  for (int t = 0; t < ntiles; ++t) {
    const int buf = t & 1;
    if (t + 1 < ntiles) gather_tile(sm, a, irow, kvb, beg + (t + 1) * AT_BK, end, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    // ---- S partial = Q[:, dims of kh] . K[keys 8kg..8kg+7]
    {
      float sacc[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t kvbase = smem_u32(&sm.kv[buf][0][0]);
      const uint32_t rowaddr = kvbase + (8 * kg + (lane & 7)) * AT_ROWB;
#pragma unroll
      for (int jj = 0; jj < 9; ++jj) {
        uint32_t b0, b1, b2, b3;
        const int col = kh * 288 + 32 * jj + 8 * (lane >> 3);
        ldsm_x4(rowaddr + col * 2, b0, b1, b2, b3);
        mma_bf16(sacc, qa[2 * jj], b0, b1);
        mma_bf16(sacc, qa[2 * jj + 1], b2, b3);
      }
      sm.s_part[kh][g][8 * kg + 2 * cq] = sacc[0];
      sm.s_part[kh][g][8 * kg + 2 * cq + 1] = sacc[1];
      sm.s_part[kh][g + 8][8 * kg + 2 * cq] = sacc[2];
      sm.s_part[kh][g + 8][8 * kg + 2 * cq + 1] = sacc[3];
    }
    __syncthreads();

    // ---- online softmax: thread -> head tid/16, keys 2*(tid%16), +1
    {
      const int h = tid >> 4, c = (tid & 15) * 2;
      const float2 p0 = *reinterpret_cast<const float2*>(&sm.s_part[0][h][c]);
      const float2 p1 = *reinterpret_cast<const float2*>(&sm.s_part[1][h][c]);
      float z0 = (p0.x + p1.x) * a.scale_log2;
      float z1 = (p0.y + p1.y) * a.scale_log2;
      if (sm.idx[buf][c] < 0) z0 = -INFINITY;
      if (sm.idx[buf][c + 1] < 0) z1 = -INFINITY;
      float tmax = fmaxf(z0, z1);
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
      const float m_old = sm.m[h];
      const float m_new = fmaxf(m_old, tmax);
      float e0 = 0.f, e1 = 0.f, alpha = 1.f;
      if (m_new != -INFINITY) {
        e0 = exp2f(z0 - m_new);
        e1 = exp2f(z1 - m_new);
        alpha = exp2f(m_old - m_new);  // 0 when m_old = -inf
      }
      float rs = e0 + e1;
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
      *reinterpret_cast<uint32_t*>(&sm.p[h][c * 2]) = pack_bf16(e0, e1);
      __syncwarp();
      if ((tid & 15) == 0) {
        sm.l[h] = sm.l[h] * alpha + rs;
        sm.m[h] = m_new;
        sm.alpha[h] = alpha;
      }
    }
    __syncthreads();

    // ---- O[:, 64w..64w+64) = alpha * O + P V
    {
      const float al0 = sm.alpha[g], al1 = sm.alpha[g + 8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o[i][0] *= al0;
        o[i][1] *= al0;
        o[i][2] *= al1;
        o[i][3] *= al1;
      }
      const uint32_t pbase = smem_u32(&sm.p[0][0]);
      const uint32_t kvbase = smem_u32(&sm.kv[buf][0][0]);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        uint32_t pa[4];
        const int pr = (lane & 7) + 8 * ((lane >> 3) & 1);
        ldsm_x4(pbase + pr * AT_PROWB + (16 * ks + 8 * (lane >> 4)) * 2, pa[0], pa[1], pa[2], pa[3]);
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
    __syncthreads();
  }
  cp_async_wait<0>();

  // ---- epilogue
  const float l0 = sm.l[g], l1 = sm.l[g + 8];
  if (a.nsplit == 1) {
    const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
    __nv_bfloat16* ob = a.out + qrow * (AT_H * AT_DV);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int d = 64 * warp + 8 * i + 2 * cq;
      *reinterpret_cast<uint32_t*>(ob + g * AT_DV + d) = pack_bf16(o[i][0] * inv0, o[i][1] * inv0);
      *reinterpret_cast<uint32_t*>(ob + (g + 8) * AT_DV + d) = pack_bf16(o[i][2] * inv1, o[i][3] * inv1);
    }
    if (a.lse && tid < AT_H) {
      const float l = sm.l[tid];
      a.lse[qrow * AT_H + tid] = l > 0.f ? (sm.m[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  } else {
    float* po = a.part_o + item * (AT_H * AT_DV);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int d = 64 * warp + 8 * i + 2 * cq;
      *reinterpret_cast<float2*>(po + g * AT_DV + d) = make_float2(o[i][0], o[i][1]);
      *reinterpret_cast<float2*>(po + (g + 8) * AT_DV + d) = make_float2(o[i][2], o[i][3]);
    }
    if (tid < AT_H) {
      a.part_ml[(item * AT_H + tid) * 2] = sm.m[tid];
      a.part_ml[(item * AT_H + tid) * 2 + 1] = sm.l[tid];
    }
  }
}

// Merges the nsplit partial results of one query: per head,
// M = max m_i, L = sum l_i 2^(m_i - M), O = sum O_i 2^(m_i - M) / L.
__global__ void attn_combine_kernel(const float* part_o, const float* part_ml, int nsplit,
                                    __nv_bfloat16* out, float* lse) {
  const long qrow = blockIdx.x;
  const int h = blockIdx.y;
  __shared__ float wsh[64];
  __shared__ float inv_l;
  if (threadIdx.x == 0) {
    float M = -INFINITY;
    for (int i = 0; i < nsplit; ++i) M = fmaxf(M, part_ml[((qrow * nsplit + i) * AT_H + h) * 2]);
    float L = 0.f;
    for (int i = 0; i < nsplit; ++i) {
      const float mi = part_ml[((qrow * nsplit + i) * AT_H + h) * 2];
      const float li = part_ml[((qrow * nsplit + i) * AT_H + h) * 2 + 1];
      const float wi = (mi == -INFINITY) ? 0.f : exp2f(mi - M);
      wsh[i] = wi;
      L += li * wi;
    }
    inv_l = L > 0.f ? 1.f / L : 0.f;
    if (lse) lse[qrow * AT_H + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
  __syncthreads();
  for (int d = threadIdx.x; d < AT_DV; d += blockDim.x) {
    float acc = 0.f;
    for (int i = 0; i < nsplit; ++i)
      acc += wsh[i] * part_o[((qrow * nsplit + i) * AT_H + h) * AT_DV + d];
    out[(qrow * AT_H + h) * AT_DV + d] = __float2bfloat16_rn(acc * inv_l);
  }
}

static int pick_splits(long items, int k) {
  const long want = 4L * num_sms();  // 2 resident CTAs per SM, two waves
  if (items >= want) return 1;
  long s = (want + items - 1) / items;
  long maxs = (k + 255) / 256;  // at least 256 entries per split
  if (s > maxs) s = maxs;
  if (s > 64) s = 64;
  return s < 1 ? 1 : static_cast<int>(s);
}

size_t attn_mla_ws_bytes(int batch, int rows, int k) {
  const long items = static_cast<long>(batch) * rows;
  const int ns = pick_splits(items, k);
  if (ns <= 1) return 0;
  return static_cast<size_t>(items) * ns * AT_H * (AT_DV + 2) * sizeof(float);
}

ic_status launch_attn_mla(const void* q, const void* kv, long ld_kv, const int* idx, int batch,
                          int rows, int Lkv, int k, float scale, void* out, float* lse, void* ws,
                          size_t ws_bytes, long long valid_entries, cudaStream_t stream) {
  const long items = static_cast<long>(batch) * rows;
  if (items == 0) return IC_OK;
  int ns = pick_splits(items, k);
  const size_t per_split = static_cast<size_t>(items) * AT_H * (AT_DV + 2) * sizeof(float);
  while (ns > 1 && (ws == nullptr || per_split * ns > ws_bytes)) --ns;
  AttnArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kv = static_cast<const __nv_bfloat16*>(kv);
  a.ld_kv = ld_kv;
  a.idx = idx;
  a.B = batch;
  a.R = rows;
  a.Lkv = Lkv;
  a.k = k;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.nsplit = ns;
  a.chunk = ((k + ns - 1) / ns + AT_BK - 1) / AT_BK * AT_BK;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.part_o = static_cast<float*>(ws);
  a.part_ml = ns > 1 ? static_cast<float*>(ws) + items * ns * AT_H * AT_DV : nullptr;
  const int smem = static_cast<int>(sizeof(AttnSmem));
  ic_status st = cuda_check(
      cudaFuncSetAttribute(attn_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
      "cudaFuncSetAttribute(attn)");
  if (st) return st;
  attn_mla_kernel<<<static_cast<unsigned>(items * ns), AT_THREADS, smem, stream>>>(a);
  st = cuda_check(cudaGetLastError(), "attn_mla_kernel launch");
  if (st) return st;
  // algorithmic bytes: each selected latent row gathered once, q read once, out written once
  const double ve = valid_entries >= 0 ? static_cast<double>(valid_entries)
                                       : static_cast<double>(items) * k;
  const double io = static_cast<double>(items) * AT_H * (AT_DK + AT_DV) * 2.0;
  trace_launch(kKindAttnMla, stream, ve * AT_DK * 2.0 + io + 4.0 * static_cast<double>(items) * k);
  if (ns == 1) return IC_OK;
  attn_combine_kernel<<<dim3(static_cast<unsigned>(items), AT_H), 128, 0, stream>>>(
      a.part_o, a.part_ml, ns, a.out, lse);
  st = cuda_check(cudaGetLastError(), "attn_combine_kernel launch");
  if (!st)
    trace_launch(kKindAttnCombine, stream,
                 static_cast<double>(items) * AT_H * (ns * (AT_DV + 2) * 4.0 + AT_DV * 2.0));
  return st;
}

// ------------------------------------------------------------------ fp32 (MQA) form
// One CTA per query row, CUDA cores: small shapes only (the fp32 workload has
// 4 heads of dim 64 over k = 64 keys).
__global__ void attn_f32_kernel(const float* q, const float* kv, long ld_kv, const float* v,
                                const int* idx, int R, int heads, int dk, int dv, int Lkv, int k,
                                float scale, float* out, float* lse) {
  extern __shared__ float f32_smem[];
  float* qs = f32_smem;        // [dk]
  float* z = f32_smem + dk;    // [k]
  __shared__ float red[32];
  const long qrow = blockIdx.x;
  const long b = qrow / R;
  const int* irow = idx + qrow * k;
  const float* kvb = kv + b * static_cast<long>(Lkv) * ld_kv;
  const float* vb = v + b * static_cast<long>(Lkv) * dv;
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
                          int k, float scale, float* out, float* lse, cudaStream_t stream) {
  const long items = static_cast<long>(batch) * rows;
  if (items == 0) return IC_OK;
  const int smem = (dk + k) * static_cast<int>(sizeof(float));
  ic_status st = cuda_check(
      cudaFuncSetAttribute(attn_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
      "cudaFuncSetAttribute(attn_f32)");
  if (st) return st;
  attn_f32_kernel<<<static_cast<unsigned>(items), 128, smem, stream>>>(
      q, kv, ld_kv, v, idx, rows, heads, dk, dv, Lkv, k, scale, out, lse);
  st = cuda_check(cudaGetLastError(), "attn_f32_kernel launch");
  if (!st)
    trace_launch(kKindAttnF32, stream,
                 4.0 * static_cast<double>(items) * (k * (dk + dv) + heads * (dk + dv) + k));
  return st;
}

}  // namespace ic
