// misc.cu -- the small kernels of the path:
//  * per-row e4m3 quantisation of indexer inputs (OCP 8-bit floating point,
//    E4M3, with one fp32 scale per token, as the fp8 indexer variant takes them);
//  * the indexer on CUDA cores for fp32 inputs (small head counts and dims:
//    the fp32 workload has 4 heads of dim 32, far too small for tensor tiles).
#include <type_traits>

#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

// One warp per row of n (<= 1024, multiple of 8) values:
//   scale = amax / 448 (1 when amax == 0);  code = e4m3_rn_satfinite(x / scale)
// Both the scale and the quotient are IEEE fp32 divisions.
template <typename T>
__global__ void quant_e4m3_kernel(const T* __restrict__ x, long rows, int n,
                                  uint8_t* __restrict__ codes, float* __restrict__ scales) {
  grid_dep_wait();
  const long row = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const T* xr = x + row * n;
  float vals[32];
  float amax = 0.f;
  int cnt = 0;
  for (int i = lane; i < n; i += 32, ++cnt) {
    const float v = static_cast<float>(xr[i]);
    vals[cnt] = v;
    amax = fmaxf(amax, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  if (lane == 0) scales[row] = scale;
  cnt = 0;
  for (int i = lane; i < n; i += 32, ++cnt)
    codes[row * n + i] = static_cast<uint8_t>(
        __nv_cvt_float_to_fp8(__fdiv_rn(vals[cnt], scale), __NV_SATFINITE, __NV_E4M3));
}

ic_status launch_quant_e4m3(const void* x, bool bf16, long rows, int n, uint8_t* codes,
                            float* scales, cudaStream_t stream) {
  if (rows == 0) return IC_OK;
  const unsigned blocks = static_cast<unsigned>((rows * 32 + 255) / 256);
  const cudaError_t e =
      bf16 ? launch_dep(quant_e4m3_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, stream, 1,
                        static_cast<const __nv_bfloat16*>(x), rows, n, codes, scales)
           : launch_dep(quant_e4m3_kernel<float>, dim3(blocks), dim3(256), 0, stream, 1,
                        static_cast<const float*>(x), rows, n, codes, scales);
  ic_status st = cuda_check(e, "quant_e4m3_kernel launch");
  if (!st)
    trace_launch(kKindQuant, stream,
                 static_cast<double>(rows) * (n * ((bf16 ? 2.0 : 4.0) + 1.0) + 4.0));
  return st;
}

// The fp8 latent-KV cache row of a 576-dim bf16 latent row (656 bytes): the 512
// latent dims as e4m3 codes in four groups of 128, each group quantised as a row
// of quant_e4m3_kernel (scale = amax / 448, 1 for an all-zero group; code =
// e4m3_rn_satfinite(x / scale)); the four fp32 scales; the 64 rope dims in bf16.
// One warp per row: lane l quantises latent dims 16l..16l+15 (group l / 8).
__global__ void pack_kv_e4m3_kernel(const __nv_bfloat16* __restrict__ kv, long rows, long ld_kv,
                                    uint8_t* __restrict__ out, long ld_out) {
  grid_dep_wait();
  const long row = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const __nv_bfloat16* x = kv + row * ld_kv;
  uint8_t* o = out + row * ld_out;
  float v[16];
  const uint4 a = *reinterpret_cast<const uint4*>(x + 16 * lane);
  const uint4 b = *reinterpret_cast<const uint4*>(x + 16 * lane + 8);
  const __nv_bfloat16* pa = reinterpret_cast<const __nv_bfloat16*>(&a);
  const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(&b);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = __bfloat162float(pa[i]);
    v[8 + i] = __bfloat162float(pb[i]);
    amax = fmaxf(amax, fmaxf(fabsf(v[i]), fabsf(v[8 + i])));
  }
#pragma unroll
  for (int off = 4; off > 0; off >>= 1)  // the 8 lanes of the group
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint32_t c[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      word |= static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fdiv_rn(v[4 * w + j], scale),
                                                           __NV_SATFINITE, __NV_E4M3))
              << (8 * j);
    c[w] = word;
  }
  *reinterpret_cast<uint4*>(o + 16 * lane) = make_uint4(c[0], c[1], c[2], c[3]);
  if ((lane & 7) == 0) *reinterpret_cast<float*>(o + 512 + 4 * (lane / 8)) = scale;
  if (lane < 8)  // rope: dims 512..575, 16 bytes per lane
    *reinterpret_cast<uint4*>(o + 528 + 16 * lane) =
        *reinterpret_cast<const uint4*>(x + 512 + 8 * lane);
}

ic_status launch_pack_kv_e4m3(const void* kv, long rows, long ld_kv, uint8_t* out, long ld_out,
                              cudaStream_t stream) {
  if (rows == 0) return IC_OK;
  const unsigned blocks = static_cast<unsigned>((rows * 32 + 255) / 256);
  ic_status st = cuda_check(launch_dep(pack_kv_e4m3_kernel, dim3(blocks), dim3(256), 0, stream, 1,
                                       static_cast<const __nv_bfloat16*>(kv), rows, ld_kv, out,
                                       ld_out),
                            "pack_kv_e4m3_kernel launch");
  if (!st) trace_launch(kKindPackKv, stream, static_cast<double>(rows) * (576.0 * 2 + 656.0));
  return st;
}

// I[b,r,s] = sum_h w[b,r,h] * max(0, q[b,r,h,:] . k[b,s,:]) on CUDA cores.
// Grid (batch * rows, ceil(Lk / 128)); one key per thread, the query row in smem.
// Packed segments for the fp32 indexer (the rows of a launch that belong to each).
struct F32IdxSegs {
  int nseg;
  IdxSeg seg[IC_MAXSEG];
};
struct F32NoSegs {
  int unused;
};
template <bool SEGS>
using F32SegParam = typename std::conditional<SEGS, F32IdxSegs, F32NoSegs>::type;

// One CTA per (query row, 128-key tile).  With segments, launch row r belongs to
// the last segment j with seg[j].orow0 <= r: its position is seg.pos0 + (r -
// seg.orow0) and its keys are rows seg.krow0 .. seg.krow0 + seg.Lk - 1 of k.
template <bool SEGS>
__global__ void indexer_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                   const float* __restrict__ w, int R, int H, int D, int Lk,
                                   long pos0, float* __restrict__ scores, long ld,
                                   const __grid_constant__ F32SegParam<SEGS> sg) {
  extern __shared__ float qs[];  // [H * D] then w [H]
  const long row = blockIdx.x;   // b * R + r
  long kbase, pos;
  int lk;
  if constexpr (SEGS) {
    int lo = 0, hi = sg.nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sg.seg[mid].orow0 <= row)
        lo = mid;
      else
        hi = mid - 1;
    }
    kbase = sg.seg[lo].krow0;
    pos = sg.seg[lo].pos0 + (row - sg.seg[lo].orow0);
    lk = sg.seg[lo].Lk;
  } else {
    const long b = row / R, r = row % R;
    kbase = b * Lk;
    pos = pos0 + r;
    lk = Lk;
  }
  float* ws = qs + H * D;
  for (int i = threadIdx.x; i < H * D; i += blockDim.x) qs[i] = q[row * H * D + i];
  for (int i = threadIdx.x; i < H; i += blockDim.x) ws[i] = w[row * H + i];
  __syncthreads();
  const long s = static_cast<long>(blockIdx.y) * blockDim.x + threadIdx.x;
  if (s >= lk) return;
  float res = -INFINITY;
  if (s <= pos) {
    const float* ks = k + (kbase + s) * D;
    res = 0.f;
    for (int h = 0; h < H; ++h) {
      float dot = 0.f;
      for (int d = 0; d < D; ++d) dot = fmaf(qs[h * D + d], ks[d], dot);
      res = fmaf(ws[h], fmaxf(dot, 0.f), res);
    }
  }
  scores[row * ld + s] = res;
}

ic_status launch_indexer_f32(const float* q, const float* k, const float* w, int batch, int H,
                             int D, int rows, int Lk, long pos0, float* scores, long ld,
                             cudaStream_t stream) {
  if (static_cast<long>(batch) * rows == 0 || Lk == 0) return IC_OK;
  const int smem = (H * D + H) * static_cast<int>(sizeof(float));
  ic_status st = cuda_check(
      cudaFuncSetAttribute(indexer_f32_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem),
      "cudaFuncSetAttribute(indexer_f32)");
  if (st) return st;
  dim3 grid(static_cast<unsigned>(static_cast<long>(batch) * rows), static_cast<unsigned>((Lk + 127) / 128));
  indexer_f32_kernel<false><<<grid, 128, smem, stream>>>(q, k, w, rows, H, D, Lk, pos0, scores, ld,
                                                         F32NoSegs{0});
  st = cuda_check(cudaGetLastError(), "indexer_f32_kernel launch");
  if (!st)
    trace_launch(kKindIndexerF32, stream,
                 2.0 * H * D * static_cast<double>(causal_pairs(rows, Lk, pos0)) * batch);
  return st;
}

ic_status launch_indexer_f32_segs(const float* q, const float* k, const float* w, int H, int D,
                                  const IdxSeg* segs, int nseg, long rows, float* scores, long ld,
                                  cudaStream_t stream) {
  if (rows == 0) return IC_OK;
  if (nseg < 1 || nseg > IC_MAXSEG) return fail(IC_ERR_INVALID_ARG, "indexer: %d segments", nseg);
  F32IdxSegs sg;
  sg.nseg = nseg;
  int lkmax = 0;
  double flop = 0.0;
  for (int j = 0; j < nseg; ++j) {
    sg.seg[j] = segs[j];
    lkmax = segs[j].Lk > lkmax ? segs[j].Lk : lkmax;
    flop += 2.0 * H * D * static_cast<double>(causal_pairs(segs[j].R, segs[j].Lk, segs[j].pos0));
  }
  const int smem = (H * D + H) * static_cast<int>(sizeof(float));
  ic_status st = cuda_check(
      cudaFuncSetAttribute(indexer_f32_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem),
      "cudaFuncSetAttribute(indexer_f32)");
  if (st) return st;
  dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>((lkmax + 127) / 128));
  indexer_f32_kernel<true><<<grid, 128, smem, stream>>>(q, k, w, 1, H, D, lkmax, 0, scores, ld, sg);
  st = cuda_check(cudaGetLastError(), "indexer_f32_kernel launch");
  if (!st) trace_launch(kKindIndexerF32, stream, flop);
  return st;
}

// ------------------------------------------------------------------ packed rows
// valid_len[r] = position + 1 of score row r of a block of packed sequences: the
// block's rows of segment j are rows orow0.. at positions pos0.. (IdxSeg).
struct ValidSegs {
  int nseg;
  long orow0[IC_MAXSEG];
  long pos0[IC_MAXSEG];
};
__global__ void fill_valid_len_kernel(const __grid_constant__ ValidSegs v, long rows, int* out) {
  grid_dep_wait();
  const long r = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  int lo = 0, hi = v.nseg - 1;  // the last segment starting at or before row r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (v.orow0[mid] <= r)
      lo = mid;
    else
      hi = mid - 1;
  }
  out[r] = static_cast<int>(v.pos0[lo] + (r - v.orow0[lo]) + 1);
}

ic_status launch_fill_valid_len(const IdxSeg* segs, int nseg, long rows, int* out,
                                cudaStream_t stream) {
  if (rows <= 0) return IC_OK;
  if (nseg < 1 || nseg > IC_MAXSEG) return fail(IC_ERR_INVALID_ARG, "valid_len: %d segments", nseg);
  ValidSegs v;
  v.nseg = nseg;
  for (int j = 0; j < nseg; ++j) {
    v.orow0[j] = segs[j].orow0;
    v.pos0[j] = segs[j].pos0;
  }
  ic_status st = cuda_check(launch_dep(fill_valid_len_kernel,
                                       dim3(static_cast<unsigned>((rows + 255) / 256)), dim3(256), 0,
                                       stream, 1, v, rows, out),
                            "fill_valid_len_kernel launch");
  if (!st) trace_launch(kKindFillValid, stream, 4.0 * static_cast<double>(rows));
  return st;
}

}  // namespace ic
