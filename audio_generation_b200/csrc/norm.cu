// a3 / a7: LayerNorm + AdaLN modulate, one warp per packed row.
//
// h = (x - mean) / sqrt(var + eps) * (1 + scale) + shift, the modulation of a
// row being selected by its modality tag and fed by its timestep
// ("MiniMaxH3Transformer3DModel" page: the per-row modality tag selects the
// AdaLN modulation parameters; norm_eps is the epsilon of the pre-attention
// and pre-feed-forward norms). shift / scale = ada_table[tag] + tmod[t_idx].
//
// HBM-bound: per row it reads H bf16 of x, 2H fp32 of tmod (per-row timestep)
// and writes H bf16 of h; the 3-row AdaLN table stays in L2, and the second
// read of x hits L1 / L2. All traffic is 16-byte vectors, lane-interleaved so a
// warp touches 512 contiguous bytes.
#include <cuda_fp8.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace h3 {
namespace {

constexpr int kMaxVecPerLane = 24;  // hidden <= 24 * 256 = 6144 (a limit of the other kernels)

// Eight values divided by the row scale (IEEE division, as the scale) and
// rounded to e4m3 codes (nearest even, saturating at +-448), packed in order.
__device__ __forceinline__ uint2 e4m3x8(const float* v, float sc) {
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t r = 0;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const float2 f = make_float2(__fdiv_rn(v[4 * h + 2 * p], sc), __fdiv_rn(v[4 * h + 2 * p + 1], sc));
      const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
      r |= (uint32_t)c << (16 * p);
    }
    w[h] = r;
  }
  return make_uint2(w[0], w[1]);
}

// Eight consecutive elements of a row, as floats.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* v) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
  v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}
__device__ __forceinline__ void load8(const float* p, float* v) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// XT is the storage type of the residual stream x: bf16 for a single block,
// fp32 inside the stack. Pass 1 accumulates the sum and the sum of squares of
// x - c (c = the row's first element, so the variance keeps its precision when
// the mean is far from zero); pass 2 reads x again (L1 / L2) together with the
// row's modulation and writes h. Nothing is held across the passes, so the
// kernel runs with few registers and many rows in flight per SM.
template <typename XT>
__global__ void __launch_bounds__(256) k_norm_modulate(
    int rows, int S, int H, int chunk_shift, int chunk_scale, float eps,
    const XT* __restrict__ x, const int32_t* __restrict__ tags,
    const int32_t* __restrict__ t_idx, const float* __restrict__ table,
    const float* __restrict__ tmod, uint4* __restrict__ h) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int s = row % S;
  const int nv = H >> 8;  // 8-element vectors per lane
  const XT* xr = x + (size_t)row * H;
  uint4* hr = h + (size_t)row * (H >> 3);
  const int tag = tags[s];
  if (tag < 0) {
    for (int i = 0; i < nv; ++i) hr[lane + 32 * i] = make_uint4(0, 0, 0, 0);
    return;
  }
  const int ti = t_idx[s];
  float c;
  {
    float v[8];
    load8(xr, v);
    c = __shfl_sync(0xffffffffu, v[0], 0);
  }
  float sum = 0.f, sq = 0.f;
#pragma unroll 4
  for (int i = 0; i < nv; ++i) {
    float v[8];
    load8(xr + 8 * (lane + 32 * i), v);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float d = v[k] - c;
      sum += d;
      sq = fmaf(d, d, sq);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
  }
  const float dm = sum / (float)H;
  const float mean = c + dm;
  const float var = fmaxf(sq / (float)H - dm * dm, 0.f);
  const float rstd = rsqrtf(var + eps);
  const float4* sh_t = reinterpret_cast<const float4*>(table + ((size_t)tag * 6 + chunk_shift) * H);
  const float4* sc_t = reinterpret_cast<const float4*>(table + ((size_t)tag * 6 + chunk_scale) * H);
  const float4* sh_m = reinterpret_cast<const float4*>(tmod + ((size_t)ti * 6 + chunk_shift) * H);
  const float4* sc_m = reinterpret_cast<const float4*>(tmod + ((size_t)ti * 6 + chunk_scale) * H);
#pragma unroll 2
  for (int i = 0; i < nv; ++i) {
    const int e4 = 2 * (lane + 32 * i);  // float4 index of the first of the 8 elements
    float xs[8];
    load8(xr + 8 * (lane + 32 * i), xs);
    float shv[8], scv[8];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float4 a = __ldg(sh_t + e4 + q), b = __ldg(sh_m + e4 + q);
      const float4 cc = __ldg(sc_t + e4 + q), d = __ldg(sc_m + e4 + q);
      shv[4 * q + 0] = a.x + b.x; shv[4 * q + 1] = a.y + b.y;
      shv[4 * q + 2] = a.z + b.z; shv[4 * q + 3] = a.w + b.w;
      scv[4 * q + 0] = cc.x + d.x; scv[4 * q + 1] = cc.y + d.y;
      scv[4 * q + 2] = cc.z + d.z; scv[4 * q + 3] = cc.w + d.w;
    }
    uint4 out;
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float y0 = (xs[2 * k] - mean) * rstd * (1.f + scv[2 * k]) + shv[2 * k];
      const float y1 = (xs[2 * k + 1] - mean) * rstd * (1.f + scv[2 * k + 1]) + shv[2 * k + 1];
      o[k] = pack_bf16x2(y0, y1);
    }
    hr[lane + 32 * i] = out;
  }
}

// The same h as e4m3 codes with one scale per row (s = max|h| / 448, codes =
// e4m3(h / s), round to nearest even, saturating), the A operand of the 8-bit
// QKV and W1 || W3 GEMMs. Pass 2 computes h for the row maximum, pass 3
// computes it again for the codes (x and the modulation rows come from L1 / L2
// by then). Padding rows get zero codes and scale 1.
template <typename XT>
__global__ void __launch_bounds__(256) k_norm_modulate_e4m3(
    int rows, int S, int H, int chunk_shift, int chunk_scale, float eps,
    const XT* __restrict__ x, const int32_t* __restrict__ tags,
    const int32_t* __restrict__ t_idx, const float* __restrict__ table,
    const float* __restrict__ tmod, uint2* __restrict__ codes, float* __restrict__ row_scale) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int s = row % S;
  const int nv = H >> 8;
  const XT* xr = x + (size_t)row * H;
  uint2* cr = codes + (size_t)row * (H >> 3);
  const int tag = tags[s];
  if (tag < 0) {
    for (int i = 0; i < nv; ++i) cr[lane + 32 * i] = make_uint2(0, 0);
    if (lane == 0) row_scale[row] = 1.f;
    return;
  }
  const int ti = t_idx[s];
  float c;
  {
    float v[8];
    load8(xr, v);
    c = __shfl_sync(0xffffffffu, v[0], 0);
  }
  float sum = 0.f, sq = 0.f;
#pragma unroll 4
  for (int i = 0; i < nv; ++i) {
    float v[8];
    load8(xr + 8 * (lane + 32 * i), v);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float d = v[k] - c;
      sum += d;
      sq = fmaf(d, d, sq);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
  }
  const float dm = sum / (float)H;
  const float mean = c + dm;
  const float var = fmaxf(sq / (float)H - dm * dm, 0.f);
  const float rstd = rsqrtf(var + eps);
  const float4* sh_t = reinterpret_cast<const float4*>(table + ((size_t)tag * 6 + chunk_shift) * H);
  const float4* sc_t = reinterpret_cast<const float4*>(table + ((size_t)tag * 6 + chunk_scale) * H);
  const float4* sh_m = reinterpret_cast<const float4*>(tmod + ((size_t)ti * 6 + chunk_shift) * H);
  const float4* sc_m = reinterpret_cast<const float4*>(tmod + ((size_t)ti * 6 + chunk_scale) * H);
  auto h8 = [&](int i, float* y) {
    const int e4 = 2 * (lane + 32 * i);
    float xs[8];
    load8(xr + 8 * (lane + 32 * i), xs);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float4 a = __ldg(sh_t + e4 + q), b = __ldg(sh_m + e4 + q);
      const float4 cc = __ldg(sc_t + e4 + q), d = __ldg(sc_m + e4 + q);
      y[4 * q + 0] = (xs[4 * q + 0] - mean) * rstd * (1.f + (cc.x + d.x)) + (a.x + b.x);
      y[4 * q + 1] = (xs[4 * q + 1] - mean) * rstd * (1.f + (cc.y + d.y)) + (a.y + b.y);
      y[4 * q + 2] = (xs[4 * q + 2] - mean) * rstd * (1.f + (cc.z + d.z)) + (a.z + b.z);
      y[4 * q + 3] = (xs[4 * q + 3] - mean) * rstd * (1.f + (cc.w + d.w)) + (a.w + b.w);
    }
  };
  float amax = 0.f;
#pragma unroll 2
  for (int i = 0; i < nv; ++i) {
    float y[8];
    h8(i, y);
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(y[k]));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  float sc = amax / 448.f;
  if (!(sc > 0.f)) sc = 1.f;
  if (lane == 0) row_scale[row] = sc;
#pragma unroll 2
  for (int i = 0; i < nv; ++i) {
    float y[8];
    h8(i, y);
    cr[lane + 32 * i] = e4m3x8(y, sc);
  }
}

// Weight rows [rows, K] bf16 -> e4m3 codes with one scale per row (max|w| / 448).
__global__ void __launch_bounds__(256) k_quantize_rows_e4m3(int rows, int K,
                                                            const __nv_bfloat16* __restrict__ w,
                                                            uint2* __restrict__ codes,
                                                            float* __restrict__ row_scale) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const __nv_bfloat16* wr = w + (size_t)row * K;
  uint2* cr = codes + (size_t)row * (K >> 3);
  const int nv = K >> 3;
  float amax = 0.f;
  for (int i = lane; i < nv; i += 32) {
    float v[8];
    load8(wr + 8 * i, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(v[k]));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  float sc = amax / 448.f;
  if (!(sc > 0.f)) sc = 1.f;
  if (lane == 0) row_scale[row] = sc;
  for (int i = lane; i < nv; i += 32) {
    float v[8];
    load8(wr + 8 * i, v);
    cr[i] = e4m3x8(v, sc);
  }
}

}  // namespace

cudaError_t launch_norm_modulate_e4m3(const LayoutView& L, int B, int H, int chunk_shift,
                                      int chunk_scale, float eps, const void* x, bool x_f32,
                                      const float* table, const float* tmod, void* codes,
                                      float* row_scale, cudaStream_t st) {
  const int rows = B * L.S;
  if (rows == 0) return cudaSuccess;
  if (H % 256 != 0 || H / 256 > kMaxVecPerLane) return cudaErrorInvalidValue;
  const int grid = (rows + 7) / 8;
  if (x_f32)
    k_norm_modulate_e4m3<float><<<grid, 256, 0, st>>>(rows, L.S, H, chunk_shift, chunk_scale, eps,
                                                      (const float*)x, L.tags, L.t_idx, table,
                                                      tmod, (uint2*)codes, row_scale);
  else
    k_norm_modulate_e4m3<__nv_bfloat16><<<grid, 256, 0, st>>>(
        rows, L.S, H, chunk_shift, chunk_scale, eps, (const __nv_bfloat16*)x, L.tags, L.t_idx,
        table, tmod, (uint2*)codes, row_scale);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows_e4m3(int rows, int K, const void* w, void* codes,
                                      float* row_scale, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  if (K % 8 != 0) return cudaErrorInvalidValue;
  k_quantize_rows_e4m3<<<(rows + 7) / 8, 256, 0, st>>>(rows, K, (const __nv_bfloat16*)w,
                                                       (uint2*)codes, row_scale);
  return cudaGetLastError();
}

cudaError_t launch_norm_modulate(const LayoutView& L, int B, int H, int chunk_shift,
                                 int chunk_scale, float eps, const void* x, bool x_f32,
                                 const float* table, const float* tmod, void* h,
                                 cudaStream_t st) {
  const int rows = B * L.S;
  if (rows == 0) return cudaSuccess;
  if (H % 256 != 0 || H / 256 > kMaxVecPerLane) return cudaErrorInvalidValue;
  const int warps_per_block = 8;
  const int grid = (rows + warps_per_block - 1) / warps_per_block;
  if (x_f32)
    k_norm_modulate<float><<<grid, 32 * warps_per_block, 0, st>>>(
        rows, L.S, H, chunk_shift, chunk_scale, eps, (const float*)x, L.tags, L.t_idx, table,
        tmod, (uint4*)h);
  else
    k_norm_modulate<__nv_bfloat16><<<grid, 32 * warps_per_block, 0, st>>>(
        rows, L.S, H, chunk_shift, chunk_scale, eps, (const __nv_bfloat16*)x, L.tags, L.t_idx,
        table, tmod, (uint4*)h);
  return cudaGetLastError();
}

}  // namespace h3
