// a3 / a7: LayerNorm + AdaLN modulate, one warp per packed row.
//
// h = (x - mean) / sqrt(var + eps) * (1 + scale) + shift, the modulation of a
// row being selected by its modality tag and fed by its timestep
// ("MiniMaxH3Transformer3DModel" page: the per-row modality tag selects the
// AdaLN modulation parameters; norm_eps is the epsilon of the pre-attention
// and pre-feed-forward norms). shift / scale = ada_table[tag] + tmod[t_idx].
//
// HBM-bound: per row it reads H bf16 of x, 2H fp32 of tmod (per-row timestep)
// and writes H bf16 of h; the 3-row AdaLN table stays in L2. All traffic is
// 16-byte vectors, lane-interleaved so a warp touches 512 contiguous bytes.
#include "internal.cuh"
#include "sm100.cuh"

namespace h3 {
namespace {

constexpr int kMaxVecPerLane = 24;  // hidden <= 24 * 256 = 6144

__global__ void __launch_bounds__(256) k_norm_modulate(
    int rows, int S, int H, int chunk_shift, int chunk_scale, float eps,
    const uint4* __restrict__ x, const int32_t* __restrict__ tags,
    const int32_t* __restrict__ t_idx, const float* __restrict__ table,
    const float* __restrict__ tmod, uint4* __restrict__ h) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int s = row % S;
  const int nv = H >> 8;  // 16-byte vectors per lane
  const uint4* xr = x + (size_t)row * (H >> 3);
  uint4* hr = h + (size_t)row * (H >> 3);
  const int tag = tags[s];
  if (tag < 0) {
    for (int i = 0; i < nv; ++i) hr[lane + 32 * i] = make_uint4(0, 0, 0, 0);
    return;
  }
  uint4 v[kMaxVecPerLane];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxVecPerLane; ++i) {
    if (i < nv) {
      v[i] = xr[lane + 32 * i];
      const uint32_t* u = reinterpret_cast<const uint32_t*>(&v[i]);
#pragma unroll
      for (int k = 0; k < 4; ++k) sum += bf16lo(u[k]) + bf16hi(u[k]);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / (float)H;
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxVecPerLane; ++i) {
    if (i < nv) {
      const uint32_t* u = reinterpret_cast<const uint32_t*>(&v[i]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float a = bf16lo(u[k]) - mean, b = bf16hi(u[k]) - mean;
        sq += a * a + b * b;
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = rsqrtf(sq / (float)H + eps);
  const int ti = t_idx[s];
  const float4* sh_t = reinterpret_cast<const float4*>(table + ((size_t)tag * 6 + chunk_shift) * H);
  const float4* sc_t = reinterpret_cast<const float4*>(table + ((size_t)tag * 6 + chunk_scale) * H);
  const float4* sh_m = reinterpret_cast<const float4*>(tmod + ((size_t)ti * 6 + chunk_shift) * H);
  const float4* sc_m = reinterpret_cast<const float4*>(tmod + ((size_t)ti * 6 + chunk_scale) * H);
#pragma unroll
  for (int i = 0; i < kMaxVecPerLane; ++i) {
    if (i < nv) {
      const int e4 = 2 * (lane + 32 * i);  // float4 index of the first of 8 elements
      const uint32_t* u = reinterpret_cast<const uint32_t*>(&v[i]);
      float xs[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        xs[2 * k] = bf16lo(u[k]);
        xs[2 * k + 1] = bf16hi(u[k]);
      }
      float shv[8], scv[8];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const float4 a = __ldg(sh_t + e4 + q), b = __ldg(sh_m + e4 + q);
        const float4 c = __ldg(sc_t + e4 + q), d = __ldg(sc_m + e4 + q);
        shv[4 * q + 0] = a.x + b.x; shv[4 * q + 1] = a.y + b.y;
        shv[4 * q + 2] = a.z + b.z; shv[4 * q + 3] = a.w + b.w;
        scv[4 * q + 0] = c.x + d.x; scv[4 * q + 1] = c.y + d.y;
        scv[4 * q + 2] = c.z + d.z; scv[4 * q + 3] = c.w + d.w;
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
}

}  // namespace

cudaError_t launch_norm_modulate(const LayoutView& L, int B, int H, int chunk_shift,
                                 int chunk_scale, float eps, const void* x, const float* table,
                                 const float* tmod, void* h, cudaStream_t st) {
  const int rows = B * L.S;
  if (rows == 0) return cudaSuccess;
  if (H % 256 != 0 || H / 256 > kMaxVecPerLane) return cudaErrorInvalidValue;
  const int warps_per_block = 8;
  const int grid = (rows + warps_per_block - 1) / warps_per_block;
  k_norm_modulate<<<grid, 32 * warps_per_block, 0, st>>>(rows, L.S, H, chunk_shift, chunk_scale,
                                                          eps, (const uint4*)x, L.tags, L.t_idx,
                                                          table, tmod, (uint4*)h);
  return cudaGetLastError();
}

}  // namespace h3
