// a2: timestep embedding -> timestep MLP -> shared AdaLN projection, fp32.
//
// "MiniMaxH3Transformer3DModel" page, constructor parameters: freq_dim is the
// size of the sinusoidal timestep embedding (timesteps consumed unscaled in
// [0, 1]); time_embed_hidden_dim is the timestep MLP's inner width;
// time_embed_dim is its output and the input of every AdaLN projection. The
// page also states that the timestep MLP is kept in float32.
//
//   e     = [cos(t f_i), sin(t f_i)],  f_i = 10^4^(-i / (freq_dim / 2))
//   h1    = W_t1 e
//   temb  = W_t2 SiLU(h1)
//   tmod  = W_proj SiLU(temb)          -> [n_t, 6, H]
//
// Runs once per forward for the distinct timestep values; tiny next to the
// blocks, so a plain shared-memory-tiled fp32 GEMM is used.
#include <math.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace h3 {
namespace {

__global__ void k_sinusoid(int n_t, int freq_dim, const float* __restrict__ t,
                           float* __restrict__ e) {
  const int half = freq_dim / 2;
  const int n = n_t * half;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += gridDim.x * blockDim.x) {
    const int r = idx / half, i = idx % half;
    const float f = expf(-9.210340371976184f * (float)i / (float)half);  // ln(10^4) = 9.2103...
    const float a = t[r] * f;
    float s, c;
    sincosf(a, &s, &c);
    e[(size_t)r * freq_dim + i] = c;
    e[(size_t)r * freq_dim + half + i] = s;
  }
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.f + expf(-x)); }

// C[n, o] = sum_k act(A[n, k]) * W[o, k]; 64x64 tile, 16-wide K slices, 4x4 per thread.
template <bool kSiluA>
__global__ void __launch_bounds__(256) k_sgemm_nt(int N, int O, int K,
                                                  const float* __restrict__ A,
                                                  const float* __restrict__ W,
                                                  float* __restrict__ C) {
  __shared__ float As[16][64 + 4];
  __shared__ float Ws[16][64 + 4];
  const int tid = threadIdx.x;
  const int n0 = blockIdx.y * 64, o0 = blockIdx.x * 64;
  const int tr = tid / 16, tc = tid % 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    // 64 rows x 16 k of A and of W: 1024 values each, 4 per thread
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = tid + 256 * q;
      const int r = e / 16, kk = e % 16;
      float a = 0.f, w = 0.f;
      if (n0 + r < N && k0 + kk < K) {
        a = A[(size_t)(n0 + r) * K + k0 + kk];
        if (kSiluA) a = silu_f(a);
      }
      if (o0 + r < O && k0 + kk < K) w = W[(size_t)(o0 + r) * K + k0 + kk];
      As[kk][r] = a;
      Ws[kk][r] = w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][tr * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tc * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = n0 + tr * 4 + i;
    if (n >= N) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = o0 + tc * 4 + j;
      if (o < O) C[(size_t)n * O + o] = acc[i][j];
    }
  }
}

template <bool kSilu>
cudaError_t sgemm(int N, int O, int K, const float* A, const float* W, float* C,
                  cudaStream_t st) {
  dim3 grid((O + 63) / 64, (N + 63) / 64);
  k_sgemm_nt<kSilu><<<grid, 256, 0, st>>>(N, O, K, A, W, C);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_timestep(const h3_dims& d, int n_t, const float* t, const float* w_t1,
                            const float* w_t2, const float* w_proj, float* tmod, float* ws,
                            cudaStream_t st) {
  if (n_t == 0) return cudaSuccess;
  float* e = ws;                                     // [n_t, freq_dim]
  float* h1 = e + (size_t)n_t * d.freq_dim;          // [n_t, time_hidden]
  float* temb = h1 + (size_t)n_t * d.time_hidden;    // [n_t, time_embed_dim]
  const int half = d.freq_dim / 2;
  int grid = (n_t * half + 255) / 256;
  if (grid > 4096) grid = 4096;
  k_sinusoid<<<grid, 256, 0, st>>>(n_t, d.freq_dim, t, e);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if ((err = sgemm<false>(n_t, d.time_hidden, d.freq_dim, e, w_t1, h1, st)) != cudaSuccess)
    return err;
  if ((err = sgemm<true>(n_t, d.time_embed_dim, d.time_hidden, h1, w_t2, temb, st)) !=
      cudaSuccess)
    return err;
  return sgemm<true>(n_t, 6 * d.hidden, d.time_embed_dim, temb, w_proj, tmod, st);
}

}  // namespace h3
