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
// Runs once per forward for the distinct timestep values. Two forms of the
// three fp32 GEMMs:
//  * few timesteps: a shared-memory-tiled fp32 GEMM on the CUDA cores (the
//    weights are read once, which dominates);
//  * many timesteps (n_t >= kSplitMinRows): each fp32 operand x is split into
//    three bf16 pieces x1 = bf16(x), x2 = bf16(x - x1), x3 = bf16(x - x1 - x2)
//    (24 significant bits, exact differences), and the six products of pieces
//    whose orders sum to at most 4 (x1y1, x1y2, x2y1, x1y3, x2y2, x3y1) are laid
//    side by side along K, so one bf16 tensor-core GEMM over K' = 6 K with fp32
//    accumulation gives the fp32 product to ~2^-22 relative (the dropped
//    products are below 2^-24 of the leading one).
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

constexpr int kSplitMinRows = 256;

// dst[r, p K + k] = piece(p) of act(src[r, k]), p = 0..5, with pieces
// (x1, x1, x2, x1, x2, x3) on the A side and (y1, y2, y1, y3, y2, y1) on the B
// side, so that the K' = 6 K dot product of an A row and a B row is
// x1y1 + x1y2 + x2y1 + x1y3 + x2y2 + x3y1. Four consecutive k per thread.
template <bool kSilu, bool kBSide>
__global__ void k_split3(int rows, int K, const float* __restrict__ src,
                         __nv_bfloat16* __restrict__ dst) {
  const int kq = K >> 2;
  const size_t n = (size_t)rows * kq;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (size_t)gridDim.x * blockDim.x) {
    const size_t r = idx / kq;
    const int k = (int)(idx - r * kq) * 4;
    float4 v = *reinterpret_cast<const float4*>(src + r * K + k);
    float x[4] = {v.x, v.y, v.z, v.w};
    __nv_bfloat16 pc[3][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a = kSilu ? silu_f(x[i]) : x[i];
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        pc[q][i] = __float2bfloat16_rn(a);
        a -= __bfloat162float(pc[q][i]);
      }
    }
    constexpr int kA[6] = {0, 0, 1, 0, 1, 2}, kB[6] = {0, 1, 0, 2, 1, 0};
    __nv_bfloat16* d = dst + r * 6 * (size_t)K + k;
#pragma unroll
    for (int p = 0; p < 6; ++p) {
      const int q = kBSide ? kB[p] : kA[p];
      uint2 u;
      u.x = (uint32_t)__bfloat16_as_ushort(pc[q][0]) | ((uint32_t)__bfloat16_as_ushort(pc[q][1]) << 16);
      u.y = (uint32_t)__bfloat16_as_ushort(pc[q][2]) | ((uint32_t)__bfloat16_as_ushort(pc[q][3]) << 16);
      *reinterpret_cast<uint2*>(d + (size_t)p * K) = u;
    }
  }
}

template <bool kSilu, bool kBSide>
cudaError_t split3(int rows, int K, const float* src, __nv_bfloat16* dst, cudaStream_t st) {
  const size_t n = (size_t)rows * (K >> 2);
  const int grid = (int)((n + 255) / 256 < 16384 ? (n + 255) / 256 : 16384);
  k_split3<kSilu, kBSide><<<grid, 256, 0, st>>>(rows, K, src, dst);
  return cudaGetLastError();
}

inline size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// The split form needs every K to be a multiple of 32 (K' = 6 K a multiple of
// the GEMM's 64-wide K slice) and every N a multiple of 256 or 224.
bool use_split(const h3_dims& d, int n_t, bool allow_split) {
  auto n_ok = [](int n) { return n % 256 == 0 || n % 224 == 0; };
  return allow_split && n_t >= kSplitMinRows && d.freq_dim % 32 == 0 &&
         d.time_hidden % 32 == 0 && d.time_embed_dim % 32 == 0 && n_ok(d.time_hidden) &&
         n_ok(d.time_embed_dim) && n_ok(6 * d.hidden);
}

// Bytes of the split operands of one GEMM stage: A' [n_t, 6K] and B' [N, 6K] bf16.
size_t stage_bytes(int n_t, int K, int N) {
  return align256((size_t)n_t * 6 * K * 2) + align256((size_t)N * 6 * K * 2);
}

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

size_t timestep_workspace_bytes(const h3_dims& d, int n_t, bool allow_split) {
  const size_t base = align256((size_t)n_t * (d.freq_dim + d.time_hidden + d.time_embed_dim) * 4);
  if (!use_split(d, n_t, allow_split)) return base;
  size_t st = stage_bytes(n_t, d.freq_dim, d.time_hidden);
  const size_t s2 = stage_bytes(n_t, d.time_hidden, d.time_embed_dim);
  const size_t s3 = stage_bytes(n_t, d.time_embed_dim, 6 * d.hidden);
  if (s2 > st) st = s2;
  if (s3 > st) st = s3;
  return base + st;
}

cudaError_t launch_timestep(const h3_dims& d, int n_t, const float* t, const float* w_t1,
                            const float* w_t2, const float* w_proj, float* tmod, void* ws,
                            bool allow_split, cudaStream_t st) {
  if (n_t == 0) return cudaSuccess;
  float* e = static_cast<float*>(ws);               // [n_t, freq_dim]
  float* h1 = e + (size_t)n_t * d.freq_dim;          // [n_t, time_hidden]
  float* temb = h1 + (size_t)n_t * d.time_hidden;    // [n_t, time_embed_dim]
  const int half = d.freq_dim / 2;
  int grid = (n_t * half + 255) / 256;
  if (grid > 4096) grid = 4096;
  k_sinusoid<<<grid, 256, 0, st>>>(n_t, d.freq_dim, t, e);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (!use_split(d, n_t, allow_split)) {
    if ((err = sgemm<false>(n_t, d.time_hidden, d.freq_dim, e, w_t1, h1, st)) != cudaSuccess)
      return err;
    if ((err = sgemm<true>(n_t, d.time_embed_dim, d.time_hidden, h1, w_t2, temb, st)) !=
        cudaSuccess)
      return err;
    return sgemm<true>(n_t, 6 * d.hidden, d.time_embed_dim, temb, w_proj, tmod, st);
  }
  // Split operands of one stage at a time, after the fp32 activations.
  uint8_t* stage = static_cast<uint8_t*>(ws) +
                   align256((size_t)n_t * (d.freq_dim + d.time_hidden + d.time_embed_dim) * 4);
  auto gemm_stage = [&](int K, int N, const float* a, bool silu_a, const float* w,
                        float* out) -> cudaError_t {
    __nv_bfloat16* as = reinterpret_cast<__nv_bfloat16*>(stage);
    __nv_bfloat16* bs = reinterpret_cast<__nv_bfloat16*>(stage + align256((size_t)n_t * 6 * K * 2));
    cudaError_t e2 = silu_a ? split3<true, false>(n_t, K, a, as, st)
                            : split3<false, false>(n_t, K, a, as, st);
    if (e2 != cudaSuccess) return e2;
    if ((e2 = split3<false, true>(N, K, w, bs, st)) != cudaSuccess) return e2;
    GemmEpiArgs ea{};
    ea.L.err = nullptr;
    ea.out = out;
    return launch_gemm(EPI_F32, n_t, N, 6 * K, as, bs, ea, st);
  };
  if ((err = gemm_stage(d.freq_dim, d.time_hidden, e, false, w_t1, h1)) != cudaSuccess) return err;
  if ((err = gemm_stage(d.time_hidden, d.time_embed_dim, h1, true, w_t2, temb)) != cudaSuccess)
    return err;
  return gemm_stage(d.time_embed_dim, 6 * d.hidden, temb, true, w_proj, tmod);
}

}  // namespace h3
