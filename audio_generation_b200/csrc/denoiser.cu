// The denoiser around the block stack: input projections, the text refiner's
// output norm, and norm_out with the two output heads.
//
// "MiniMaxH3Transformer3DModel" page: the two input patch projections
// (in_channels * prod(patch_size) -> hidden for video rows, audio_in_channels
// -> hidden for audio rows), the timestep MLP and the two output heads are
// float32 modules, the block stack bf16; text rows are the projected text
// condition (text_dim -> hidden) refined by num_refiner_layers token-refiner
// blocks; final_norm_eps is the epsilon of the refiner's output norm and of
// norm_out; `forward` returns the video and audio velocities in the row order
// of video_indices and audio_indices. "MiniMax H3 Inference Engine voor Mac
// computers", section "Exacte DiT fusions": per-modality final AdaLN before
// the heads.
//
// Every kernel here writes or reads the stack's compact fp32 residual stream
// xc [B, V, H] (the valid rows in packed order): a latent row i of a modality
// lives at xc row c_of_row[idx[i]].
//
// The patch projections (K = 96 or 32) and the heads (N = 96 or 32) are too
// narrow for the tensor cores' tiles; they run on the CUDA cores in fp32,
// with each thread holding one output column's weights (projections) or a
// 2-row x C/16-column block of outputs (heads).
#include "internal.cuh"
#include "sm100.cuh"

namespace h3 {
namespace {

constexpr int kProjRows = 32;        // latent rows staged per step
constexpr int kProjRowsPerCta = 256;

// xc[b, c_of_row[idx[i]], col] = sum_k W[col, k] lat[b, i, k]. Block: 256
// output columns (H % 256 == 0); each thread keeps its column's C weights in
// registers and streams the CTA's latent rows through shared memory.
template <int C>
__global__ void __launch_bounds__(256) k_patch_project(int rows, int n, int H, int V,
                                                       const float* __restrict__ lat,
                                                       const float* __restrict__ W,
                                                       const int32_t* __restrict__ idx,
                                                       const int32_t* __restrict__ c_of_row,
                                                       float* __restrict__ xc) {
  __shared__ __align__(16) float lat_s[kProjRows][C];
  __shared__ int dst_s[kProjRows];
  const int col = blockIdx.y * 256 + threadIdx.x;
  float w[C];
  {
    const float4* wr = reinterpret_cast<const float4*>(W + (size_t)col * C);
#pragma unroll
    for (int q = 0; q < C / 4; ++q) {
      const float4 v = __ldg(wr + q);
      w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
    }
  }
  const int r_begin = blockIdx.x * kProjRowsPerCta;
  const int r_end = min(rows, r_begin + kProjRowsPerCta);
  for (int r0 = r_begin; r0 < r_end; r0 += kProjRows) {
    __syncthreads();
    for (int e = threadIdx.x; e < kProjRows * C / 4; e += 256) {
      const int r = e / (C / 4), q = e % (C / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r0 + r < r_end) v = __ldg(reinterpret_cast<const float4*>(lat + (size_t)(r0 + r) * C) + q);
      reinterpret_cast<float4*>(&lat_s[r][0])[q] = v;
    }
    if (threadIdx.x < kProjRows) {
      const int g = r0 + threadIdx.x;
      int dst = -1;
      if (g < r_end) {
        const int b = g / n, i = g - b * n;
        dst = b * V + c_of_row[idx[i]];
      }
      dst_s[threadIdx.x] = dst;
    }
    __syncthreads();
    const int nr = min(kProjRows, r_end - r0);
    for (int r = 0; r < nr; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < C; ++k) acc = fmaf(w[k], lat_s[r][k], acc);
      xc[(size_t)dst_s[r] * H + col] = acc;
    }
  }
}

// LayerNorm (no affine) of fp32 rows src[b, i] into xc[b, c_of_row[idx[i]]]:
// one warp per row, shifted sums (shift = the row's first element) then a
// second read of the row.
__global__ void __launch_bounds__(256) k_rows_layer_norm(int rows, int n, int H, int V,
                                                         float eps, const float* __restrict__ src,
                                                         const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ c_of_row,
                                                         float* __restrict__ xc) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int b = row / n, i = row - b * n;
  const float4* x = reinterpret_cast<const float4*>(src + (size_t)row * H);
  float4* y = reinterpret_cast<float4*>(xc + ((size_t)b * V + c_of_row[idx[i]]) * H);
  const int n4 = H / 4;
  const float c = __shfl_sync(0xffffffffu, lane == 0 ? src[(size_t)row * H] : 0.f, 0);
  float sum = 0.f, sq = 0.f;
  for (int q = lane; q < n4; q += 32) {
    const float4 v = x[q];
    const float d0 = v.x - c, d1 = v.y - c, d2 = v.z - c, d3 = v.w - c;
    sum += (d0 + d1) + (d2 + d3);
    sq = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, sq))));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
  }
  const float dm = sum / (float)H;
  const float mean = c + dm;
  const float rstd = rsqrtf(fmaxf(sq / (float)H - dm * dm, 0.f) + eps);
  for (int q = lane; q < n4; q += 32) {
    const float4 v = x[q];
    y[q] = make_float4((v.x - mean) * rstd, (v.y - mean) * rstd, (v.z - mean) * rstd,
                       (v.w - mean) * rstd);
  }
}

constexpr int kHeadRows = 32;  // rows per CTA
constexpr int kHeadK = 64;     // K chunk staged in shared memory

// out[b, i, c] = sum_k W[c, k] h[k], h = LN(x) (1 + scale) + shift with x =
// xc[b, c_of_row[idx[i]]] and (shift, scale) = table[0..1] + tmod_out[t][0..1]
// for the row's timestep t. Row statistics first (one warp per row), then the
// K loop: a 32 x 64 chunk of h and a 64 x C chunk of W in shared memory, each
// thread accumulating 2 rows x C / 16 columns.
template <int C>
__global__ void __launch_bounds__(256) k_out_head(int rows, int n, int H, int V, float eps,
                                                  const float* __restrict__ xc,
                                                  const int32_t* __restrict__ idx,
                                                  const int32_t* __restrict__ c_of_row,
                                                  const int32_t* __restrict__ t_idx,
                                                  const float* __restrict__ table,
                                                  const float* __restrict__ tmod_out,
                                                  const float* __restrict__ W,
                                                  float* __restrict__ out) {
  constexpr int CPT = C / 16;  // columns per thread
  __shared__ float h_s[kHeadRows][kHeadK + 1];
  __shared__ float w_s[kHeadK][C];
  __shared__ float mu_s[kHeadRows], rs_s[kHeadRows];
  __shared__ long long src_s[kHeadRows];
  __shared__ int ti_s[kHeadRows];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kHeadRows;
  for (int rr = warp; rr < kHeadRows; rr += 8) {
    const int g = row0 + rr;
    float mean = 0.f, rstd = 0.f;
    long long src = 0;
    int ti = 0;
    if (g < rows) {
      const int b = g / n, i = g - b * n;
      const int r = idx[i];
      src = ((long long)b * V + c_of_row[r]) * H;
      ti = t_idx[r];
      const float4* x = reinterpret_cast<const float4*>(xc + src);
      const float c = __shfl_sync(0xffffffffu, lane == 0 ? xc[src] : 0.f, 0);
      float sum = 0.f, sq = 0.f;
      for (int q = lane; q < H / 4; q += 32) {
        const float4 v = x[q];
        const float d0 = v.x - c, d1 = v.y - c, d2 = v.z - c, d3 = v.w - c;
        sum += (d0 + d1) + (d2 + d3);
        sq = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, sq))));
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
      }
      const float dm = sum / (float)H;
      mean = c + dm;
      rstd = rsqrtf(fmaxf(sq / (float)H - dm * dm, 0.f) + eps);
    }
    if (lane == 0) {
      mu_s[rr] = mean;
      rs_s[rr] = rstd;
      src_s[rr] = src;
      ti_s[rr] = ti;
    }
  }
  const int rp = threadIdx.x / 16, cg = threadIdx.x % 16;  // rows 2 rp, 2 rp + 1
  float acc[2][CPT];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc[a][j] = 0.f;
  for (int k0 = 0; k0 < H; k0 += kHeadK) {
    __syncthreads();
    // h chunk: thread -> row t / 8, eight consecutive k
    {
      const int r = threadIdx.x / 8, kk = (threadIdx.x % 8) * 8;
      const bool live = row0 + r < rows;
      const float* x = xc + src_s[r] + k0 + kk;
      const float* sh = table + k0 + kk;
      const float* sc = table + H + k0 + kk;
      const float* msh = tmod_out + (size_t)ti_s[r] * 2 * H + k0 + kk;
      const float* msc = msh + H;
      const float mu = mu_s[r], rs = rs_s[r];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float v = live ? x[e] : 0.f;
        h_s[r][kk + e] = live ? fmaf((v - mu) * rs, 1.f + sc[e] + msc[e], sh[e] + msh[e]) : 0.f;
      }
    }
    // W chunk: w_s[k][c] = W[c, k0 + k]
    for (int e = threadIdx.x; e < kHeadK * C; e += 256) {
      const int k = e / C, c = e % C;
      w_s[k][c] = __ldg(W + (size_t)c * H + k0 + k);
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kHeadK; ++k) {
      const float h0 = h_s[2 * rp][k], h1 = h_s[2 * rp + 1][k];
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const float wv = w_s[k][cg * CPT + j];
        acc[0][j] = fmaf(h0, wv, acc[0][j]);
        acc[1][j] = fmaf(h1, wv, acc[1][j]);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    const int g = row0 + 2 * rp + a;
    if (g < rows) {
#pragma unroll
      for (int j = 0; j < CPT; ++j) out[(size_t)g * C + cg * CPT + j] = acc[a][j];
    }
  }
}

template <template <int> class Launch, typename... Args>
cudaError_t by_channels(int C, Args... args) {
  switch (C) {
    case 32: return Launch<32>::run(args...);
    case 64: return Launch<64>::run(args...);
    case 96: return Launch<96>::run(args...);
    case 128: return Launch<128>::run(args...);
    default: return cudaErrorInvalidValue;
  }
}

template <int C>
struct ProjectLaunch {
  static cudaError_t run(int B, int n, int H, int V, const float* lat, const float* W,
                         const int32_t* idx, const int32_t* c_of_row, float* xc,
                         cudaStream_t st) {
    const int rows = B * n;
    dim3 grid((rows + kProjRowsPerCta - 1) / kProjRowsPerCta, H / 256);
    k_patch_project<C><<<grid, 256, 0, st>>>(rows, n, H, V, lat, W, idx, c_of_row, xc);
    return cudaGetLastError();
  }
};

template <int C>
struct HeadLaunch {
  static cudaError_t run(int B, int n, int H, int V, float eps, const float* xc,
                         const int32_t* idx, const int32_t* c_of_row, const int32_t* t_idx,
                         const float* table, const float* tmod_out, const float* W, float* out,
                         cudaStream_t st) {
    const int rows = B * n;
    k_out_head<C><<<(rows + kHeadRows - 1) / kHeadRows, 256, 0, st>>>(
        rows, n, H, V, eps, xc, idx, c_of_row, t_idx, table, tmod_out, W, out);
    return cudaGetLastError();
  }
};

// y[i] = a[i] + s * y[i] over n floats (s = -1: the core residual a - y; the
// stored residual is added with a = y_old, s = 1 as y = x + r).
__global__ void k_combine(size_t n4, const float4* __restrict__ a, float s, float4* __restrict__ y) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 u = a[i], v = y[i];
    y[i] = make_float4(u.x + s * v.x, u.y + s * v.y, u.z + s * v.z, u.w + s * v.w);
  }
}

}  // namespace

cudaError_t launch_combine(size_t n, const float* a, float s, float* y, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const size_t n4 = n / 4;
  size_t grid = (n4 + 255) / 256;
  if (grid > (size_t)num_sms() * 16) grid = (size_t)num_sms() * 16;
  k_combine<<<(unsigned)grid, 256, 0, st>>>(n4, reinterpret_cast<const float4*>(a), s,
                                            reinterpret_cast<float4*>(y));
  return cudaGetLastError();
}

bool io_channels_supported(int C) { return C == 32 || C == 64 || C == 96 || C == 128; }

cudaError_t launch_patch_project(int B, int n, int H, int V, int C, const float* lat,
                                 const float* W, const int32_t* idx, const int32_t* c_of_row,
                                 float* xc, cudaStream_t st) {
  if (B == 0 || n == 0) return cudaSuccess;
  return by_channels<ProjectLaunch>(C, B, n, H, V, lat, W, idx, c_of_row, xc, st);
}

cudaError_t launch_rows_layer_norm(int B, int n, int H, int V, float eps, const float* src,
                                   const int32_t* idx, const int32_t* c_of_row, float* xc,
                                   cudaStream_t st) {
  const int rows = B * n;
  if (rows == 0) return cudaSuccess;
  k_rows_layer_norm<<<(rows + 7) / 8, 256, 0, st>>>(rows, n, H, V, eps, src, idx, c_of_row, xc);
  return cudaGetLastError();
}

cudaError_t launch_out_head(int B, int n, int H, int V, int C, float eps, const float* xc,
                            const int32_t* idx, const int32_t* c_of_row, const int32_t* t_idx,
                            const float* table, const float* tmod_out, const float* W,
                            float* out, cudaStream_t st) {
  if (B == 0 || n == 0) return cudaSuccess;
  return by_channels<HeadLaunch>(C, B, n, H, V, eps, xc, idx, c_of_row, t_idx, table, tmod_out,
                                 W, out, st);
}

}  // namespace h3
