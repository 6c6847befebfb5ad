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
//   tmod_out = W_out SiLU(temb)        -> [n_t, 2, H] (norm_out's shift and scale,
//                                         when the caller asks for it)
//
// Runs once per forward for the distinct timestep values. Two forms of the
// three fp32 GEMMs:
//  * few timesteps (n_t < kSplitMinRows): a skinny fp32 kernel on the CUDA cores
//    that streams the weights once per chunk of eight timesteps (HBM-bound);
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

// Error word of the split form's GEMMs (which have no layout object): a wait
// that runs out records H3_DEVERR_TIMEOUT here; h3_timestep_error reads and
// clears it. One int per GPU that loads the library.
static __device__ int g_prologue_err;

SymbolAddressCache g_err_cache;

cudaError_t lookup_err(void** p) { return cudaGetSymbolAddress(p, g_prologue_err); }

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

constexpr int kSplitMinRows = 65;

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

// C[n, o] = sum_k A[n, k] W[o, k] for few rows n: each warp streams two rows
// of W once (16-byte loads, coalesced across the warp) against a chunk of up to
// kSkinnyRows rows of A (small enough to stay in L1 / L2), keeps the 2 x
// kSkinnyRows partial dot products per lane and reduces them across the warp
// at the end. Blocks along y take successive chunks of A's rows. HBM-bound on
// W for a handful of rows.
constexpr int kSkinnyRows = 8;

__global__ void __launch_bounds__(256) k_skinny_nt(int N, int O, int K,
                                                   const float* __restrict__ A,
                                                   const float* __restrict__ W,
                                                   float* __restrict__ C) {
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.y * kSkinnyRows;
  const int nr = min(kSkinnyRows, N - n0);
  const int k4n = K >> 2;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long wp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       2 * wp < O; wp += warps) {
    const int o0 = (int)(2 * wp), o1 = min(o0 + 1, O - 1);
    const float4* w0 = reinterpret_cast<const float4*>(W + (size_t)o0 * K);
    const float4* w1 = reinterpret_cast<const float4*>(W + (size_t)o1 * K);
    float acc0[kSkinnyRows] = {}, acc1[kSkinnyRows] = {};
    for (int k4 = lane; k4 < k4n; k4 += 32) {
      const float4 a0 = __ldg(w0 + k4), a1 = __ldg(w1 + k4);
#pragma unroll
      for (int r = 0; r < kSkinnyRows; ++r) {
        if (r < nr) {
          const float4 x = __ldg(reinterpret_cast<const float4*>(A + (size_t)(n0 + r) * K) + k4);
          acc0[r] = fmaf(a0.x, x.x, fmaf(a0.y, x.y, fmaf(a0.z, x.z, fmaf(a0.w, x.w, acc0[r]))));
          acc1[r] = fmaf(a1.x, x.x, fmaf(a1.y, x.y, fmaf(a1.z, x.z, fmaf(a1.w, x.w, acc1[r]))));
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kSkinnyRows; ++r) {
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        acc0[r] += __shfl_xor_sync(0xffffffffu, acc0[r], off);
        acc1[r] += __shfl_xor_sync(0xffffffffu, acc1[r], off);
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < kSkinnyRows; ++r) {
        if (r < nr) {
          C[(size_t)(n0 + r) * O + o0] = acc0[r];
          if (o1 != o0) C[(size_t)(n0 + r) * O + o1] = acc1[r];
        }
      }
    }
  }
}

__global__ void k_silu_inplace(size_t n, float* __restrict__ x) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    x[i] = silu_f(x[i]);
}

cudaError_t skinny(int N, int O, int K, const float* A, const float* W, float* C,
                   cudaStream_t st) {
  const int chunks = (N + kSkinnyRows - 1) / kSkinnyRows;
  int gx = (O / 2 + 7) / 8;  // eight warps (two rows of W each) per block
  if (gx > 4 * 148 * 8) gx = 4 * 148 * 8;
  k_skinny_nt<<<dim3(gx, chunks), 256, 0, st>>>(N, O, K, A, W, C);
  return cudaGetLastError();
}

cudaError_t silu_inplace(size_t n, float* x, cudaStream_t st) {
  size_t grid = (n + 255) / 256;
  if (grid > 16384) grid = 16384;
  k_silu_inplace<<<(unsigned)grid, 256, 0, st>>>(n, x);
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
                            bool allow_split, cudaStream_t st, const float* w_out,
                            float* tmod_out) {
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
    // SiLU is applied once, in place, to each GEMM's input activations.
    if ((err = skinny(n_t, d.time_hidden, d.freq_dim, e, w_t1, h1, st)) != cudaSuccess) return err;
    if ((err = silu_inplace((size_t)n_t * d.time_hidden, h1, st)) != cudaSuccess) return err;
    if ((err = skinny(n_t, d.time_embed_dim, d.time_hidden, h1, w_t2, temb, st)) != cudaSuccess)
      return err;
    if ((err = silu_inplace((size_t)n_t * d.time_embed_dim, temb, st)) != cudaSuccess) return err;
    if (w_out && (err = skinny(n_t, 2 * d.hidden, d.time_embed_dim, temb, w_out, tmod_out, st)) !=
                     cudaSuccess)
      return err;
    return skinny(n_t, 6 * d.hidden, d.time_embed_dim, temb, w_proj, tmod, st);
  }
  // Split operands of one stage at a time, after the fp32 activations.
  void* err_word = nullptr;
  if (symbol_address(g_err_cache, lookup_err, &err_word) != H3_OK) return cudaErrorUnknown;
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
    ea.L.err = static_cast<int*>(err_word);
    ea.out = out;
    return launch_gemm(EPI_F32, n_t, N, 6 * K, as, bs, ea, st);
  };
  if ((err = gemm_stage(d.freq_dim, d.time_hidden, e, false, w_t1, h1)) != cudaSuccess) return err;
  if ((err = gemm_stage(d.time_hidden, d.time_embed_dim, h1, true, w_t2, temb)) != cudaSuccess)
    return err;
  if (w_out && (err = gemm_stage(d.time_embed_dim, 2 * d.hidden, temb, true, w_out, tmod_out)) !=
                   cudaSuccess)
    return err;
  return gemm_stage(d.time_embed_dim, 6 * d.hidden, temb, true, w_proj, tmod);
}

}  // namespace h3

extern "C" h3_status h3_timestep_error(void) {
  void* p = nullptr;
  if (h3::symbol_address(h3::g_err_cache, h3::lookup_err, &p) != H3_OK) return H3_ERR_CUDA;
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return H3_ERR_CUDA;
  if (cudaMemcpy(&v, p, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return H3_ERR_CUDA;
  if (v != 0 && cudaMemset(p, 0, 4) != cudaSuccess) return H3_ERR_CUDA;
  return v == 0 ? H3_OK : H3_ERR_TIMEOUT;
}
