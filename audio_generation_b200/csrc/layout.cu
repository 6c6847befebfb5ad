// a0 layout validation / tables and a1 packed-row gather-scatter.
//
// The packed layout is the one the `forward` arguments of
// MiniMaxH3Transformer3DModel describe (diffusers docs): per-row tags
// (0 video, 1 text, 2 audio, -1 padding), per-row timestep indices, (t, h, w)
// positions and the video / audio / text index tensors. Rows tagged -1 form
// their own attention document.
#include <math.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace h3 {

namespace {

constexpr int ST_TAG = 1, ST_TIDX = 2, ST_POS = 4, ST_IDX_RANGE = 8, ST_IDX_TAG = 16,
              ST_IDX_DUP = 32, ST_COUNT = 64;

__global__ void k_validate_rows(int S, int n_t, const int32_t* __restrict__ tags,
                                const int32_t* __restrict__ t_idx, const float* __restrict__ pos,
                                int32_t* __restrict__ src_of_row, int32_t* __restrict__ hits,
                                int32_t* __restrict__ tile_pad, int32_t* __restrict__ counts,
                                int* __restrict__ status) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < S; r += gridDim.x * blockDim.x) {
    const int tg = tags[r];
    int st = 0;
    if (tg < -1 || tg > 2) st |= ST_TAG;
    const int ti = t_idx[r];
    if (ti < 0 || ti >= n_t) st |= ST_TIDX;
    if (!isfinite(pos[3 * r]) || !isfinite(pos[3 * r + 1]) || !isfinite(pos[3 * r + 2]))
      st |= ST_POS;
    if (st) atomicOr(status, st);
    if (tg >= -1 && tg <= 2) atomicAdd(&counts[tg + 1], 1);
    if (tg < 0) atomicAdd(&tile_pad[r / kTile], 1);
    src_of_row[r] = -1;
    hits[r] = 0;
  }
}

__global__ void k_validate_index(int S, int n, int tag, const int32_t* __restrict__ idx,
                                 const int32_t* __restrict__ tags, int32_t* __restrict__ hits,
                                 int32_t* __restrict__ src_of_row, int* __restrict__ status) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int r = idx[i];
    if (r < 0 || r >= S) {
      atomicOr(status, ST_IDX_RANGE);
      continue;
    }
    if (tags[r] != tag) atomicOr(status, ST_IDX_TAG);
    atomicAdd(&hits[r], 1);
    src_of_row[r] = (tag << 28) | i;
  }
}

// cos / sin of pos[r][a] * rope_theta^(-j/16), evaluated in double and rounded once.
__global__ void k_rope_table(int S, const float* __restrict__ pos, double theta,
                             float2* __restrict__ rope) {
  const int n = S * kRopePairs;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const int r = e / kRopePairs, aj = e % kRopePairs, a = aj / kRopeFreqs, j = aj % kRopeFreqs;
    const double inv = pow(theta, -(double)j / (double)kRopeFreqs);
    const double ang = (double)pos[3 * r + a] * inv;
    double s, c;
    sincos(ang, &s, &c);
    rope[e] = make_float2((float)c, (float)s);
  }
}

// One block of 1024 threads: duplicate / count checks, tile classes, valid-key
// bitmasks and the compaction order (stable partition by a block-wide scan).
__global__ void __launch_bounds__(1024) k_finalize(
    int S, int n_tiles, int n_video, int n_text, int n_audio, const int32_t* __restrict__ tags,
    const int32_t* __restrict__ hits, const int32_t* __restrict__ tile_pad,
    const int32_t* __restrict__ counts, uint8_t* __restrict__ tile_class,
    uint32_t* __restrict__ key_valid, int32_t* __restrict__ perm, int* __restrict__ status,
    int* __restrict__ n_valid_out) {
  __shared__ int warp_sums[32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  int st = 0;
  for (int r = tid; r < S; r += blockDim.x)
    if (hits[r] > 1) st |= ST_IDX_DUP;
  if (tid == 0) {
    if (counts[1] != n_video || counts[2] != n_text || counts[3] != n_audio) st |= ST_COUNT;
  }
  if (st) atomicOr(status, st);
  for (int t = tid; t < n_tiles; t += blockDim.x) {
    const int rows = min(kTile, S - t * kTile);
    const int p = tile_pad[t];
    tile_class[t] = p == 0 ? 0 : (p == rows ? 1 : 2);
  }
  // valid-key bitmask, one 32-row word per warp iteration
  const int n_words = n_tiles * 4;
  for (int w0 = wid; w0 < n_words; w0 += 32) {
    const int r = w0 * 32 + lane;
    const bool valid = r < S && tags[r] >= 0;
    const uint32_t m = __ballot_sync(0xffffffffu, valid);
    if (lane == 0) key_valid[w0] = m;
  }
  // stable partition: valid rows first, then padding rows
  const int chunk = (S + blockDim.x - 1) / blockDim.x;
  const int r0 = min(S, tid * chunk), r1 = min(S, r0 + chunk);
  int cnt = 0;
  for (int r = r0; r < r1; ++r) cnt += tags[r] >= 0;
  int incl = cnt;
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int v = warp_sums[lane];
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    warp_sums[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  const int before = incl - cnt + (wid > 0 ? warp_sums[wid - 1] : 0);
  const int total_valid = warp_sums[31];
  int vpos = before, ppos = total_valid + (r0 - before);
  for (int r = r0; r < r1; ++r) {
    if (tags[r] >= 0)
      perm[vpos++] = r;
    else
      perm[ppos++] = r;
  }
  if (tid == 0) *n_valid_out = total_valid;
}

// Tables of the compacted (valid rows only) sequence.
__global__ void k_compact_tables(int V, int c_tiles, const int32_t* __restrict__ perm,
                                 const int32_t* __restrict__ tags,
                                 const int32_t* __restrict__ t_idx,
                                 const float2* __restrict__ rope, int32_t* __restrict__ c_tags,
                                 int32_t* __restrict__ c_tidx, float2* __restrict__ c_rope,
                                 uint8_t* __restrict__ c_tile_class,
                                 uint32_t* __restrict__ c_key_valid) {
  const int stride = gridDim.x * blockDim.x;
  const int t0 = blockIdx.x * blockDim.x + threadIdx.x;
  for (int j = t0; j < V; j += stride) {
    const int r = perm[j];
    c_tags[j] = tags[r];
    c_tidx[j] = t_idx[r];
  }
  for (int e = t0; e < V * kRopePairs; e += stride) {
    const int j = e / kRopePairs;
    c_rope[e] = rope[(size_t)perm[j] * kRopePairs + (e % kRopePairs)];
  }
  for (int t = t0; t < c_tiles; t += stride) c_tile_class[t] = 0;
  for (int w = t0; w < c_tiles * 4; w += stride) {
    const int lo = w * 32;
    const int nval = max(0, min(32, V - lo));
    c_key_valid[w] = nval == 32 ? 0xffffffffu : ((1u << nval) - 1u);
  }
}

// c_of_row[perm[j]] = j for the V valid rows (the caller fills c_of_row with -1).
__global__ void k_compact_position(int V, const int32_t* __restrict__ perm,
                                   int32_t* __restrict__ c_of_row) {
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < V; j += gridDim.x * blockDim.x)
    c_of_row[perm[j]] = j;
}

// ---- a1: packed-row gather / scatter, one warp per row, 16-byte vectors ----

__global__ void k_pack(int B, int S, int vec_per_row, const int32_t* __restrict__ src_of_row,
                       const uint4* __restrict__ video, int n_video,
                       const uint4* __restrict__ text, int n_text,
                       const uint4* __restrict__ audio, int n_audio, uint4* __restrict__ x) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < (long long)B * S; row += warps) {
    const int b = (int)(row / S), s = (int)(row % S);
    const int src = src_of_row[s];
    uint4* dst = x + row * vec_per_row;
    if (src < 0) {
      for (int v = lane; v < vec_per_row; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const int tag = src >> 28, i = src & 0x0FFFFFFF;
    const uint4* base = tag == 0 ? video : (tag == 1 ? text : audio);
    const int n = tag == 0 ? n_video : (tag == 1 ? n_text : n_audio);
    const uint4* sp = base + ((long long)b * n + i) * vec_per_row;
    for (int v = lane; v < vec_per_row; v += 32) dst[v] = sp[v];
  }
}

__global__ void k_unpack(int B, int S, int vec_per_row, const int32_t* __restrict__ src_of_row,
                         const uint4* __restrict__ x, uint4* __restrict__ video, int n_video,
                         uint4* __restrict__ text, int n_text, uint4* __restrict__ audio,
                         int n_audio) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < (long long)B * S; row += warps) {
    const int b = (int)(row / S), s = (int)(row % S);
    const int src = src_of_row[s];
    if (src < 0) continue;
    const int tag = src >> 28, i = src & 0x0FFFFFFF;
    uint4* base = tag == 0 ? video : (tag == 1 ? text : audio);
    if (base == nullptr) continue;
    const int n = tag == 0 ? n_video : (tag == 1 ? n_text : n_audio);
    uint4* dp = base + ((long long)b * n + i) * vec_per_row;
    const uint4* sp = x + row * vec_per_row;
    for (int v = lane; v < vec_per_row; v += 32) dp[v] = sp[v];
  }
}

__global__ void k_permute(int B, int n, int S_full, int vec_per_row,
                          const int32_t* __restrict__ perm, const uint4* __restrict__ src,
                          uint4* __restrict__ dst, int gather) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < (long long)B * n; row += warps) {
    const int b = (int)(row / n), j = (int)(row % n);
    const long long full_row = (long long)b * S_full + perm[j];
    const uint4* sp = src + (gather ? full_row : row) * vec_per_row;
    uint4* dp = dst + (gather ? row : full_row) * vec_per_row;
    for (int v = lane; v < vec_per_row; v += 32) dp[v] = sp[v];
  }
}

// Row gather / scatter with conversion: gather reads bf16 rows and writes fp32,
// scatter reads fp32 rows and writes bf16 (round to nearest even).
__global__ void k_permute_convert(int B, int n, int S_full, int vec8_per_row,
                                  const int32_t* __restrict__ perm, const void* __restrict__ src,
                                  void* __restrict__ dst, int gather) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < (long long)B * n; row += warps) {
    const int b = (int)(row / n), j = (int)(row % n);
    const long long full_row = (long long)b * S_full + perm[j];
    if (gather) {
      const uint4* sp = reinterpret_cast<const uint4*>(src) + full_row * vec8_per_row;
      float4* dp = reinterpret_cast<float4*>(dst) + row * vec8_per_row * 2;
      for (int v = lane; v < vec8_per_row; v += 32) {
        const uint4 u = sp[v];
        dp[2 * v] = make_float4(bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y));
        dp[2 * v + 1] = make_float4(bf16lo(u.z), bf16hi(u.z), bf16lo(u.w), bf16hi(u.w));
      }
    } else {
      const float4* sp = reinterpret_cast<const float4*>(src) + row * vec8_per_row * 2;
      uint4* dp = reinterpret_cast<uint4*>(dst) + full_row * vec8_per_row;
      for (int v = lane; v < vec8_per_row; v += 32) {
        const float4 a = sp[2 * v], c = sp[2 * v + 1];
        dp[v] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(c.x, c.y),
                           pack_bf16x2(c.z, c.w));
      }
    }
  }
}

int grid_for(long long work, int per_block) {
  long long g = (work + per_block - 1) / per_block;
  const long long cap = (long long)num_sms() * 16;
  if (g > cap) g = cap;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_layout_prepare(h3_layout* L, float rope_theta, int* d_status,
                                  int32_t* d_scratch, cudaStream_t st) {
  const int S = L->S;
  int32_t* hits = d_scratch;                 // [S]
  int32_t* tile_pad = d_scratch + S;         // [n_tiles]
  int32_t* counts = tile_pad + L->n_tiles;   // [4]
  int* n_valid = counts + 4;                 // [1]
  if (S > 0) {
    k_validate_rows<<<grid_for(S, 256), 256, 0, st>>>(S, L->n_t, L->tags, L->t_idx, L->pos,
                                                       L->src_of_row, hits, tile_pad, counts,
                                                       d_status);
    if (L->n_video)
      k_validate_index<<<grid_for(L->n_video, 256), 256, 0, st>>>(
          S, L->n_video, 0, L->video_idx, L->tags, hits, L->src_of_row, d_status);
    if (L->n_text)
      k_validate_index<<<grid_for(L->n_text, 256), 256, 0, st>>>(
          S, L->n_text, 1, L->text_idx, L->tags, hits, L->src_of_row, d_status);
    if (L->n_audio)
      k_validate_index<<<grid_for(L->n_audio, 256), 256, 0, st>>>(
          S, L->n_audio, 2, L->audio_idx, L->tags, hits, L->src_of_row, d_status);
    k_rope_table<<<grid_for((long long)S * kRopePairs, 256), 256, 0, st>>>(
        S, L->pos, (double)rope_theta, L->rope);
  }
  k_finalize<<<1, 1024, 0, st>>>(S, L->n_tiles, L->n_video, L->n_text, L->n_audio, L->tags,
                                 hits, tile_pad, counts, L->tile_class, L->key_valid, L->perm,
                                 d_status, n_valid);
  return cudaGetLastError();
}

cudaError_t launch_compact_tables(h3_layout* L, cudaStream_t st) {
  const int V = L->n_valid;
  k_compact_tables<<<grid_for((long long)(V > 0 ? V : 1) * kRopePairs, 256), 256, 0, st>>>(
      V, L->c_tiles, L->perm, L->tags, L->t_idx, L->rope, L->c_tags, L->c_tidx, L->c_rope,
      L->c_tile_class, L->c_key_valid);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // The text rows as a sequence of their own, in text_idx order: the same
  // gather over text_idx instead of the compaction order.
  const int T = L->n_text;
  k_compact_tables<<<grid_for((long long)(T > 0 ? T : 1) * kRopePairs, 256), 256, 0, st>>>(
      T, L->t_tiles, L->text_idx, L->tags, L->t_idx, L->rope, L->t_tags, L->t_tidx, L->t_rope,
      L->t_tile_class, L->t_key_valid);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (L->S > 0) {
    if ((e = cudaMemsetAsync(L->c_of_row, 0xff, (size_t)L->S * 4, st)) != cudaSuccess) return e;
    if (V > 0) k_compact_position<<<grid_for(V, 256), 256, 0, st>>>(V, L->perm, L->c_of_row);
  }
  return cudaGetLastError();
}

cudaError_t launch_pack(const h3_layout* L, int B, int row_elems, const void* video,
                        const void* audio, const void* text, void* x, cudaStream_t st) {
  const long long rows = (long long)B * L->S;
  if (rows == 0) return cudaSuccess;
  k_pack<<<grid_for(rows, 8), 256, 0, st>>>(B, L->S, row_elems / 8, L->src_of_row,
                                             (const uint4*)video, L->n_video, (const uint4*)text,
                                             L->n_text, (const uint4*)audio, L->n_audio,
                                             (uint4*)x);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const h3_layout* L, int B, int row_elems, const void* x, void* video,
                          void* audio, void* text, cudaStream_t st) {
  const long long rows = (long long)B * L->S;
  if (rows == 0) return cudaSuccess;
  k_unpack<<<grid_for(rows, 8), 256, 0, st>>>(B, L->S, row_elems / 8, L->src_of_row,
                                               (const uint4*)x, (uint4*)video, L->n_video,
                                               (uint4*)text, L->n_text, (uint4*)audio,
                                               L->n_audio);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows(int B, int n, int S_full, int row_elems, const int32_t* perm,
                                const void* src, void* dst, bool gather, cudaStream_t st) {
  const long long rows = (long long)B * n;
  if (rows == 0) return cudaSuccess;
  k_permute<<<grid_for(rows, 8), 256, 0, st>>>(B, n, S_full, row_elems / 8, perm,
                                                (const uint4*)src, (uint4*)dst, gather ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows_convert(int B, int n, int S_full, int row_elems,
                                        const int32_t* perm, const void* src, void* dst,
                                        bool gather, cudaStream_t st) {
  const long long rows = (long long)B * n;
  if (rows == 0) return cudaSuccess;
  k_permute_convert<<<grid_for(rows, 8), 256, 0, st>>>(B, n, S_full, row_elems / 8, perm, src,
                                                        dst, gather ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace h3
