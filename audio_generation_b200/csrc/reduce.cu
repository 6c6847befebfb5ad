// Token reduction in the middle blocks of the stack ("MiniMax H3 Inference
// Engine voor Mac computers", section "Token-reduction internals": after
// block 3, adjacent horizontal target-video tokens are paired while text,
// audio and reference tokens stay exact; the full-resolution state is kept as
// a bypass and restored before a later block).
//
// Pairs: packed rows r, r + 1 that are both target-video rows with the same
// t_idx, the same t and h coordinates and w coordinates 2k and 2k + 1 (a local
// test, so no two pairs overlap: the second row has an odd w). The reduced
// sequence keeps every row except the second of each pair, in packed order; a
// pair's row has the mean of the two positions. Merge: a pair's fp32 stream
// rows averaged; restore: each row of a pair, and every unpaired row, gets its
// reduced row's change since the merge added to the bypass.
#include "internal.cuh"
#include "sm100.cuh"

namespace h3 {
namespace {

__global__ void k_pair_heads(int S, const int32_t* __restrict__ tags,
                             const int32_t* __restrict__ t_idx, const float* __restrict__ pos,
                             const int32_t* __restrict__ target, uint8_t* __restrict__ head) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < S; r += gridDim.x * blockDim.x) {
    bool h = false;
    if (r + 1 < S && tags[r] == 0 && tags[r + 1] == 0 && target[r] && target[r + 1] &&
        t_idx[r] == t_idx[r + 1]) {
      const float w = pos[3 * r + 2];
      h = pos[3 * r] == pos[3 * (r + 1)] && pos[3 * r + 1] == pos[3 * (r + 1) + 1] &&
          fmodf(w, 2.f) == 0.f && pos[3 * (r + 1) + 2] == w + 1.f;
    }
    head[r] = h ? 1 : 0;
  }
}

// Block-wide exclusive scan of four counters (1024 threads).
__device__ __forceinline__ void block_scan4(int4 v, int4& excl, int4& total) {
  __shared__ int4 warp_tot[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int4 inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, inc.x, o), b = __shfl_up_sync(0xffffffffu, inc.y, o);
    const int c = __shfl_up_sync(0xffffffffu, inc.z, o), d = __shfl_up_sync(0xffffffffu, inc.w, o);
    if (lane >= o) { inc.x += a; inc.y += b; inc.z += c; inc.w += d; }
  }
  if (lane == 31) warp_tot[wid] = inc;
  __syncthreads();
  if (wid == 0) {
    int4 t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, t.x, o), b = __shfl_up_sync(0xffffffffu, t.y, o);
      const int c = __shfl_up_sync(0xffffffffu, t.z, o), d = __shfl_up_sync(0xffffffffu, t.w, o);
      if (lane >= o) { t.x += a; t.y += b; t.z += c; t.w += d; }
    }
    warp_tot[lane] = t;  // inclusive totals of warps 0..lane
  }
  __syncthreads();
  const int4 before = wid > 0 ? warp_tot[wid - 1] : make_int4(0, 0, 0, 0);
  excl = make_int4(before.x + inc.x - v.x, before.y + inc.y - v.y, before.z + inc.z - v.z,
                   before.w + inc.w - v.w);
  total = warp_tot[31];
}

// One block of 1024 threads, each over a contiguous chunk of packed rows: the
// reduced rows (every row that is not the second of a pair), their tags,
// timestep indices and positions, their source rows and the three index
// tensors of the reduced sequence. out_n[0..3] = (rows, video, text, audio).
__global__ void __launch_bounds__(1024) k_reduce_build(
    int S, const int32_t* __restrict__ tags, const int32_t* __restrict__ t_idx,
    const float* __restrict__ pos, const uint8_t* __restrict__ head, int32_t* __restrict__ r_tags,
    int32_t* __restrict__ r_tidx, float* __restrict__ r_pos, int32_t* __restrict__ r_src_a,
    int32_t* __restrict__ r_src_b, int32_t* __restrict__ r_video, int32_t* __restrict__ r_text,
    int32_t* __restrict__ r_audio, int32_t* __restrict__ out_n) {
  const int chunk = (S + 1023) / 1024;
  const int r0 = min(S, threadIdx.x * chunk), r1 = min(S, r0 + chunk);
  auto is_tail = [&](int r) { return r > 0 && head[r - 1]; };
  int4 cnt = make_int4(0, 0, 0, 0);
  for (int r = r0; r < r1; ++r) {
    if (is_tail(r)) continue;
    cnt.x += 1;
    const int tg = tags[r];
    cnt.y += tg == 0;
    cnt.z += tg == 1;
    cnt.w += tg == 2;
  }
  int4 base, total;
  block_scan4(cnt, base, total);
  for (int r = r0; r < r1; ++r) {
    if (is_tail(r)) continue;
    const int j = base.x++;
    const int tg = tags[r];
    r_tags[j] = tg;
    r_tidx[j] = t_idx[r];
    r_src_a[j] = r;
    float p0 = pos[3 * r], p1 = pos[3 * r + 1], p2 = pos[3 * r + 2];
    if (head[r]) {
      r_src_b[j] = r + 1;
      p0 = 0.5f * (p0 + pos[3 * r + 3]);
      p1 = 0.5f * (p1 + pos[3 * r + 4]);
      p2 = 0.5f * (p2 + pos[3 * r + 5]);
    } else {
      r_src_b[j] = -1;
    }
    r_pos[3 * j] = p0;
    r_pos[3 * j + 1] = p1;
    r_pos[3 * j + 2] = p2;
    if (tg == 0) r_video[base.y++] = j;
    if (tg == 1) r_text[base.z++] = j;
    if (tg == 2) r_audio[base.w++] = j;
  }
  if (threadIdx.x == 0) {
    out_n[0] = total.x;
    out_n[1] = total.y;
    out_n[2] = total.z;
    out_n[3] = total.w;
  }
}

// map[c_of_row_r[j]] = (c_of_row_full[a], c_of_row_full[b] or -1) for the valid
// reduced rows: the source rows in the compact streams of both sequences.
__global__ void k_reduce_map(int Sr, const int32_t* __restrict__ r_tags,
                             const int32_t* __restrict__ src_a, const int32_t* __restrict__ src_b,
                             const int32_t* __restrict__ c_of_row_r,
                             const int32_t* __restrict__ c_of_row_full, int2* __restrict__ map) {
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < Sr; j += gridDim.x * blockDim.x) {
    if (r_tags[j] < 0) continue;
    const int b = src_b[j];
    map[c_of_row_r[j]] = make_int2(c_of_row_full[src_a[j]], b >= 0 ? c_of_row_full[b] : -1);
  }
}

// xr[b, j] = mean of the source rows of reduced row j (one warp per row).
__global__ void k_merge(int B, int Vr, int V, int H, const int2* __restrict__ map,
                        const float* __restrict__ xc, float* __restrict__ xr) {
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)B * Vr;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const int b = (int)(row / Vr), j = (int)(row % Vr);
    const int2 m = map[j];
    const float4* a = reinterpret_cast<const float4*>(xc + ((size_t)b * V + m.x) * H);
    float4* d = reinterpret_cast<float4*>(xr + (size_t)row * H);
    if (m.y < 0) {
      for (int q = lane; q < H / 4; q += 32) d[q] = a[q];
    } else {
      const float4* c = reinterpret_cast<const float4*>(xc + ((size_t)b * V + m.y) * H);
      for (int q = lane; q < H / 4; q += 32) {
        const float4 u = a[q], v = c[q];
        d[q] = make_float4(0.5f * (u.x + v.x), 0.5f * (u.y + v.y), 0.5f * (u.z + v.z),
                           0.5f * (u.w + v.w));
      }
    }
  }
}

// xc[b, a] += xr[b, j] - merge_j(xc) (and the same for b's partner).
__global__ void k_restore(int B, int Vr, int V, int H, const int2* __restrict__ map,
                          const float* __restrict__ xr, float* __restrict__ xc) {
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)B * Vr;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const int b = (int)(row / Vr), j = (int)(row % Vr);
    const int2 m = map[j];
    float4* a = reinterpret_cast<float4*>(xc + ((size_t)b * V + m.x) * H);
    const float4* r = reinterpret_cast<const float4*>(xr + (size_t)row * H);
    if (m.y < 0) {
      for (int q = lane; q < H / 4; q += 32) {
        const float4 u = a[q], v = r[q];
        a[q] = make_float4(u.x + (v.x - u.x), u.y + (v.y - u.y), u.z + (v.z - u.z),
                           u.w + (v.w - u.w));
      }
    } else {
      float4* c = reinterpret_cast<float4*>(xc + ((size_t)b * V + m.y) * H);
      for (int q = lane; q < H / 4; q += 32) {
        const float4 u = a[q], w = c[q], v = r[q];
        const float4 dd = make_float4(v.x - 0.5f * (u.x + w.x), v.y - 0.5f * (u.y + w.y),
                                      v.z - 0.5f * (u.z + w.z), v.w - 0.5f * (u.w + w.w));
        a[q] = make_float4(u.x + dd.x, u.y + dd.y, u.z + dd.z, u.w + dd.w);
        c[q] = make_float4(w.x + dd.x, w.y + dd.y, w.z + dd.z, w.w + dd.w);
      }
    }
  }
}

int row_grid(long long rows) {
  long long g = (rows + 7) / 8;
  const long long cap = (long long)num_sms() * 16;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

cudaError_t launch_pair_heads(const h3_layout* L, const int32_t* target, uint8_t* head,
                              cudaStream_t st) {
  if (L->S == 0) return cudaSuccess;
  const int grid = (int)((L->S + 255) / 256 < 4096 ? (L->S + 255) / 256 : 4096);
  k_pair_heads<<<grid, 256, 0, st>>>(L->S, L->tags, L->t_idx, L->pos, target, head);
  return cudaGetLastError();
}

cudaError_t launch_reduce_build(const h3_layout* L, const uint8_t* head, int32_t* r_tags,
                                int32_t* r_tidx, float* r_pos, int32_t* r_src_a, int32_t* r_src_b,
                                int32_t* r_video, int32_t* r_text, int32_t* r_audio,
                                int32_t* out_n, cudaStream_t st) {
  k_reduce_build<<<1, 1024, 0, st>>>(L->S, L->tags, L->t_idx, L->pos, head, r_tags, r_tidx, r_pos,
                                     r_src_a, r_src_b, r_video, r_text, r_audio, out_n);
  return cudaGetLastError();
}

cudaError_t launch_reduce_map(int Sr, const int32_t* r_tags, const int32_t* src_a,
                              const int32_t* src_b, const int32_t* c_of_row_r,
                              const int32_t* c_of_row_full, int2* map, cudaStream_t st) {
  if (Sr == 0) return cudaSuccess;
  const int grid = (Sr + 255) / 256 < 4096 ? (Sr + 255) / 256 : 4096;
  k_reduce_map<<<grid, 256, 0, st>>>(Sr, r_tags, src_a, src_b, c_of_row_r, c_of_row_full, map);
  return cudaGetLastError();
}

cudaError_t launch_merge(int B, int Vr, int V, int H, const int2* map, const float* xc,
                         float* xr, cudaStream_t st) {
  if ((long long)B * Vr == 0) return cudaSuccess;
  k_merge<<<row_grid((long long)B * Vr), 256, 0, st>>>(B, Vr, V, H, map, xc, xr);
  return cudaGetLastError();
}

cudaError_t launch_restore(int B, int Vr, int V, int H, const int2* map, const float* xr,
                           float* xc, cudaStream_t st) {
  if ((long long)B * Vr == 0) return cudaSuccess;
  k_restore<<<row_grid((long long)B * Vr), 256, 0, st>>>(B, Vr, V, H, map, xr, xc);
  return cudaGetLastError();
}

}  // namespace h3
