// a4 / a6 / a8 / a9: persistent tcgen05 GEMM, C = A . B^T (bf16 in, fp32 in
// TMEM), with the block's fused epilogues.
//
// Structure (one CTA per SM, 6 warps):
//   warp 0        TMA producer: 128x64 A and 256x64 B tiles (128-B swizzle)
//                 into a 4-stage shared-memory ring
//   warp 1        TMEM owner and MMA issuer: tcgen05.mma M=128 N=256 K=16,
//                 accumulator double-buffered in TMEM (2 x 256 columns)
//   warps 2..5    epilogue: tcgen05.ld of the accumulator (one TMEM lane per
//                 row), fused math, global stores; overlaps the next tile's
//                 main loop
// Tiles are walked M-fastest so that the CTAs in flight share B (weights)
// tiles and re-read A (activations) from L2.
//
// Epilogues:
//   EPI_QKV    head-interleaved QKV rows ("MiniMax H3 Inference Engine voor Mac
//              computers", section "Checkpoint layout en media pipeline": QKV
//              rows interleaved per head feed a fused QK-norm / RoPE kernel):
//              every 128-column sub-tile is one head's q, k or v. q and k get
//              RMSNorm (qk_norm_eps, learned [128] weight) then RoPE on the
//              channel pairs (32a + j, 32a + j + 16); stores head-major
//              [B, NH, S, 128] bf16.
//   EPI_RESID  x <- x + gate * acc (gated residual, "Exacte DiT fusions"),
//              gate = ada_table[tag][c] + tmod[t_idx][c]; padding rows skipped;
//              x bf16 (EPI_RESID) or fp32 (EPI_RESID_F32, the stack's stream).
//   EPI_SWIGLU W1 / W3 interleaved in 128-row blocks: g = SiLU(a) * b.
//   EPI_STORE  plain bf16 store (the GEMM core on its own).
#include "host_util.cuh"
#include "internal.cuh"
#include "sm100.cuh"

namespace h3 {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;  // 16 KB
constexpr int B_STAGE = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 192;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;

__device__ __forceinline__ void store_bf16x32(void* dst, const float* y) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    u.x = pack_bf16x2(y[8 * q + 0], y[8 * q + 1]);
    u.y = pack_bf16x2(y[8 * q + 2], y[8 * q + 3]);
    u.z = pack_bf16x2(y[8 * q + 4], y[8 * q + 5]);
    u.w = pack_bf16x2(y[8 * q + 6], y[8 * q + 7]);
    d[q] = u;
  }
}

__device__ __forceinline__ void load_bf16x32(const void* src, float* y) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = s[q];
    y[8 * q + 0] = bf16lo(u.x); y[8 * q + 1] = bf16hi(u.x);
    y[8 * q + 2] = bf16lo(u.y); y[8 * q + 3] = bf16hi(u.y);
    y[8 * q + 4] = bf16lo(u.z); y[8 * q + 5] = bf16hi(u.z);
    y[8 * q + 6] = bf16lo(u.w); y[8 * q + 7] = bf16hi(u.w);
  }
}

__device__ __forceinline__ void ld_acc(uint32_t taddr, float* v) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Epilogue for one 128 x 256 accumulator tile. Every lane of the warp executes
// the TMEM loads (they are warp-collective); stores are predicated per row.
template <int EPI>
__device__ __forceinline__ void epilogue_tile(uint32_t taddr, int m, int n0, int M, int N,
                                              const GemmEpiArgs& e) {
  const bool row_ok = m < M;
  if constexpr (EPI == EPI_STORE) {
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(e.out);
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      float v[32];
      ld_acc(taddr + 32 * c, v);
      if (row_ok) store_bf16x32(out + (size_t)m * N + n0 + 32 * c, v);
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(e.out);
    const int ldo = N / 2;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float a[32], b[32];
      ld_acc(taddr + 32 * c, a);
      ld_acc(taddr + 128 + 32 * c, b);
#pragma unroll
      for (int i = 0; i < 32; ++i) a[i] = a[i] / (1.f + __expf(-a[i])) * b[i];
      if (row_ok) store_bf16x32(out + (size_t)m * ldo + n0 / 2 + 32 * c, a);
    }
  } else if constexpr (EPI == EPI_RESID || EPI == EPI_RESID_F32) {
    const int s = row_ok ? m % e.L.S : 0;
    const int tag = row_ok ? e.L.tags[s] : -1;
    const int ti = row_ok ? e.L.t_idx[s] : 0;
    const bool active = row_ok && tag >= 0;
    const float* gt = e.table + ((size_t)(active ? tag : 0) * 6 + e.gate_chunk) * N + n0;
    const float* gm = e.tmod + ((size_t)ti * 6 + e.gate_chunk) * N + n0;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      float v[32];
      ld_acc(taddr + 32 * c, v);
      if (active) {
        float xv[32];
        const size_t off = (size_t)m * N + n0 + 32 * c;
        if constexpr (EPI == EPI_RESID) {
          load_bf16x32(reinterpret_cast<const __nv_bfloat16*>(e.x) + off, xv);
        } else {
          const float4* xp = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(e.x) + off);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 a = xp[q];
            xv[4 * q] = a.x; xv[4 * q + 1] = a.y; xv[4 * q + 2] = a.z; xv[4 * q + 3] = a.w;
          }
        }
        const float4* g1 = reinterpret_cast<const float4*>(gt + 32 * c);
        const float4* g2 = reinterpret_cast<const float4*>(gm + 32 * c);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 a = __ldg(g1 + q), b = __ldg(g2 + q);
          xv[4 * q + 0] = fmaf(a.x + b.x, v[4 * q + 0], xv[4 * q + 0]);
          xv[4 * q + 1] = fmaf(a.y + b.y, v[4 * q + 1], xv[4 * q + 1]);
          xv[4 * q + 2] = fmaf(a.z + b.z, v[4 * q + 2], xv[4 * q + 2]);
          xv[4 * q + 3] = fmaf(a.w + b.w, v[4 * q + 3], xv[4 * q + 3]);
        }
        if constexpr (EPI == EPI_RESID) {
          store_bf16x32(reinterpret_cast<__nv_bfloat16*>(e.x) + off, xv);
        } else {
          float4* xp = reinterpret_cast<float4*>(reinterpret_cast<float*>(e.x) + off);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            xp[q] = make_float4(xv[4 * q], xv[4 * q + 1], xv[4 * q + 2], xv[4 * q + 3]);
        }
      }
    }
  } else if constexpr (EPI == EPI_QKV) {
    const int S = e.L.S;
    const int b = row_ok ? m / S : 0;
    const int s = row_ok ? m % S : 0;
    const float2* rope = e.L.rope + (size_t)s * kRopePairs;
#pragma unroll 1
    for (int su = 0; su < 2; ++su) {
      const int u = n0 / 128 + su;
      const int head = u / 3, kind = u % 3;
      const uint32_t tbase = taddr + 128 * su;
      __nv_bfloat16* dst =
          reinterpret_cast<__nv_bfloat16*>(kind == 0 ? e.q : (kind == 1 ? e.k : e.v)) +
          (((size_t)b * e.NH + head) * S + s) * 128;
      if (kind == 2) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[32];
          ld_acc(tbase + 32 * c, v);
          if (row_ok) store_bf16x32(dst + 32 * c, v);
        }
        continue;
      }
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32];
        ld_acc(tbase + 32 * c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
      }
      const float rstd = rsqrtf(ss * (1.f / 128.f) + e.qk_eps);
      const __nv_bfloat16* nw = reinterpret_cast<const __nv_bfloat16*>(kind == 0 ? e.q_norm
                                                                                 : e.k_norm);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32], w[32];
        ld_acc(tbase + 32 * c, v);
        load_bf16x32(nw + 32 * c, w);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = v[i] * rstd * w[i];
        if (c < 3 && row_ok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float2 cs = __ldg(rope + 16 * c + j);
            const float x0 = v[j], x1 = v[j + 16];
            v[j] = x0 * cs.x - x1 * cs.y;
            v[j + 16] = x0 * cs.y + x1 * cs.x;
          }
        }
        if (row_ok) store_bf16x32(dst + 32 * c, v);
      }
    }
  }
}

// Tile order: the N tiles are cut into groups of `group_n` columns; within a
// group the tiles run N-fastest, then down M. The CTAs in flight then share a
// group of weight tiles that stays in L2 while the row blocks stream past it.
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int group_n,
                                            int& m0, int& n0) {
  const int per_group = group_n * tiles_m;
  const int g = t / per_group, r = t - g * per_group;
  const int width = min(group_n, tiles_n - g * group_n);
  m0 = (r / width) * BM;
  n0 = (g * group_n + r % width) * BN;
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           int M, int N, int K, int group_n, const GemmEpiArgs e) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (M + BM - 1) / BM, tiles_n = N / BN;
  const int T = tiles_m * tiles_n, kb_n = K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{e.L.err, abort_flag};

  if (warp == 0) {
    if (lane == 0) {
      uint32_t n = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < T && ok; t += gridDim.x) {
        int m0, n0;
        tile_coords(t, tiles_m, tiles_n, group_n, m0, n0);
        for (int kb = 0; kb < kb_n; ++kb) {
          const uint32_t s = n % STAGES, ph = (n / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(sa, &tmA, &full[s], kb * BK, m0);
          tma_load_2d(sa + A_STAGE, &tmB, &full[s], kb * BK, n0);
          ++n;
        }
      }
      if (!ok) {  // let issued copies land before the CTA retires
        const uint32_t first = n > STAGES ? n - STAGES : 0;
        for (uint32_t i = first; i < n; ++i) mbar_drain(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, false);
      uint32_t n = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < T && ok; t += gridDim.x, ++it) {
        const uint32_t acc = it & 1, aph = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1, wc)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = 0; kb < kb_n; ++kb) {
          const uint32_t s = n % STAGES, ph = (n / STAGES) & 1;
          if (!mbar_wait(&full[s], ph, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b0 = a0 + A_STAGE;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            umma_bf16_ss(d, sdesc_sw128(a0 + 32 * k, 16, 1024), sdesc_sw128(b0 + 32 * k, 16, 1024),
                         idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          ++n;
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
      umma_commit(drain);  // every MMA this thread issued is complete past this point
      mbar_drain(drain, 0);
    }
  } else {
    const int quarter = warp & 3;
    const int row_local = quarter * 32 + lane;
    uint32_t it = 0;
    for (int t = blockIdx.x; t < T; t += gridDim.x, ++it) {
      const uint32_t acc = it & 1, aph = (it >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, wc))) break;
      tc_fence_after();
      int m0, n0;
      tile_coords(t, tiles_m, tiles_n, group_n, m0, n0);
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
      epilogue_tile<EPI>(taddr, m0 + row_local, n0, M, N, e);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int EPI>
cudaError_t run(int M, int N, int K, const void* A, const void* Bm, const GemmEpiArgs& e,
                cudaStream_t st) {
  cudaError_t err =
      cudaFuncSetAttribute(k_gemm<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (err != cudaSuccess) return err;
  CUtensorMap ta, tb;
  const uint64_t da[2] = {(uint64_t)K, (uint64_t)M}, sa[1] = {(uint64_t)K * 2};
  const uint32_t ba[2] = {BK, BM};
  const uint64_t db[2] = {(uint64_t)K, (uint64_t)N}, sb[1] = {(uint64_t)K * 2};
  const uint32_t bb[2] = {BK, BN};
  if (!make_tmap_bf16(&ta, A, 2, da, sa, ba) || !make_tmap_bf16(&tb, Bm, 2, db, sb, bb))
    return cudaErrorInvalidValue;
  const int T = ((M + BM - 1) / BM) * (N / BN);
  const int grid = T < num_sms() ? T : num_sms();
  // Weight tiles kept L2-resident per group: about 48 MB of B.
  const long long b_tile_bytes = (long long)BN * K * 2;
  int group_n = (int)((48ll << 20) / b_tile_bytes);
  if (group_n < 1) group_n = 1;
  if (group_n > N / BN) group_n = N / BN;
  k_gemm<EPI><<<grid, NUM_THREADS, SMEM_BYTES, st>>>(ta, tb, M, N, K, group_n, e);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(int epi, int M, int N, int K, const void* A, const void* Bm,
                        const GemmEpiArgs& e, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (N % BN != 0 || K % BK != 0 || K == 0) return cudaErrorInvalidValue;
  switch (epi) {
    case EPI_STORE: return run<EPI_STORE>(M, N, K, A, Bm, e, st);
    case EPI_QKV: return run<EPI_QKV>(M, N, K, A, Bm, e, st);
    case EPI_RESID: return run<EPI_RESID>(M, N, K, A, Bm, e, st);
    case EPI_SWIGLU: return run<EPI_SWIGLU>(M, N, K, A, Bm, e, st);
    case EPI_RESID_F32: return run<EPI_RESID_F32>(M, N, K, A, Bm, e, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace h3
