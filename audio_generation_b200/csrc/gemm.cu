// a4 / a6 / a8 / a9: persistent tcgen05 GEMM, C = A . B^T (bf16 in, fp32 in
// TMEM), with the block's fused epilogues.
//
// Two CTAs of a (2, 1, 1) cluster compute each 256 x BN output tile together
// with cta_group::2 MMAs (M = 256, N = BN, K = 16) issued by rank 0: each CTA
// loads its own 128 rows of A and its own BN / 2-row half of the B tile, and
// holds its 128 rows of the accumulator in its own TMEM. An MMA instruction
// costs tens of cycles to issue whatever its size, so the pair form (twice the
// work of a 128-row MMA per instruction) keeps the tensor core fed; it also
// halves each SM's share of B traffic and shared-memory operand reads.
// BN is 256, or 224 (except for the QKV and SwiGLU epilogues) when N is not a
// multiple of 256 or when 224 fills the last wave of tiles better (the
// launcher compares waves x tile width for both).
// Per CTA (6 warps):
//   warp 0        TMA producer: 128x64 A and (BN/2)x64 B-half tiles (128-B
//                 swizzle) into a 6-stage shared-memory ring; completion is
//                 counted on rank 0's barrier for both CTAs
//   warp 1        TMEM owner (both CTAs) and, in rank 0, the MMA issuer (the
//                 whole warp runs the loop, an elected lane issues);
//                 accumulator double-buffered in TMEM (2 x BN columns)
//   warps 2..5    epilogue: tcgen05.ld of the CTA's 128 accumulator rows (one
//                 TMEM lane per row), fused math, global stores; overlaps the
//                 next tile's main loop
// Tiles run in N-groups whose weight tiles stay L2-resident while the row
// blocks stream past them.
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
//   EPI_F32    plain fp32 store (the prologue's split-operand GEMMs).
// The QKV, SwiGLU and gated-residual epilogues also come in an e4m3 form
// (kind::f8f6f4 MMAs over 128-element K stages of 8-bit codes, BN = 256), whose
// accumulator is multiplied by the row's activation scale and the column's
// weight scale first.
// EPI_QKV places each head's rows through a HeadMap (internal.cuh): the plain
// block's [B, NH, S, 128] layout, or the receive buffers of the ranks of the
// sequence-parallel block.
#include "host_util.cuh"
#include "internal.cuh"
#include "sm100.cuh"

namespace h3 {
namespace {

constexpr int BM = 128, BK = 64;  // BM: rows per CTA; a pair tile is 2 BM x BN
// Tile width BN: 256, or 224 for the gated-residual GEMMs whose N is a
// multiple of 224 (N = 5376 gives 24 tiles of 224 instead of 21 of 256, so the
// 768 tiles fill the 74 CTA pairs' last wave better than 672 do).
constexpr int A_STAGE = BM * BK * 2;  // 16 KB
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 192;

#ifdef H3_FAULT_INJECTION
// Test-only build: when set, the producer issues no loads, so the MMA warp's
// bounded wait on the first stage runs out (nothing else sets that barrier).
static __device__ int g_fault_skip_loads;
#endif

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

// The accumulator of an e4m3 GEMM times the row's activation scale and each
// column's weight scale (a bf16 GEMM's accumulator as it is).
template <bool F8>
__device__ __forceinline__ void ld_acc_s(uint32_t taddr, float* v, float sa, const float* sw) {
  ld_acc(taddr, v);
  if constexpr (F8) {
    const float4* w4 = reinterpret_cast<const float4*>(sw);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 w = __ldg(w4 + q);
      v[4 * q] *= sa * w.x;
      v[4 * q + 1] *= sa * w.y;
      v[4 * q + 2] *= sa * w.z;
      v[4 * q + 3] *= sa * w.w;
    }
  }
}

// Epilogue for one 128 x 256 accumulator tile. Every lane of the warp executes
// the TMEM loads (they are warp-collective); stores are predicated per row.
template <int EPI, int BN, bool F8>
__device__ __forceinline__ void epilogue_tile(uint32_t taddr, int m, int n0, int M, int N,
                                              const GemmEpiArgs& e) {
  const bool row_ok = m < M;
  [[maybe_unused]] float sa = 1.f;
  if constexpr (F8) sa = row_ok ? e.a_scale[m] : 0.f;
  if constexpr (EPI == EPI_STORE) {
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(e.out);
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      float v[32];
      ld_acc(taddr + 32 * c, v);
      if (row_ok) store_bf16x32(out + (size_t)m * N + n0 + 32 * c, v);
    }
  } else if constexpr (EPI == EPI_F32) {
    float* out = reinterpret_cast<float*>(e.out);
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      float v[32];
      ld_acc(taddr + 32 * c, v);
      if (row_ok) {
        float4* d = reinterpret_cast<float4*>(out + (size_t)m * N + n0 + 32 * c);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(e.out);
    const int ldo = N / 2;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float a[32], b[32];
      ld_acc_s<F8>(taddr + 32 * c, a, sa, e.b_scale + n0 + 32 * c);
      ld_acc_s<F8>(taddr + 128 + 32 * c, b, sa, e.b_scale + n0 + 128 + 32 * c);
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
    for (int c = 0; c < BN / 32; ++c) {
      float v[32];
      ld_acc_s<F8>(taddr + 32 * c, v, sa, e.b_scale + n0 + 32 * c);
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
      const HeadMap& hm = e.heads;
      const int g = head / hm.heads_per_dst, lh = head - g * hm.heads_per_dst;
      __nv_bfloat16* dst =
          reinterpret_cast<__nv_bfloat16*>(kind == 0 ? hm.q[g] : (kind == 1 ? hm.k[g] : hm.v[g])) +
          (((size_t)b * hm.heads_per_dst + lh) * hm.dst_rows + hm.row_offset + s) * 128;
      const float* sw = e.b_scale + n0 + 128 * su;
      if (kind == 2) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[32];
          ld_acc_s<F8>(tbase + 32 * c, v, sa, sw + 32 * c);
          if (row_ok) store_bf16x32(dst + 32 * c, v);
        }
        continue;
      }
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32];
        ld_acc_s<F8>(tbase + 32 * c, v, sa, sw + 32 * c);
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
      }
      const float rstd = rsqrtf(ss * (1.f / 128.f) + e.qk_eps);
      const __nv_bfloat16* nw = reinterpret_cast<const __nv_bfloat16*>(kind == 0 ? e.q_norm
                                                                                 : e.k_norm);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32], w[32];
        ld_acc_s<F8>(tbase + 32 * c, v, sa, sw + 32 * c);
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
template <int BN>
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int group_n,
                                            int& m0, int& n0) {
  const int per_group = group_n * tiles_m;
  const int g = t / per_group, r = t - g * per_group;
  const int width = min(group_n, tiles_n - g * group_n);
  m0 = (r / width) * BM;
  n0 = (g * group_n + r % width) * BN;
}

constexpr int PNST = 6;
// Stage: 128 A rows + the CTA's BN / 2 B rows, 64 K-elements each (multiple of 1 KB).
template <int BN>
constexpr int p_stage() { return (BM + BN / 2) * BK * 2; }
template <int BN>
constexpr int p_smem_bytes() { return PNST * p_stage<BN>() + 1024 + 256; }

template <int EPI, int BN, bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                int M, int N, int K, int group_n, const __grid_constant__ GemmEpiArgs e) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int P_STAGE = p_stage<BN>();
  static_assert(P_STAGE % 1024 == 0, "stage alignment");
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + PNST * P_STAGE);
  uint64_t* empty = full + PNST;
  uint64_t* tfull = empty + PNST;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int tiles_m = (M + 2 * BM - 1) / (2 * BM), tiles_n = N / BN;
  // K elements per stage: 64 bf16 or 128 e4m3 (128 bytes either way)
  constexpr int BKE = F8 ? 2 * BK : BK;
  const int T = tiles_m * tiles_n, kb_n = K / BKE;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PNST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);  // one arrival per epilogue warp of both CTAs
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
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers and TMEM exist before either uses the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{e.L.err, abort_flag};
  auto at = [&](uint64_t* bar, uint32_t r) { return mapa_shared(smem_u32(bar), r); };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t n = 0;
      bool ok = true;
#ifdef H3_FAULT_INJECTION
      if (*(volatile int*)&g_fault_skip_loads) ok = false;
#endif
      for (int t = pair; t < T && ok; t += n_pairs) {
        int m0, n0;
        tile_coords<BN>(t, tiles_m, tiles_n, group_n, m0, n0);
        m0 = 2 * m0 + BM * rank;  // tile_coords counts 128-row units; pair tiles are 256 rows
        for (int kb = 0; kb < kb_n; ++kb) {
          const uint32_t s = n % PNST, ph = (n / PNST) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * P_STAGE;
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * P_STAGE);
          tma_load_2d_pair(sa, &tmA, at(&full[s], 0), kb * BKE, m0);
          tma_load_2d_pair(sa + A_STAGE, &tmB, at(&full[s], 0), kb * BKE, n0 + (BN / 2) * rank);
          ++n;
        }
      }
      if (!ok && leader) {  // let issued copies land before the CTA retires
        const uint32_t first = n > PNST ? n - PNST : 0;
        for (uint32_t i = first; i < n; ++i) mbar_drain(&full[i % PNST], (i / PNST) & 1);
      }
    }
  } else if (warp == 1) {
    if (leader) {  // the whole warp runs the loop; one elected lane issues
      constexpr uint32_t idesc =
          F8 ? idesc_e4m3_f32(2 * BM, BN) : idesc_bf16_f32(2 * BM, BN, false, false);
      constexpr uint32_t hi = sdesc_hi_sw128(1024);
      const uint32_t base_lo = sdesc_lo(smem_u32(smem), 16);
      uint32_t n = 0, it = 0;
      bool ok = true;
      for (int t = pair; t < T && ok; t += n_pairs, ++it) {
        const uint32_t acc = it & 1, aph = (it >> 1) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&tempty[acc], aph ^ 1, wc))) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = 0; kb < kb_n; ++kb) {
          const uint32_t s = n % PNST, ph = (n / PNST) & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, wc))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_lo = base_lo + s * (P_STAGE >> 4);
          const uint32_t b_lo = a_lo + (A_STAGE >> 4);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {  // 32 bytes of K per instruction
            if constexpr (F8)
              umma_ss_w_pair_elect_f8(d, a_lo + 2 * k, hi, b_lo + 2 * k, hi, idesc,
                                      (kb | k) != 0 ? 1u : 0u);
            else
              umma_ss_w_pair_elect(d, a_lo + 2 * k, hi, b_lo + 2 * k, hi, idesc,
                                   (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit_pair_elect(at(&empty[s], 0));
          umma_commit_pair_elect(at(&empty[s], 1));
          ++n;
        }
        if (!ok) break;
        umma_commit_pair_elect(at(&tfull[acc], 0));
        umma_commit_pair_elect(at(&tfull[acc], 1));
      }
      umma_commit_pair_elect(at(drain, 0));  // every MMA issued is complete past this point
      mbar_drain(drain, 0);
    }
  } else {
    const int quarter = warp & 3;
    const int row_local = quarter * 32 + lane;
    const uint32_t tempty0 = at(&tempty[0], 0), tempty1 = at(&tempty[1], 0);
    uint32_t it = 0;
    for (int t = pair; t < T; t += n_pairs, ++it) {
      const uint32_t acc = it & 1, aph = (it >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, wc))) break;
      tc_fence_after();
      int m0, n0;
      tile_coords<BN>(t, tiles_m, tiles_n, group_n, m0, n0);
      m0 = 2 * m0 + BM * rank;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
      epilogue_tile<EPI, BN, F8>(taddr, m0 + row_local, n0, M, N, e);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty1 : tempty0);
    }
  }
  __syncthreads();
  cluster_sync();  // no CTA leaves while the pair's MMAs or signals may still reach it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

template <int EPI, int BN, bool F8 = false>
cudaError_t run(int M, int N, int K, const void* A, const void* Bm, const GemmEpiArgs& e,
                cudaStream_t st) {
  constexpr int P_SMEM_BYTES = p_smem_bytes<BN>();
  cudaError_t err = cudaFuncSetAttribute(k_gemm_pair<EPI, BN, F8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         P_SMEM_BYTES);
  if (err != cudaSuccess) return err;
  CUtensorMap ta, tb;
  constexpr uint64_t esz = F8 ? 1 : 2;
  constexpr uint32_t bke = F8 ? 2 * BK : BK;  // 128 bytes of K per box row
  const CUtensorMapDataType type =
      F8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t da[2] = {(uint64_t)K, (uint64_t)M}, sa[1] = {(uint64_t)K * esz};
  const uint32_t ba[2] = {bke, BM};
  const uint64_t db[2] = {(uint64_t)K, (uint64_t)N}, sb[1] = {(uint64_t)K * esz};
  const uint32_t bb[2] = {bke, BN / 2};  // each CTA of the pair loads half of the tile's B rows
  if (!make_tmap(&ta, A, type, 2, da, sa, ba) || !make_tmap(&tb, Bm, type, 2, db, sb, bb))
    return cudaErrorInvalidValue;
  const int T = ((M + 2 * BM - 1) / (2 * BM)) * (N / BN);
  const int max_pairs = num_sms() / 2;
  const int n_pairs = T < max_pairs ? T : max_pairs;
  // Weight tiles kept L2-resident per group: about 48 MB of B.
  const long long b_tile_bytes = (long long)BN * K * esz;
  int group_n = (int)((48ll << 20) / b_tile_bytes);
  if (group_n < 1) group_n = 1;
  if (group_n > N / BN) group_n = N / BN;
  k_gemm_pair<EPI, BN, F8><<<2 * n_pairs, NUM_THREADS, P_SMEM_BYTES, st>>>(ta, tb, M, N, K,
                                                                          group_n, e);
  return cudaGetLastError();
}

// Waves x tile width for a tile width: the time of the persistent loop in
// units of one 256-wide tile column, up to the per-tile constant.
long long wave_cost(int M, int N, int bn) {
  const long long tiles = (long long)((M + 2 * BM - 1) / (2 * BM)) * (N / bn);
  const long long pairs = num_sms() / 2;
  return (tiles + pairs - 1) / pairs * bn;
}

}  // namespace

cudaError_t launch_gemm_e4m3(int epi, int M, int N, int K, const void* A, const void* Bm,
                             const GemmEpiArgs& e, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (K % (2 * BK) != 0 || K == 0 || N % 256 != 0 || !e.a_scale || !e.b_scale)
    return cudaErrorInvalidValue;
  switch (epi) {
    case EPI_QKV: return run<EPI_QKV, 256, true>(M, N, K, A, Bm, e, st);
    case EPI_SWIGLU: return run<EPI_SWIGLU, 256, true>(M, N, K, A, Bm, e, st);
    case EPI_RESID: return run<EPI_RESID, 256, true>(M, N, K, A, Bm, e, st);
    case EPI_RESID_F32: return run<EPI_RESID_F32, 256, true>(M, N, K, A, Bm, e, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(int epi, int M, int N, int K, const void* A, const void* Bm,
                        const GemmEpiArgs& e, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (K % BK != 0 || K == 0) return cudaErrorInvalidValue;
  // QKV and SwiGLU epilogues pair 128-column halves of a 256-wide tile. The
  // others also come in a 224-wide form, used when N is not a multiple of 256
  // or when it fills the CTA pairs' waves better.
  const bool w256 = N % 256 == 0, w224 = N % 224 == 0;
  if (epi == EPI_QKV || epi == EPI_SWIGLU) {
    if (!w256) return cudaErrorInvalidValue;
  } else if (!w256 && !w224) {
    return cudaErrorInvalidValue;
  }
  const bool narrow = w224 && (!w256 || wave_cost(M, N, 224) < wave_cost(M, N, 256));
  switch (epi) {
    case EPI_STORE:
      return narrow ? run<EPI_STORE, 224>(M, N, K, A, Bm, e, st)
                    : run<EPI_STORE, 256>(M, N, K, A, Bm, e, st);
    case EPI_QKV: return run<EPI_QKV, 256>(M, N, K, A, Bm, e, st);
    case EPI_RESID:
      return narrow ? run<EPI_RESID, 224>(M, N, K, A, Bm, e, st)
                    : run<EPI_RESID, 256>(M, N, K, A, Bm, e, st);
    case EPI_SWIGLU: return run<EPI_SWIGLU, 256>(M, N, K, A, Bm, e, st);
    case EPI_RESID_F32:
      return narrow ? run<EPI_RESID_F32, 224>(M, N, K, A, Bm, e, st)
                    : run<EPI_RESID_F32, 256>(M, N, K, A, Bm, e, st);
    case EPI_F32:
      return narrow ? run<EPI_F32, 224>(M, N, K, A, Bm, e, st)
                    : run<EPI_F32, 256>(M, N, K, A, Bm, e, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace h3

#ifdef H3_FAULT_INJECTION
// Test-only build: turn the GEMM producer's load skipping on (1) or off (0).
extern "C" __attribute__((visibility("default"))) int h3_test_gemm_skip_loads(int on) {
  return cudaMemcpyToSymbol(h3::g_fault_skip_loads, &on, sizeof(int)) == cudaSuccess ? 0 : -1;
}
#endif
