// a5: bidirectional attention over the packed sequence, padding rows in their
// own document ("MiniMaxH3Transformer3DModel" page: a layout with padding rows,
// tag -1, needs a masked attention backend because those rows stay in their
// own attention document under a boolean mask).
//
// o = softmax(q k^T / sqrt(128)) v per head, flash style on tcgen05:
//   warps 0..3  softmax: one query row per thread (= one TMEM lane); reads the
//               128-key score row from TMEM, online max / sum in fp32, writes
//               P (bf16) to shared memory in the 128-B swizzled K-major layout,
//               rescales the O accumulator in TMEM only when the running max
//               grows by more than 2^8 (lazy rescale), normalises at the end
//   warp 4      TMA producer: Q once, K and V tiles double-buffered
//   warp 5      TMEM owner and MMA issuer: S_j = Q K_j^T (two S buffers, so
//               S_{j+1} overlaps softmax j), O += P_j V_j (V as an MN-major
//               operand)
// Document mask: per 128-row tile the layout step records whether it is all
// valid, all padding or mixed, plus a valid-row bitmask. Valid query tiles
// skip all-padding key tiles entirely and mask padding keys in mixed tiles;
// all-padding query tiles are not computed (their rows leave the block
// unchanged) and their output rows are written as zeros.
#include "host_util.cuh"
#include "internal.cuh"
#include "sm100.cuh"

namespace h3 {
namespace {

constexpr int D = 128;
constexpr int HALF = 128 * 64 * 2;  // one 128-row x 64-column bf16 half tile: 16 KB
constexpr int TILE_BYTES = 2 * HALF;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;  // S0 [0,128), S1 [128,256), O [256,384)
constexpr float kLazyRescale = 8.0f;  // log2 units
// smem: Q | K0 K1 | V0 V1 | P | barriers
constexpr int OFF_Q = 0, OFF_K = TILE_BYTES, OFF_V = 3 * TILE_BYTES, OFF_P = 5 * TILE_BYTES;
constexpr int OFF_BAR = 6 * TILE_BYTES;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;

struct Bars {
  uint64_t q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], s_empty[2], p_full,
      o_done, drain;
};

__device__ __forceinline__ bool key_tile_skipped(const LayoutView& L, int kt) {
  return L.tile_class[kt] == 1;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_attention(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const LayoutView L, int NH,
                __nv_bfloat16* __restrict__ o, float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int qt = blockIdx.x, head = blockIdx.y, b = blockIdx.z;
  const int S = L.S;
  const int bh = b * NH + head;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = qt * 128;

  if (L.tile_class[qt] == 1) {  // all padding rows: not computed, zero output
    if (threadIdx.x < 128) {
      const int s = q0 + threadIdx.x;
      if (s < S) {
        uint4* dst = reinterpret_cast<uint4*>(o + (((size_t)b * S + s) * NH + head) * D);
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[i] = make_uint4(0, 0, 0, 0);
      }
    }
    return;
  }
  const int n_kt = L.n_tiles;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_empty[i], 128);
    }
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{L.err, abort_flag};

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      mbar_arrive_expect_tx(&bars->q_full, TILE_BYTES);
      tma_load_3d(smem + OFF_Q, &tq, &bars->q_full, 0, q0, bh);
      tma_load_3d(smem + OFF_Q + HALF, &tq, &bars->q_full, 64, q0, bh);
      int nk = 0, nv = 0;
      bool ok = true;
      for (int kt = 0; kt < n_kt && ok; ++kt) {
        if (key_tile_skipped(L, kt)) continue;
        const int st = nk & 1;
        const uint32_t ph = ((nk >> 1) & 1) ^ 1;
        if (!mbar_wait(&bars->k_empty[st], ph, wc)) { ok = false; break; }
        uint8_t* kd = smem + OFF_K + st * TILE_BYTES;
        mbar_arrive_expect_tx(&bars->k_full[st], TILE_BYTES);
        tma_load_3d(kd, &tk, &bars->k_full[st], 0, kt * 128, bh);
        tma_load_3d(kd + HALF, &tk, &bars->k_full[st], 64, kt * 128, bh);
        ++nk;
        if (!mbar_wait(&bars->v_empty[st], ph, wc)) { ok = false; break; }
        uint8_t* vd = smem + OFF_V + st * TILE_BYTES;
        mbar_arrive_expect_tx(&bars->v_full[st], TILE_BYTES);
        tma_load_3d(vd, &tv, &bars->v_full[st], 0, kt * 128, bh);
        tma_load_3d(vd + HALF, &tv, &bars->v_full[st], 64, kt * 128, bh);
        ++nv;
      }
      if (!ok) {
        mbar_drain(&bars->q_full, 0);
        for (int j = nk > 2 ? nk - 2 : 0; j < nk; ++j) mbar_drain(&bars->k_full[j & 1], (j >> 1) & 1);
        for (int j = nv > 2 ? nv - 2 : 0; j < nv; ++j) mbar_drain(&bars->v_full[j & 1], (j >> 1) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
      const uint32_t q_s = smem_u32(smem + OFF_Q);
      const uint32_t p_s = smem_u32(smem + OFF_P);
      bool ok = mbar_wait(&bars->q_full, 0, wc);
      tc_fence_after();
      // key tiles that are processed, in order
      int n = 0;
      for (int kt = 0; kt < n_kt; ++kt) n += key_tile_skipped(L, kt) ? 0 : 1;
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&bars->k_full[st], (j >> 1) & 1, wc)) return false;
        if (!mbar_wait(&bars->s_empty[st], ((j >> 1) & 1) ^ 1, wc)) return false;
        tc_fence_after();
        const uint32_t k_s = smem_u32(smem + OFF_K + st * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
          umma_bf16_ss(tmem + st * 128, sdesc_sw128(q_s + off, 16, 1024),
                       sdesc_sw128(k_s + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[st]);
        umma_commit(&bars->k_empty[st]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n && !issue_s(j + 1)) { ok = false; break; }
        const int st = j & 1;
        if (!mbar_wait(&bars->p_full, j & 1, wc)) { ok = false; break; }
        if (!mbar_wait(&bars->v_full[st], (j >> 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t v_s = smem_u32(smem + OFF_V + st * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a_off = (kk >> 2) * HALF + (kk & 3) * 32;
          umma_bf16_ss(tmem + 256, sdesc_sw128(p_s + a_off, 16, 1024),
                       sdesc_sw128(v_s + kk * 2048, HALF, 1024), idesc_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->o_done);
        umma_commit(&bars->v_empty[st]);
      }
      umma_commit(&bars->drain);
      mbar_drain(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0..3)
    const int r = warp * 32 + lane;  // query row in the tile = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    uint8_t* p_row = smem + OFF_P + r * 128;
    const uint32_t sw = r & 7;
    float m_run = -INFINITY, l_run = 0.f;
    int j = 0;
    uint32_t o_seen = 0;  // completed PV phases observed
    bool ok = true;
    for (int kt = 0; kt < n_kt && ok; ++kt) {
      if (key_tile_skipped(L, kt)) continue;
      const int st = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[st], (j >> 1) & 1, wc))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sc[128];
      {
        uint32_t rr[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(lane_base + st * 128 + 32 * c, rr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) sc[32 * c + i] = __uint_as_float(rr[i]) * scale_log2;
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->s_empty[st]);
      const bool need_mask = L.tile_class[kt] != 0 || (kt + 1) * 128 > S;
      if (need_mask) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint32_t bits = L.key_valid[kt * 4 + w];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (!((bits >> i) & 1u)) sc[32 * w + i] = -INFINITY;
        }
      }
      float mx = sc[0];
#pragma unroll
      for (int i = 1; i < 128; ++i) mx = fmaxf(mx, sc[i]);
      // every PV before this tile must be complete before O is rescaled or P rewritten
      while (o_seen < (uint32_t)j) {
        const bool w = mbar_wait(&bars->o_done, o_seen & 1, wc);
        ++o_seen;
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      }
      if (!ok) break;
      // TMEM loads and stores are warp-collective: the warp rescales together
      // when any of its rows needs it; the other rows use alpha = 1.
      const bool need = mx > m_run + kLazyRescale;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mx : m_run;
        if (j > 0) {
          const float alpha = exp2f(m_run - m_new);
          l_run *= alpha;
          tc_fence_after();
          uint32_t rr[32];
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            tmem_ld32(lane_base + 256 + 32 * c, rr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
            tmem_st32(lane_base + 256 + 32 * c, rr);
          }
          tmem_wait_st();
        }
        m_run = m_new;
      }
      float lsum = 0.f;
#pragma unroll
      for (int c16 = 0; c16 < 16; ++c16) {
        float p[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          p[i] = exp2f(sc[8 * c16 + i] - m_run);
          lsum += p[i];
        }
        uint4 u;
        u.x = pack_bf16x2(p[0], p[1]);
        u.y = pack_bf16x2(p[2], p[3]);
        u.z = pack_bf16x2(p[4], p[5]);
        u.w = pack_bf16x2(p[6], p[7]);
        const uint32_t half = c16 >> 3, cc = c16 & 7;
        *reinterpret_cast<uint4*>(p_row + half * HALF + ((cc ^ sw) << 4)) = u;
      }
      l_run += lsum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
      ++j;
    }
    // final: wait for the last PV, normalise, store
    while (ok && o_seen < (uint32_t)j) {
      const bool w = mbar_wait(&bars->o_done, o_seen & 1, wc);
      ++o_seen;
      if (!__all_sync(0xffffffffu, w)) ok = false;
    }
    tc_fence_after();
    const int s = q0 + r;
    const bool row_ok = ok && s < S;
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    __nv_bfloat16* dst = o + (((size_t)b * S + (row_ok ? s : 0)) * NH + head) * D;
    uint32_t rr[32];
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      tmem_ld32(lane_base + 256 + 32 * c, rr);
      tmem_wait_ld();
      if (row_ok) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(rr[8 * q + 0]) * inv_l, __uint_as_float(rr[8 * q + 1]) * inv_l);
          u.y = pack_bf16x2(__uint_as_float(rr[8 * q + 2]) * inv_l, __uint_as_float(rr[8 * q + 3]) * inv_l);
          u.z = pack_bf16x2(__uint_as_float(rr[8 * q + 4]) * inv_l, __uint_as_float(rr[8 * q + 5]) * inv_l);
          u.w = pack_bf16x2(__uint_as_float(rr[8 * q + 6]) * inv_l, __uint_as_float(rr[8 * q + 7]) * inv_l);
          d4[q] = u;
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_attention(const LayoutView& L, int B, int NH, const void* q, const void* k,
                             const void* v, void* o, cudaStream_t st) {
  if (L.S == 0 || B == 0) return cudaSuccess;
  cudaError_t err =
      cudaFuncSetAttribute(k_attention, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (err != cudaSuccess) return err;
  CUtensorMap tq, tk, tv;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)L.S, (uint64_t)B * NH};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)L.S * D * 2};
  const uint32_t box[3] = {64, 128, 1};
  if (!make_tmap_bf16(&tq, q, 3, dims, strides, box) ||
      !make_tmap_bf16(&tk, k, 3, dims, strides, box) ||
      !make_tmap_bf16(&tv, v, 3, dims, strides, box))
    return cudaErrorInvalidValue;
  const float scale_log2 = 1.4426950408889634f / 11.313708498984761f;  // log2(e) / sqrt(128)
  dim3 grid(L.n_tiles, NH, B);
  k_attention<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(tq, tk, tv, L, NH,
                                                     reinterpret_cast<__nv_bfloat16*>(o),
                                                     scale_log2);
  return cudaGetLastError();
}

}  // namespace h3
