// a5: bidirectional attention over the packed sequence, padding rows in their
// own document ("MiniMaxH3Transformer3DModel" page: a layout with padding rows,
// tag -1, needs a masked attention backend because those rows stay in their
// own attention document under a boolean mask).
//
// o = softmax(q k^T / sqrt(128)) v per head, flash style on tcgen05. One CTA
// takes two 128-row query tiles of one head, so the tensor core works on one
// tile while the other tile's softmax runs:
//   warps 0..3   softmax of query tile 0 (one row per thread = one TMEM lane)
//   warps 4..7   softmax of query tile 1
//   warp 8       TMA producer: both Q tiles once, K and V tiles double-buffered
//   warp 9       TMEM owner and MMA issuer (the whole warp runs the issue loop;
//                one elected lane issues each tcgen05 instruction)
//   warps 10, 11 idle (they complete the third warpgroup, whose register
//                budget is handed to the softmax warpgroups)
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512). A
// softmax warpgroup reads its S row into registers, then writes P (bf16, two
// keys per 32-bit column) over the first 64 columns of the same S buffer;
// O += P V takes P straight from TMEM (A operand in tensor memory) and V from
// shared memory as an MN-major operand. The MMA warp issues, per key tile j:
//   PV0(j), S0(j+1), PV1(j), S1(j+1)
// tcgen05 MMAs of one thread run in issue order, so S_i(j+1) overwrites P_i(j)
// only after PV_i(j) has read it, and the commit that signals S_i(j+1) also
// guarantees PV_i(j) is complete: the softmax may then rescale O_i in place.
// O is rescaled only when a row's running max grows by more than 2^8 (lazy
// rescale), decided per warp because TMEM loads / stores are warp-collective.
// exp2 runs on the MUFU for most key pairs and as a polynomial on the FMA pipe
// for every sixth pair, to keep both pipes busy.
// P is handed to the MMA warp in two halves (keys 0..63, then 64..127), so the
// first half of P V runs while the second half's exponentials are computed.
//
// Document mask: per 128-row tile the layout step records whether it is all
// valid, all padding or mixed, plus a valid-row bitmask. Key tiles that are
// all padding are skipped; padding keys of mixed tiles are masked. Rows of
// all-padding query tiles are written as zeros.
// Output rows are placed through a RowMap (internal.cuh): the plain [B, S,
// NH * 128] layout, or, for a rank of the sequence-parallel block, the receive
// buffer of the rank that owns each row.
#include "host_util.cuh"
#include "internal.cuh"
#include "sm100.cuh"

namespace h3 {
namespace {

constexpr int D = 128;
constexpr int HALF = 128 * 64 * 2;  // one 128-row x 64-column bf16 half tile: 16 KB
constexpr int TILE_BYTES = 2 * HALF;
constexpr int NUM_THREADS = 384;
// Registers per thread after the split; launched at 65536 / 384 -> 168 each:
// 2 * 128 * kSoftmaxRegs + 128 * kControlRegs must not exceed 384 * 168. With
// 216 / 72 neither the softmax nor the producer / MMA loops spill (224 / 56
// spills in the control warps, 208 / 88 in the softmax warps).
constexpr uint32_t kSoftmaxRegs = 216, kControlRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= 384 * 168, "register split");
constexpr int TMEM_COLS = 512;
constexpr float kLazyRescale = 8.0f;  // log2 units
// smem: Q0 Q1 | K0 K1 | V0 V1 | barriers | processed key-tile list
constexpr int OFF_Q = 0, OFF_K = 2 * TILE_BYTES, OFF_V = 4 * TILE_BYTES;
constexpr int OFF_BAR = 6 * TILE_BYTES;
constexpr int OFF_LIST = OFF_BAR + 256;
constexpr int kMaxKeyTiles = kMaxRows / 128;  // the key-tile list below (S <= kMaxRows)
constexpr int SMEM_BYTES = OFF_LIST + 2 * kMaxKeyTiles + 1024;

struct Bars {
  uint64_t q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_half[2],
      p_full[2], o_final[2], drain;
};


__device__ __forceinline__ float exp2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe, for two values at once: split x = j + f with
// j = round(x) (adding 1.5 * 2^23 leaves the rounded integer in the low
// mantissa bits) and f in [-1/2, 1/2]; 2^f by a cubic fitted by least squares
// (relative error weighted) at 256 Chebyshev nodes of [-1/2, 1/2], max
// relative error 7.7e-5 wherever 2^x is a normal float (x >= -125; bf16 keeps
// 3.9e-3); j is added to the exponent field. Inputs below -126 are clamped;
// below -125 the result is off by less than 2^-135 in absolute terms,
// negligible next to the row sum, which is >= 1.
constexpr float kExpC3 = 0.05508868396f, kExpC2 = 0.24260404706f, kExpC1 = 0.69327622652f,
                kExpC0 = 0.99992895126f;
constexpr float kRoundMagic = 12582912.f;  // 1.5 * 2^23

// Packed fp32 pair arithmetic (one instruction for two lanes of work).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ void exp2_poly2(uint64_t x2, float& p0, float& p1) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  const uint64_t xc = f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t t = f2_add(xc, f2_pack(kRoundMagic, kRoundMagic));
  const uint64_t jf = f2_add(t, f2_pack(-kRoundMagic, -kRoundMagic));     // j, exact
  const uint64_t f = f2_fma(jf, f2_pack(-1.f, -1.f), xc);                  // x - j, exact
  uint64_t p = f2_fma(f2_pack(kExpC3, kExpC3), f, f2_pack(kExpC2, kExpC2));
  p = f2_fma(p, f, f2_pack(kExpC1, kExpC1));
  p = f2_fma(p, f, f2_pack(kExpC0, kExpC0));
  float q0, q1, t0, t1;
  f2_unpack(p, q0, q1);
  f2_unpack(t, t0, t1);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

// Which key pairs of a 64-key half take the FMA-pipe exp2 (bit e of the mask
// for pair e), spread among the MUFU pairs so that both pipes work at the same
// time. Default: every sixth pair (pairs 5, 11, 17, 23, 29: 16 %), the fastest
// of the splits measured (50, 40, 33, 25, 16, 12.5 and 0 %).
#ifndef H3_ATTN_POLY_MASK
#define H3_ATTN_POLY_MASK 0x20820820u
#endif
constexpr uint32_t kPolyMask = H3_ATTN_POLY_MASK;

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Start of the 128 output values of row s, head h of batch element b.
__device__ __forceinline__ __nv_bfloat16* out_row(const RowMap& m, int b, int s, int h) {
  const int g = s / m.rows_per_dst, sl = s - g * m.rows_per_dst;
  return reinterpret_cast<__nv_bfloat16*>(m.o[g]) +
         (((size_t)b * m.rows_per_dst + sl) * m.row_heads + m.head_offset + h) * D;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_attention(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const LayoutView L, int NH,
                const __grid_constant__ RowMap om, float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int pair = blockIdx.x, head = blockIdx.y, b = blockIdx.z;
  const int S = L.S;
  const int bh = b * NH + head;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = pair * 256;
  const int qt0 = 2 * pair, qt1 = 2 * pair + 1;
  const bool pad0 = L.tile_class[qt0] == 1;
  const bool pad1 = qt1 >= L.n_tiles || L.tile_class[qt1] == 1;

  if (pad0 && pad1) {  // nothing to compute: zero the rows that exist
    if (threadIdx.x < 256) {
      const int s = q0 + threadIdx.x;
      if (s < S) {
        uint4* dst = reinterpret_cast<uint4*>(out_row(om, b, s, head));
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[i] = make_uint4(0, 0, 0, 0);
      }
    }
    return;
  }
  // The key tiles this CTA visits, in order: index | 0x8000 when the tile needs
  // the per-key mask (mixed, or the ragged last tile). All-padding tiles are
  // left out. Built once, read by every role from shared memory.
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + OFF_LIST);
  __shared__ int s_n;
  if (warp == 0) {
    int base = 0;
    for (int k0 = 0; k0 < L.n_tiles; k0 += 32) {
      const int kt = k0 + lane;
      const int cls = kt < L.n_tiles ? L.tile_class[kt] : 1;
      const bool keep = cls != 1;
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const bool masked = cls == 2 || (kt + 1) * 128 > S;
        list[base + __popc(m & ((1u << lane) - 1u))] =
            static_cast<uint16_t>(kt | (masked ? 0x8000 : 0));
      }
      base += __popc(m);
    }
    if (lane == 0) s_n = base;
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_half[i], 4);  // one arrival per softmax warp
      mbar_init(&bars->p_full[i], 4);
      mbar_init(&bars->o_final[i], 1);
    }
    mbar_init(&bars->drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{L.err, abort_flag};
  const int n = s_n;  // number of key tiles visited

  if (warp >= 8) {
    setmaxnreg_dec<kControlRegs>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      mbar_arrive_expect_tx(&bars->q_full, 2 * TILE_BYTES);
      tma_load_3d(smem + OFF_Q, &tq, &bars->q_full, 0, q0, bh);
      tma_load_3d(smem + OFF_Q + HALF, &tq, &bars->q_full, 64, q0, bh);
      tma_load_3d(smem + OFF_Q + TILE_BYTES, &tq, &bars->q_full, 0, q0 + 128, bh);
      tma_load_3d(smem + OFF_Q + TILE_BYTES + HALF, &tq, &bars->q_full, 64, q0 + 128, bh);
      int nk = 0, nv = 0;
      bool ok = true;
      for (int jj = 0; jj < n && ok; ++jj) {
        const int kt = list[jj] & 0x7fff;
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
      if (!ok) {  // let issued copies land before the CTA retires
        mbar_drain(&bars->q_full, 0);
        for (int j = nk > 2 ? nk - 2 : 0; j < nk; ++j) mbar_drain(&bars->k_full[j & 1], (j >> 1) & 1);
        for (int j = nv > 2 ? nv - 2 : 0; j < nv; ++j) mbar_drain(&bars->v_full[j & 1], (j >> 1) & 1);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp runs the loop; one lane elected per instruction issues
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
      const uint32_t q_s = smem_u32(smem + OFF_Q);
      auto wait_all = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
      };
      bool ok = wait_all(&bars->q_full, 0);
      tc_fence_after();
      // S_i(j) = Q_i K_j^T into TMEM columns [128 i, 128 i + 128)
      constexpr uint32_t hi = sdesc_hi_sw128(1024);
      const uint32_t q_lo = sdesc_lo(q_s, 16);
      const uint32_t k_lo = sdesc_lo(smem_u32(smem + OFF_K), 16);
      const uint32_t v_lo = sdesc_lo(smem_u32(smem + OFF_V), HALF);
      auto issue_s = [&](int i, int j) -> bool {
        const int st = j & 1;
        if (i == 0) {
          if (!wait_all(&bars->k_full[st], (j >> 1) & 1)) return false;
          tc_fence_after();
        }
        const uint32_t kl = k_lo + st * (TILE_BYTES >> 4);
        const uint32_t ql = q_lo + i * (TILE_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * HALF + (kk & 3) * 32) >> 4;
          umma_ss_w_elect(tmem + i * 128, ql + off, hi, kl + off, hi, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit_elect(&bars->s_full[i]);
        if (i == 1) umma_commit_elect(&bars->k_empty[st]);
        return true;
      };
      // O_i += P_i(j) V_j, P_i from TMEM columns [128 i, 128 i + 64). Keys
      // 0..63 (P columns [0, 32)) go as soon as the softmax has stored them,
      // keys 64..127 when the rest of P is in.
      auto issue_pv = [&](int i, int j) -> bool {
        const int st = j & 1;
        if (!wait_all(&bars->p_half[i], j & 1)) return false;
        if (i == 0 && !wait_all(&bars->v_full[st], (j >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t vl = v_lo + st * (TILE_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          umma_ts_w_elect(tmem + 256 + i * 128, tmem + i * 128 + kk * 8, vl + kk * (2048 >> 4), hi,
                          idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        if (!wait_all(&bars->p_full[i], j & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 4; kk < 8; ++kk) {
          umma_ts_w_elect(tmem + 256 + i * 128, tmem + i * 128 + kk * 8, vl + kk * (2048 >> 4), hi,
                          idesc_pv, 1u);
        }
        if (i == 1) umma_commit_elect(&bars->v_empty[st]);
        if (j == n - 1) umma_commit_elect(&bars->o_final[i]);
        return true;
      };
      if (ok) ok = issue_s(0, 0) && issue_s(1, 0);
      for (int j = 0; j < n && ok; ++j) {
        ok = issue_pv(0, j);
        if (ok && j + 1 < n) ok = issue_s(0, j + 1);
        if (ok) ok = issue_pv(1, j);
        if (ok && j + 1 < n) ok = issue_s(1, j + 1);
      }
      umma_commit_elect(&bars->drain);  // every MMA issued is complete past this point
      mbar_drain(&bars->drain, 0);
    }
  }
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax (warps 0..7)
    const int i = warp >> 2;  // query tile of this warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row in the tile = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t s_col = lane_base + i * 128;
    const uint32_t o_col = lane_base + 256 + i * 128;
    float m_run = -INFINITY, l_run = 0.f;
    const uint64_t scale2 = f2_pack(scale_log2, scale_log2);
    int j = 0;
    bool ok = true;
    for (; j < n; ++j) {
      const int entry = list[j];
      const int kt = entry & 0x7fff;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[i], j & 1, wc))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sc[128];
      {
        uint32_t rr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_col + 32 * c, rr[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) sc[32 * c + e] = __uint_as_float(rr[c][e]);
      }
      if (entry & 0x8000) {  // padding keys or keys past the end: masked out
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint32_t bits = L.key_valid[kt * 4 + w];
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (!((bits >> e) & 1u)) sc[32 * w + e] = -INFINITY;
        }
      }
      // row max: 8 independent partial maxima
      float pm[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) pm[k] = max3(sc[2 * k], sc[2 * k + 1], sc[16 + 2 * k]);
#pragma unroll
      for (int e = 32; e < 128; e += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) pm[k] = max3(pm[k], sc[e + 2 * k], sc[e + 2 * k + 1]);
#pragma unroll
      for (int k = 0; k < 8; ++k) pm[k] = fmaxf(pm[k], sc[16 + 2 * k + 1]);
      float mx = max3(max3(pm[0], pm[1], pm[2]), max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
      mx *= scale_log2;
      // O_i is stable here: the commit that signalled S_i(j) follows PV_i(j-1).
      const bool need = mx > m_run + kLazyRescale;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mx : m_run;
        if (j > 0) {
          const float alpha = exp2_mufu(m_run - m_new);
          l_run *= alpha;
          uint32_t rr[32];
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            tmem_ld32(o_col + 32 * c, rr);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
            tmem_st32(o_col + 32 * c, rr);
          }
        }
        m_run = m_new;
      }
      // P = 2^(s * scale - m), written as packed bf16 pairs over S columns
      // already held in registers: keys 0..63, then keys 64..127, each half
      // signalled to the MMA warp as soon as it is stored (one arrival per warp,
      // after the warp's stores are complete). The key pairs in kPolyMask take
      // the FMA-pipe exp2, the others the MUFU.
      const uint64_t negm2 = f2_pack(-m_run, -m_run);
      uint64_t sum2[4] = {0, 0, 0, 0};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int key = 64 * h + 2 * e;
          const uint64_t x2 = f2_fma(f2_pack(sc[key], sc[key + 1]), scale2, negm2);
          float p0, p1;
          if ((kPolyMask >> e) & 1u) {
            exp2_poly2(x2, p0, p1);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p0 = exp2_mufu(x0);
            p1 = exp2_mufu(x1);
          }
          sum2[e & 3] = f2_add(sum2[e & 3], f2_pack(p0, p1));
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_col + 32 * h, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(h == 0 ? &bars->p_half[i] : &bars->p_full[i]);
      }
      float a0, a1, b0, b1;
      f2_unpack(f2_add(sum2[0], sum2[1]), a0, a1);
      f2_unpack(f2_add(sum2[2], sum2[3]), b0, b1);
      l_run += (a0 + a1) + (b0 + b1);
    }
    if (ok && j > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_final[i], 0, wc));
    tc_fence_after();
    const int s = q0 + 128 * i + r;
    const bool tile_pad = i == 0 ? pad0 : pad1;
    const bool row_ok = ok && s < S;
    const float inv_l = (l_run > 0.f && !tile_pad) ? 1.f / l_run : 0.f;
    __nv_bfloat16* dst = out_row(om, b, row_ok ? s : 0, head);
    uint32_t rr[32];
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      tmem_ld32(o_col + 32 * c, rr);
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
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_attention(const LayoutView& L, int B, int NH, const void* q, const void* k,
                             const void* v, const RowMap& out, cudaStream_t st) {
  if (L.S == 0 || B == 0) return cudaSuccess;
  if (L.n_tiles > kMaxKeyTiles || B > kMaxBatch) return cudaErrorInvalidValue;
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
  dim3 grid((L.n_tiles + 1) / 2, NH, B);
  if (out.rows_per_dst <= 0 || (L.S + out.rows_per_dst - 1) / out.rows_per_dst > kMaxDst)
    return cudaErrorInvalidValue;
  k_attention<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(tq, tk, tv, L, NH, out, scale_log2);
  return cudaGetLastError();
}

}  // namespace h3
