// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/h3.h"

namespace h3 {

constexpr int kTile = 128;        // row tile (attention q/kv tiles, GEMM M tile)
// Rows of one packed sequence: the attention kernel keeps the list of key tiles
// it visits in shared memory (kMaxRows / 128 entries), and the layout step
// packs a row index into 28 bits.
constexpr int kMaxRows = 524288;
static_assert(kMaxRows < (1 << 28), "row index must fit the layout step's 28-bit field");
// Batch elements: the attention grid's z extent, and B * S must fit an int.
constexpr int kMaxBatch = 65535;
constexpr int kRopeFreqs = 16;    // rope_freq_dim supported by the kernels
constexpr int kRopePairs = 3 * kRopeFreqs;  // (cos, sin) entries per row

// Device view of a packed layout, passed by value to kernels.
struct LayoutView {
  int S;                    // rows per batch element
  int n_tiles;              // ceil(S / 128)
  const int32_t* tags;      // [S]
  const int32_t* t_idx;     // [S]
  const float2* rope;       // [S, 48] (cos, sin) of pos[r][a] * inv_freq[j], index 16a + j
  const uint8_t* tile_class;  // [n_tiles] 0 valid, 1 padding, 2 mixed
  const uint32_t* key_valid;  // [n_tiles * 4] bit i of word w: row 128 t + 32 w + i is valid
  int* err;                 // device error word
};

}  // namespace h3

// The opaque layout object of the C ABI.
struct h3_layout {
  int S = 0, n_t = 0, n_video = 0, n_audio = 0, n_text = 0, n_valid = 0, n_tiles = 0;
  int device = 0;
  void* block = nullptr;  // single device allocation holding every table
  int32_t *tags = nullptr, *t_idx = nullptr, *video_idx = nullptr, *audio_idx = nullptr,
          *text_idx = nullptr, *src_of_row = nullptr, *perm = nullptr;
  float* pos = nullptr;
  float2* rope = nullptr;
  uint8_t* tile_class = nullptr;
  uint32_t* key_valid = nullptr;
  // compacted (valid rows only) view
  int32_t *c_tags = nullptr, *c_tidx = nullptr;
  float2* c_rope = nullptr;
  uint8_t* c_tile_class = nullptr;
  uint32_t* c_key_valid = nullptr;
  int c_tiles = 0;
  int32_t* c_of_row = nullptr;  // [S] compact position of each packed row, -1 for padding
  // the text rows alone (text_idx order): the refiner's sequence
  int32_t *t_tags = nullptr, *t_tidx = nullptr;
  float2* t_rope = nullptr;
  uint8_t* t_tile_class = nullptr;
  uint32_t* t_key_valid = nullptr;
  int t_tiles = 0;
  // a token-reduced layout (from h3_layout_reduce): for each of its compact
  // rows, the source rows in its parent's compact stream (second -1 if single)
  void* extra = nullptr;
  int2* red_map = nullptr;
  int red_parent_S = -1, red_parent_V = -1;
  int* err = nullptr;
  std::vector<uint8_t> tile_class_host;

  h3::LayoutView view() const {
    return h3::LayoutView{S, n_tiles, tags, t_idx, rope, tile_class, key_valid, err};
  }
  h3::LayoutView compact_view() const {
    return h3::LayoutView{n_valid, c_tiles, c_tags, c_tidx, c_rope, c_tile_class, c_key_valid,
                          err};
  }
  h3::LayoutView text_view() const {
    return h3::LayoutView{n_text, t_tiles, t_tags, t_tidx, t_rope, t_tile_class, t_key_valid,
                          err};
  }
};

namespace h3 {

// ---- launchers (each returns cudaError_t of the launch) ----

cudaError_t launch_layout_prepare(h3_layout* L, float rope_theta, int* d_status,
                                  int32_t* d_scratch, cudaStream_t st);
cudaError_t launch_compact_tables(h3_layout* L, cudaStream_t st);
cudaError_t launch_pack(const h3_layout* L, int B, int row_elems, const void* video,
                        const void* audio, const void* text, void* x, cudaStream_t st);
cudaError_t launch_unpack(const h3_layout* L, int B, int row_elems, const void* x, void* video,
                          void* audio, void* text, cudaStream_t st);
// dst[b, j] = src[b, perm[j]] (gather == true, src [B, S_src, E], dst [B, n, E])
// dst[b, perm[j]] = src[b, j] (gather == false, src [B, n, E], dst [B, S_dst, E])
cudaError_t launch_permute_rows(int B, int n, int S_full, int row_elems, const int32_t* perm,
                                const void* src, void* dst, bool gather, cudaStream_t st);
// Same, converting the rows: gather bf16 -> fp32, scatter fp32 -> bf16 (round to nearest even).
cudaError_t launch_permute_rows_convert(int B, int n, int S_full, int row_elems,
                                        const int32_t* perm, const void* src, void* dst,
                                        bool gather, cudaStream_t st);

// x_f32: the residual stream x is fp32 (inside the stack) instead of bf16.
cudaError_t launch_norm_modulate(const LayoutView& L, int B, int H, int chunk_shift,
                                 int chunk_scale, float eps, const void* x, bool x_f32,
                                 const float* table, const float* tmod, void* h,
                                 cudaStream_t st);

// The same normalised, modulated rows as e4m3 codes [rows, H] with one scale
// per row (max |h| / 448), and bf16 weight rows [rows, K] as e4m3 codes with
// one scale per row.
cudaError_t launch_norm_modulate_e4m3(const LayoutView& L, int B, int H, int chunk_shift,
                                      int chunk_scale, float eps, const void* x, bool x_f32,
                                      const float* table, const float* tmod, void* codes,
                                      float* row_scale, cudaStream_t st);
cudaError_t launch_quantize_rows_e4m3(int rows, int K, const void* w, void* codes,
                                      float* row_scale, cudaStream_t st);

// The prologue's fp32 GEMMs run either on the CUDA cores or, for many distinct
// timesteps, as bf16 tensor-core GEMMs over three-way bf16 splits of both
// operands (allow_split = false forces the first form). Workspace bytes for
// either form; ws must be 256-byte aligned.
size_t timestep_workspace_bytes(const h3_dims& d, int n_t, bool allow_split);
// With w_out (else null) it also writes tmod_out = W_out . SiLU(temb) [n_t, 2H].
cudaError_t launch_timestep(const h3_dims& d, int n_t, const float* t, const float* w_t1,
                            const float* w_t2, const float* w_proj, float* tmod, void* ws,
                            bool allow_split, cudaStream_t st, const float* w_out = nullptr,
                            float* tmod_out = nullptr);

// EPI_RESID_F32: gated residual on an fp32 residual stream (inside the stack).
enum GemmEpilogue {
  EPI_STORE = 0,
  EPI_QKV = 1,
  EPI_RESID = 2,
  EPI_SWIGLU = 3,
  EPI_RESID_F32 = 4,
  EPI_F32 = 5
};

// Up to this many destination buffers for the outputs of one launch (the ranks
// of the sequence-parallel block; one for the plain block).
constexpr int kMaxDst = 8;

// Where EPI_QKV puts q / k / v of head h, row s of batch element b:
// q[h / heads_per_dst] + ((b * heads_per_dst + h % heads_per_dst) * dst_rows
// + row_offset + s) * 128 (likewise k, v). The plain block: one destination
// with all NH heads, dst_rows = S, row_offset = 0.
struct HeadMap {
  void* q[kMaxDst] = {};
  void* k[kMaxDst] = {};
  void* v[kMaxDst] = {};
  int heads_per_dst = 0, dst_rows = 0, row_offset = 0;
};

// Where attention puts the output of row s, head h (of this launch's NH heads)
// of batch element b: o[s / rows_per_dst] + ((b * rows_per_dst + s %
// rows_per_dst) * row_heads + head_offset + h) * 128. The plain block: one
// destination, rows_per_dst = S, row_heads = NH, head_offset = 0.
struct RowMap {
  void* o[kMaxDst] = {};
  int rows_per_dst = 0, row_heads = 0, head_offset = 0;
};

inline HeadMap plain_head_map(void* q, void* k, void* v, int NH, int S) {
  HeadMap m;
  m.q[0] = q;
  m.k[0] = k;
  m.v[0] = v;
  m.heads_per_dst = NH;
  m.dst_rows = S;
  return m;
}

inline RowMap plain_row_map(void* o, int NH, int S) {
  RowMap m;
  m.o[0] = o;
  m.rows_per_dst = S;
  m.row_heads = NH;
  return m;
}

struct GemmEpiArgs {
  LayoutView L;
  int B = 1, NH = 0;
  // EPI_STORE: out [M, N] bf16; EPI_F32: out [M, N] fp32; EPI_SWIGLU: out [M, N/2]
  void* out = nullptr;
  // EPI_QKV
  HeadMap heads;
  const void *q_norm = nullptr, *k_norm = nullptr;
  float qk_eps = 0.f;
  // EPI_RESID: x [M, N] in/out, gate = table[tag][gate_chunk] + tmod[t_idx][gate_chunk]
  void* x = nullptr;
  const float* table = nullptr;
  const float* tmod = nullptr;
  int gate_chunk = 0;
  // e4m3 GEMMs: per-row activation scales [M] and per-column weight scales [N]
  const float* a_scale = nullptr;
  const float* b_scale = nullptr;
};

// C[M, N] epilogue( A[M, K] . B[N, K]^T ), bf16 in, fp32 accumulate.
cudaError_t launch_gemm(int epi, int M, int N, int K, const void* A, const void* Bm,
                        const GemmEpiArgs& e, cudaStream_t st);

// The same product on e4m3 codes (A [M, K], B [N, K] bytes) with
// C[m, n] = a_scale[m] * b_scale[n] * (A . B^T)[m, n]; EPI_QKV, EPI_SWIGLU,
// EPI_RESID or EPI_RESID_F32 (N % 256 == 0, K % 128 == 0).
cudaError_t launch_gemm_e4m3(int epi, int M, int N, int K, const void* A, const void* Bm,
                             const GemmEpiArgs& e, cudaStream_t st);

cudaError_t launch_attention(const LayoutView& L, int B, int NH, const void* q, const void* k,
                             const void* v, const RowMap& out, cudaStream_t st);
inline cudaError_t launch_attention(const LayoutView& L, int B, int NH, const void* q,
                                    const void* k, const void* v, void* o, cudaStream_t st) {
  return launch_attention(L, B, NH, q, k, v, plain_row_map(o, NH, L.S), st);
}

int num_sms();

// ---- token reduction (reduce.cu) ----
cudaError_t launch_pair_heads(const h3_layout* L, const int32_t* target, uint8_t* head,
                              cudaStream_t st);
cudaError_t launch_reduce_build(const h3_layout* L, const uint8_t* head, int32_t* r_tags,
                                int32_t* r_tidx, float* r_pos, int32_t* r_src_a, int32_t* r_src_b,
                                int32_t* r_video, int32_t* r_text, int32_t* r_audio,
                                int32_t* out_n, cudaStream_t st);
cudaError_t launch_reduce_map(int Sr, const int32_t* r_tags, const int32_t* src_a,
                              const int32_t* src_b, const int32_t* c_of_row_r,
                              const int32_t* c_of_row_full, int2* map, cudaStream_t st);
cudaError_t launch_merge(int B, int Vr, int V, int H, const int2* map, const float* xc,
                         float* xr, cudaStream_t st);
cudaError_t launch_restore(int B, int Vr, int V, int H, const int2* map, const float* xr,
                           float* xc, cudaStream_t st);

// ---- the denoiser around the stack (denoiser.cu) ----
// y = a + s y elementwise over n floats (n % 4 == 0, 16-byte aligned).
cudaError_t launch_combine(size_t n, const float* a, float s, float* y, cudaStream_t st);
// Latent / velocity row widths the projection and head kernels take.
bool io_channels_supported(int C);
// xc[b, c_of_row[idx[i]]] = W . lat[b, i] (fp32; lat [B, n, C], W [H, C]).
cudaError_t launch_patch_project(int B, int n, int H, int V, int C, const float* lat,
                                 const float* W, const int32_t* idx, const int32_t* c_of_row,
                                 float* xc, cudaStream_t st);
// xc[b, c_of_row[idx[i]]] = LayerNorm(src[b, i]) (no affine).
cudaError_t launch_rows_layer_norm(int B, int n, int H, int V, float eps, const float* src,
                                   const int32_t* idx, const int32_t* c_of_row, float* xc,
                                   cudaStream_t st);
// out[b, i] = W . (LN(x) (1 + scale) + shift), x = xc[b, c_of_row[idx[i]]],
// (shift, scale) = table[0..1] + tmod_out[t_idx[idx[i]]][0..1] (fp32; W [C, H]).
cudaError_t launch_out_head(int B, int n, int H, int V, int C, float eps, const float* xc,
                            const int32_t* idx, const int32_t* c_of_row, const int32_t* t_idx,
                            const float* table, const float* tmod_out, const float* W,
                            float* out, cudaStream_t st);

// Shape checks shared by the entry points (H3_OK or the status to return).
h3_status check_dims(const h3_dims* d);

// Device address of a file-scope __device__ symbol on the current device, looked
// up once per device and again whenever the device's context changes (after a
// cudaDeviceReset the module is loaded anew, possibly at another address).
// `lookup` calls cudaGetSymbolAddress in the translation unit that defines the
// symbol.
struct SymbolAddressCache {
  static constexpr int kMaxDevices = 64;
  unsigned long long context_id[kMaxDevices] = {};
  void* address[kMaxDevices] = {};
};
h3_status symbol_address(SymbolAddressCache& cache, cudaError_t (*lookup)(void**), void** out);

}  // namespace h3
