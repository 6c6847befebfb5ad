// C ABI entry points: argument checks, layout object, block and stack
// orchestration. Every step of the computation runs in this library's kernels.
#include <stdio.h>

#include <new>

#include "internal.cuh"

using namespace h3;

namespace h3 {

h3_status check_dims(const h3_dims* d) {
  if (!d) return H3_ERR_ARG;
  if (d->head_dim != 128 || d->rope_freq_dim != kRopeFreqs) return H3_ERR_SHAPE;
  if (d->hidden <= 0 || d->hidden % 256 != 0 || d->hidden > 24 * 256) return H3_ERR_SHAPE;
  if (d->heads <= 0 || d->heads % 2 != 0) return H3_ERR_SHAPE;
  if (d->ffn <= 0 || d->ffn % 128 != 0) return H3_ERR_SHAPE;
  if (d->n_modalities < 3) return H3_ERR_SHAPE;
  // The prologue's GEMMs read rows in 16-byte vectors.
  if (d->freq_dim <= 0 || d->freq_dim % 4 != 0 || d->time_hidden <= 0 ||
      d->time_hidden % 4 != 0 || d->time_embed_dim <= 0 || d->time_embed_dim % 4 != 0)
    return H3_ERR_SHAPE;
  if (!(d->norm_eps > 0.f) || !(d->qk_norm_eps > 0.f) || !(d->rope_theta > 0.f))
    return H3_ERR_ARG;
  return H3_OK;
}

}  // namespace h3

namespace {

inline cudaStream_t as_stream(h3_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

// B batch elements of the layout's S rows: B * S rows must fit an int and B the
// attention grid.
h3_status check_batch(const h3_layout* L, int B) {
  if (!L || B < 0) return H3_ERR_ARG;
  if (B > kMaxBatch || (long long)B * L->S > 0x7fffffffLL) return H3_ERR_SHAPE;
  return H3_OK;
}

inline h3_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return H3_OK;
  if (e == cudaErrorInvalidValue) return H3_ERR_ARG;
  return H3_ERR_CUDA;
}

#define H3_TRY(expr)                      \
  do {                                    \
    const h3_status _s = (expr);          \
    if (_s != H3_OK) return _s;           \
  } while (0)

#define H3_CUDA(expr) H3_TRY(cuda_status(expr))

struct Workspace {
  void *h, *qkv_g, *o, *xc;
  void *q, *k, *v, *g;
};

// Bytes per row of the 8-bit activation codes: the widest GEMM input (h, o or g).
size_t e4m3_row_bytes(const h3_dims& d) {
  size_t m = (size_t)d.hidden;
  const size_t A = (size_t)d.heads * d.head_dim;
  if (A > m) m = A;
  if ((size_t)d.ffn > m) m = d.ffn;
  return m;
}

size_t ws_parts(const h3_dims& d, int B, int S, Workspace* w, void* base) {
  const size_t rows = (size_t)B * S;
  const size_t A = (size_t)d.heads * d.head_dim;
  const size_t h_b = align256(rows * d.hidden * 2);
  const size_t one_b = align256(rows * A * 2);          // q, k, v each
  const size_t g_b = align256(rows * (size_t)d.ffn * 2);  // g reuses the q/k/v region
  const size_t qg_b = 3 * one_b > g_b ? 3 * one_b : g_b;
  const size_t o_b = align256(rows * A * 2);
  const size_t xc_b = align256(rows * d.hidden * 4);  // the stack's fp32 residual stream
  if (w) {
    uint8_t* p = static_cast<uint8_t*>(base);
    w->h = p;
    w->qkv_g = p + h_b;
    w->o = p + h_b + qg_b;
    w->xc = p + h_b + qg_b + o_b;
    w->q = w->qkv_g;
    w->k = static_cast<uint8_t*>(w->qkv_g) + one_b;
    w->v = static_cast<uint8_t*>(w->qkv_g) + 2 * one_b;
    w->g = w->qkv_g;
  }
  return h_b + qg_b + o_b + xc_b;
}

h3_status check_weights(const h3_block_weights* w) {
  if (!w || !w->w_qkv || !w->q_norm || !w->k_norm || !w->w_o || !w->w13 || !w->w2 ||
      !w->ada_table)
    return H3_ERR_ARG;
  if (!aligned16(w->w_qkv) || !aligned16(w->q_norm) || !aligned16(w->k_norm) ||
      !aligned16(w->w_o) || !aligned16(w->w13) || !aligned16(w->w2) || !aligned16(w->ada_table))
    return H3_ERR_ALIGN;
  return H3_OK;
}

// One block over the rows described by `L` (full or compacted view), in place on
// x: bf16 for h3_block_forward, fp32 (x_f32) for the stack's residual stream.
// 8-bit operands of the QKV and W1 || W3 GEMMs (null: the bf16 block). codes
// [M, H] bytes and scales [M] are workspace for the activation rows.
struct E4m3Operands {
  const h3_block_weights_e4m3* w = nullptr;
  void* codes = nullptr;
  float* scales = nullptr;
};

h3_status run_block(const h3_dims& d, const h3_block_weights& w, const LayoutView& L,
                    const float* tmod, void* x, bool x_f32, int B, const Workspace& ws,
                    cudaStream_t st, const E4m3Operands& q8 = E4m3Operands()) {
  const int M = B * L.S;
  if (M == 0) return H3_OK;
  const int H = d.hidden, A = d.heads * d.head_dim, Fd = d.ffn;
  if (q8.w)
    H3_CUDA(launch_norm_modulate_e4m3(L, B, H, 0, 1, d.norm_eps, x, x_f32, w.ada_table, tmod,
                                      q8.codes, q8.scales, st));
  else
    H3_CUDA(launch_norm_modulate(L, B, H, 0, 1, d.norm_eps, x, x_f32, w.ada_table, tmod, ws.h,
                                 st));
  GemmEpiArgs e;
  e.L = L;
  e.B = B;
  e.NH = d.heads;
  e.heads = plain_head_map(ws.q, ws.k, ws.v, d.heads, L.S);
  e.q_norm = w.q_norm;
  e.k_norm = w.k_norm;
  e.qk_eps = d.qk_norm_eps;
  if (q8.w) {
    e.a_scale = q8.scales;
    e.b_scale = q8.w->w_qkv_scales;
    H3_CUDA(launch_gemm_e4m3(EPI_QKV, M, 3 * A, H, q8.codes, q8.w->w_qkv_codes, e, st));
  } else {
    H3_CUDA(launch_gemm(EPI_QKV, M, 3 * A, H, ws.h, w.w_qkv, e, st));
  }
  H3_CUDA(launch_attention(L, B, d.heads, ws.q, ws.k, ws.v, ws.o, st));
  GemmEpiArgs r;
  r.L = L;
  r.B = B;
  r.x = x;
  r.table = w.ada_table;
  r.tmod = tmod;
  r.gate_chunk = 2;
  const int resid = x_f32 ? EPI_RESID_F32 : EPI_RESID;
  if (q8.w && q8.w->w_o_codes) {  // o as stored (bf16), quantized per row
    H3_CUDA(launch_quantize_rows_e4m3(M, A, ws.o, q8.codes, q8.scales, st));
    GemmEpiArgs r8 = r;
    r8.a_scale = q8.scales;
    r8.b_scale = q8.w->w_o_scales;
    H3_CUDA(launch_gemm_e4m3(resid, M, H, A, q8.codes, q8.w->w_o_codes, r8, st));
  } else {
    H3_CUDA(launch_gemm(resid, M, H, A, ws.o, w.w_o, r, st));
  }
  GemmEpiArgs sg;
  sg.L = L;
  sg.out = ws.g;
  if (q8.w) {
    H3_CUDA(launch_norm_modulate_e4m3(L, B, H, 3, 4, d.norm_eps, x, x_f32, w.ada_table, tmod,
                                      q8.codes, q8.scales, st));
    sg.a_scale = q8.scales;
    sg.b_scale = q8.w->w13_scales;
    H3_CUDA(launch_gemm_e4m3(EPI_SWIGLU, M, 2 * Fd, H, q8.codes, q8.w->w13_codes, sg, st));
  } else {
    H3_CUDA(launch_norm_modulate(L, B, H, 3, 4, d.norm_eps, x, x_f32, w.ada_table, tmod, ws.h,
                                 st));
    H3_CUDA(launch_gemm(EPI_SWIGLU, M, 2 * Fd, H, ws.h, w.w13, sg, st));
  }
  r.gate_chunk = 5;
  if (q8.w && q8.w->w2_codes) {  // g as stored (bf16), quantized per row
    H3_CUDA(launch_quantize_rows_e4m3(M, Fd, ws.g, q8.codes, q8.scales, st));
    GemmEpiArgs r8 = r;
    r8.a_scale = q8.scales;
    r8.b_scale = q8.w->w2_scales;
    H3_CUDA(launch_gemm_e4m3(resid, M, H, Fd, q8.codes, q8.w->w2_codes, r8, st));
  } else {
    H3_CUDA(launch_gemm(resid, M, H, Fd, ws.g, w.w2, r, st));
  }
  return H3_OK;
}

}  // namespace

extern "C" {

const char* h3_status_string(h3_status s) {
  switch (s) {
    case H3_OK: return "ok";
    case H3_ERR_ARG: return "invalid argument";
    case H3_ERR_SHAPE: return "unsupported shape";
    case H3_ERR_ALIGN: return "pointer not 16-byte aligned";
    case H3_ERR_LAYOUT: return "inconsistent packed layout";
    case H3_ERR_WORKSPACE: return "workspace too small";
    case H3_ERR_CUDA: return "CUDA error";
    case H3_ERR_TIMEOUT: return "bounded in-kernel wait timed out";
  }
  return "unknown status";
}

int h3_abi_version(void) { return 1; }

h3_status h3_layout_prepare(const h3_dims* dims, const h3_layout_desc* desc, h3_stream_t stream,
                            h3_layout_t* out) {
  if (!out || !desc) return H3_ERR_ARG;
  *out = nullptr;
  H3_TRY(check_dims(dims));
  const int S = desc->S;
  if (S < 0 || desc->n_t < 0 || desc->n_video < 0 || desc->n_audio < 0 || desc->n_text < 0)
    return H3_ERR_ARG;
  if (S > kMaxRows) return H3_ERR_SHAPE;
  if (S > 0 && (!desc->pos || !desc->tags || !desc->t_idx)) return H3_ERR_ARG;
  if ((desc->n_video && !desc->video_idx) || (desc->n_audio && !desc->audio_idx) ||
      (desc->n_text && !desc->text_idx))
    return H3_ERR_ARG;
  if (desc->n_video + desc->n_audio + desc->n_text > S) return H3_ERR_LAYOUT;
  cudaStream_t st = as_stream(stream);
  h3_layout* L = new (std::nothrow) h3_layout();
  if (!L) return H3_ERR_CUDA;
  cudaGetDevice(&L->device);
  L->S = S;
  L->n_t = desc->n_t;
  L->n_video = desc->n_video;
  L->n_audio = desc->n_audio;
  L->n_text = desc->n_text;
  L->n_tiles = (S + kTile - 1) / kTile;
  const size_t nt = L->n_tiles;
  const size_t sz_i = align256((size_t)S * 4), sz_pos = align256((size_t)S * 12),
               sz_rope = align256((size_t)S * kRopePairs * 8), sz_tc = align256(nt),
               sz_kv = align256(nt * 16);
  const size_t n_tt = (desc->n_text + kTile - 1) / kTile;
  const size_t sz_ti = align256((size_t)desc->n_text * 4),
               sz_trope = align256((size_t)desc->n_text * kRopePairs * 8),
               sz_ttc = align256(n_tt), sz_tkv = align256(n_tt * 16);
  const size_t total = 7 * sz_i /*tags t_idx src perm c_tags c_tidx c_of_row*/ + sz_pos +
                       2 * sz_rope + 2 * sz_tc + 2 * sz_kv + align256((size_t)desc->n_video * 4) +
                       align256((size_t)desc->n_audio * 4) + align256((size_t)desc->n_text * 4) +
                       2 * sz_ti + sz_trope + sz_ttc + sz_tkv /*text view*/ + 256 /*err*/;
  if (cudaMalloc(&L->block, total) != cudaSuccess) {
    delete L;
    return H3_ERR_CUDA;
  }
  uint8_t* p = static_cast<uint8_t*>(L->block);
  auto take = [&](size_t n) {
    uint8_t* q = p;
    p += n;
    return q;
  };
  L->tags = reinterpret_cast<int32_t*>(take(sz_i));
  L->t_idx = reinterpret_cast<int32_t*>(take(sz_i));
  L->src_of_row = reinterpret_cast<int32_t*>(take(sz_i));
  L->perm = reinterpret_cast<int32_t*>(take(sz_i));
  L->c_tags = reinterpret_cast<int32_t*>(take(sz_i));
  L->c_tidx = reinterpret_cast<int32_t*>(take(sz_i));
  L->pos = reinterpret_cast<float*>(take(sz_pos));
  L->rope = reinterpret_cast<float2*>(take(sz_rope));
  L->c_rope = reinterpret_cast<float2*>(take(sz_rope));
  L->tile_class = take(sz_tc);
  L->c_tile_class = take(sz_tc);
  L->key_valid = reinterpret_cast<uint32_t*>(take(sz_kv));
  L->c_key_valid = reinterpret_cast<uint32_t*>(take(sz_kv));
  L->video_idx = reinterpret_cast<int32_t*>(take(align256((size_t)desc->n_video * 4)));
  L->audio_idx = reinterpret_cast<int32_t*>(take(align256((size_t)desc->n_audio * 4)));
  L->text_idx = reinterpret_cast<int32_t*>(take(align256((size_t)desc->n_text * 4)));
  L->c_of_row = reinterpret_cast<int32_t*>(take(sz_i));
  L->t_tags = reinterpret_cast<int32_t*>(take(sz_ti));
  L->t_tidx = reinterpret_cast<int32_t*>(take(sz_ti));
  L->t_rope = reinterpret_cast<float2*>(take(sz_trope));
  L->t_tile_class = take(sz_ttc);
  L->t_key_valid = reinterpret_cast<uint32_t*>(take(sz_tkv));
  L->t_tiles = (int)n_tt;
  L->err = reinterpret_cast<int*>(take(256));

  h3_status rc = H3_OK;
  int32_t* scratch = nullptr;  // hits[S], tile_pad[n_tiles], counts[4], n_valid, status
  const size_t scratch_n = (size_t)S + nt + 4 + 1 + 1;
  int host_st[2] = {0, 0};
  do {
    if (cudaMalloc(&scratch, scratch_n * 4) != cudaSuccess) { rc = H3_ERR_CUDA; break; }
    if (cudaMemsetAsync(scratch, 0, scratch_n * 4, st) != cudaSuccess ||
        cudaMemsetAsync(L->err, 0, 256, st) != cudaSuccess) { rc = H3_ERR_CUDA; break; }
    bool cp_ok = true;
    if (S > 0) {
      cp_ok &= cudaMemcpyAsync(L->tags, desc->tags, (size_t)S * 4, cudaMemcpyDeviceToDevice, st) == cudaSuccess;
      cp_ok &= cudaMemcpyAsync(L->t_idx, desc->t_idx, (size_t)S * 4, cudaMemcpyDeviceToDevice, st) == cudaSuccess;
      cp_ok &= cudaMemcpyAsync(L->pos, desc->pos, (size_t)S * 12, cudaMemcpyDeviceToDevice, st) == cudaSuccess;
    }
    if (desc->n_video)
      cp_ok &= cudaMemcpyAsync(L->video_idx, desc->video_idx, (size_t)desc->n_video * 4, cudaMemcpyDeviceToDevice, st) == cudaSuccess;
    if (desc->n_audio)
      cp_ok &= cudaMemcpyAsync(L->audio_idx, desc->audio_idx, (size_t)desc->n_audio * 4, cudaMemcpyDeviceToDevice, st) == cudaSuccess;
    if (desc->n_text)
      cp_ok &= cudaMemcpyAsync(L->text_idx, desc->text_idx, (size_t)desc->n_text * 4, cudaMemcpyDeviceToDevice, st) == cudaSuccess;
    if (!cp_ok) { rc = H3_ERR_CUDA; break; }
    int* d_status = scratch + S + nt + 5;
    if (launch_layout_prepare(L, dims->rope_theta, d_status, scratch, st) != cudaSuccess) {
      rc = H3_ERR_CUDA;
      break;
    }
    // n_valid (scratch[S + nt + 4]) and status are adjacent
    if (cudaMemcpyAsync(host_st, scratch + S + nt + 4, 8, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
      rc = H3_ERR_CUDA;
      break;
    }
    if (host_st[1] != 0) { rc = H3_ERR_LAYOUT; break; }
    L->n_valid = host_st[0];
    L->c_tiles = (L->n_valid + kTile - 1) / kTile;
    if (launch_compact_tables(L, st) != cudaSuccess) { rc = H3_ERR_CUDA; break; }
    L->tile_class_host.resize(nt);
    if (nt && cudaMemcpyAsync(L->tile_class_host.data(), L->tile_class, nt, cudaMemcpyDeviceToHost, st) != cudaSuccess) {
      rc = H3_ERR_CUDA;
      break;
    }
    if (cudaStreamSynchronize(st) != cudaSuccess) { rc = H3_ERR_CUDA; break; }
  } while (0);
  if (scratch) cudaFree(scratch);
  if (rc != H3_OK) {
    cudaFree(L->block);
    delete L;
    return rc;
  }
  *out = L;
  return H3_OK;
}

void h3_layout_destroy(h3_layout_t L) {
  if (!L) return;
  cudaDeviceSynchronize();
  cudaFree(L->block);
  if (L->extra) cudaFree(L->extra);
  delete L;
}

h3_status h3_layout_error(h3_layout_t L) {
  if (!L) return H3_ERR_ARG;
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return H3_ERR_CUDA;
  if (cudaMemcpy(&v, L->err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return H3_ERR_CUDA;
  if (v != 0 && cudaMemset(L->err, 0, 4) != cudaSuccess) return H3_ERR_CUDA;
  return v == 0 ? H3_OK : H3_ERR_TIMEOUT;
}

h3_status h3_layout_export(h3_layout_t L, int32_t* perm_host, uint8_t* tile_class_host,
                           int32_t* n_valid_host) {
  if (!L) return H3_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return H3_ERR_CUDA;
  if (perm_host && L->S > 0 &&
      cudaMemcpy(perm_host, L->perm, (size_t)L->S * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return H3_ERR_CUDA;
  if (tile_class_host && L->n_tiles > 0 &&
      cudaMemcpy(tile_class_host, L->tile_class, L->n_tiles, cudaMemcpyDeviceToHost) != cudaSuccess)
    return H3_ERR_CUDA;
  if (n_valid_host) *n_valid_host = L->n_valid;
  return H3_OK;
}

size_t h3_workspace_size(const h3_dims* dims, int B, int S) {
  if (check_dims(dims) != H3_OK || B < 0 || S < 0) return 0;
  return ws_parts(*dims, B, S, nullptr, nullptr);
}

h3_status h3_pack_rows(h3_layout_t L, int B, int row_elems, const void* video, const void* audio,
                       const void* text, void* x_packed, h3_stream_t stream) {
  if (!L || B < 0 || row_elems <= 0 || !x_packed) return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (row_elems % 8 != 0) return H3_ERR_SHAPE;
  if ((L->n_video && !video) || (L->n_audio && !audio) || (L->n_text && !text)) return H3_ERR_ARG;
  if (!aligned16(video) || !aligned16(audio) || !aligned16(text) || !aligned16(x_packed))
    return H3_ERR_ALIGN;
  H3_CUDA(launch_pack(L, B, row_elems, video, audio, text, x_packed, as_stream(stream)));
  return H3_OK;
}

h3_status h3_unpack_rows(h3_layout_t L, int B, int row_elems, const void* x_packed, void* video,
                         void* audio, void* text, h3_stream_t stream) {
  if (!L || B < 0 || row_elems <= 0 || !x_packed) return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (row_elems % 8 != 0) return H3_ERR_SHAPE;
  if (!aligned16(video) || !aligned16(audio) || !aligned16(text) || !aligned16(x_packed))
    return H3_ERR_ALIGN;
  H3_CUDA(launch_unpack(L, B, row_elems, x_packed, video, audio, text, as_stream(stream)));
  return H3_OK;
}

size_t h3_timestep_workspace_size(const h3_dims* dims, int n_t) {
  if (check_dims(dims) != H3_OK || n_t < 0) return 0;
  return h3::timestep_workspace_bytes(*dims, n_t, true);
}

h3_status h3_timestep_modulation(const h3_dims* dims, int n_t, const float* t, const float* w_t1,
                                 const float* w_t2, const float* w_proj, float* tmod, void* ws,
                                 size_t ws_bytes, h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (n_t < 0) return H3_ERR_ARG;
  if (n_t == 0) return H3_OK;
  if (!t || !w_t1 || !w_t2 || !w_proj || !tmod || !ws) return H3_ERR_ARG;
  if (!aligned16(t) || !aligned16(w_t1) || !aligned16(w_t2) || !aligned16(w_proj) ||
      !aligned16(tmod) || !aligned16(ws))
    return H3_ERR_ALIGN;
  if (ws_bytes < h3_timestep_workspace_size(dims, n_t)) return H3_ERR_WORKSPACE;
  H3_CUDA(launch_timestep(*dims, n_t, t, w_t1, w_t2, w_proj, tmod, ws, true, as_stream(stream)));
  return H3_OK;
}

h3_status h3_norm_modulate(const h3_dims* dims, h3_layout_t L, int B, int which, const void* x,
                           const float* ada_table, const float* tmod, void* h,
                           h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || (which != 0 && which != 1) || !x || !ada_table || !tmod || !h)
    return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (!aligned16(x) || !aligned16(ada_table) || !aligned16(tmod) || !aligned16(h))
    return H3_ERR_ALIGN;
  const int c0 = which == 0 ? 0 : 3;
  H3_CUDA(launch_norm_modulate(L->view(), B, dims->hidden, c0, c0 + 1, dims->norm_eps, x, false,
                               ada_table, tmod, h, as_stream(stream)));
  return H3_OK;
}

h3_status h3_qkv_rope(const h3_dims* dims, h3_layout_t L, int B, const void* h, const void* w_qkv,
                      const void* q_norm, const void* k_norm, void* q, void* k, void* v,
                      h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || !h || !w_qkv || !q_norm || !k_norm || !q || !k || !v) return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (!aligned16(h) || !aligned16(w_qkv) || !aligned16(q_norm) || !aligned16(k_norm) ||
      !aligned16(q) || !aligned16(k) || !aligned16(v))
    return H3_ERR_ALIGN;
  GemmEpiArgs e;
  e.L = L->view();
  e.B = B;
  e.NH = dims->heads;
  e.heads = plain_head_map(q, k, v, dims->heads, L->S);
  e.q_norm = q_norm;
  e.k_norm = k_norm;
  e.qk_eps = dims->qk_norm_eps;
  H3_CUDA(launch_gemm(EPI_QKV, B * L->S, 3 * dims->heads * dims->head_dim, dims->hidden, h,
                      w_qkv, e, as_stream(stream)));
  return H3_OK;
}

h3_status h3_attention(const h3_dims* dims, h3_layout_t L, int B, const void* q, const void* k,
                       const void* v, void* o, h3_stream_t stream) {
  // Attention alone needs only head_dim 128 and any head count (a rank of the
  // sequence-parallel block runs it on heads / P heads).
  if (!dims) return H3_ERR_ARG;
  if (dims->head_dim != 128 || dims->heads <= 0 || dims->heads > 65535) return H3_ERR_SHAPE;
  if (!L || B < 0 || !q || !k || !v || !o) return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return H3_ERR_ALIGN;
  H3_CUDA(launch_attention(L->view(), B, dims->heads, q, k, v, o, as_stream(stream)));
  return H3_OK;
}

h3_status h3_out_residual(const h3_dims* dims, h3_layout_t L, int B, const void* o,
                          const void* w_o, const float* ada_table, const float* tmod, void* x,
                          h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || !o || !w_o || !ada_table || !tmod || !x) return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (!aligned16(o) || !aligned16(w_o) || !aligned16(ada_table) || !aligned16(tmod) ||
      !aligned16(x))
    return H3_ERR_ALIGN;
  GemmEpiArgs r;
  r.L = L->view();
  r.B = B;
  r.x = x;
  r.table = ada_table;
  r.tmod = tmod;
  r.gate_chunk = 2;
  H3_CUDA(launch_gemm(EPI_RESID, B * L->S, dims->hidden, dims->heads * dims->head_dim, o, w_o, r,
                      as_stream(stream)));
  return H3_OK;
}

h3_status h3_ffn_up(const h3_dims* dims, h3_layout_t L, int B, const void* h2, const void* w13,
                    void* g, h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || !h2 || !w13 || !g) return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (!aligned16(h2) || !aligned16(w13) || !aligned16(g)) return H3_ERR_ALIGN;
  GemmEpiArgs sg;
  sg.L = L->view();
  sg.out = g;
  H3_CUDA(launch_gemm(EPI_SWIGLU, B * L->S, 2 * dims->ffn, dims->hidden, h2, w13, sg,
                      as_stream(stream)));
  return H3_OK;
}

h3_status h3_ffn_down_residual(const h3_dims* dims, h3_layout_t L, int B, const void* g,
                               const void* w2, const float* ada_table, const float* tmod,
                               void* x, h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || !g || !w2 || !ada_table || !tmod || !x) return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (!aligned16(g) || !aligned16(w2) || !aligned16(ada_table) || !aligned16(tmod) ||
      !aligned16(x))
    return H3_ERR_ALIGN;
  GemmEpiArgs r;
  r.L = L->view();
  r.B = B;
  r.x = x;
  r.table = ada_table;
  r.tmod = tmod;
  r.gate_chunk = 5;
  H3_CUDA(launch_gemm(EPI_RESID, B * L->S, dims->hidden, dims->ffn, g, w2, r, as_stream(stream)));
  return H3_OK;
}

h3_status h3_block_forward(const h3_dims* dims, const h3_block_weights* weights, h3_layout_t L,
                           const float* tmod, void* x, int B, void* ws, size_t ws_bytes,
                           h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || !tmod || !x || !ws) return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  H3_TRY(check_weights(weights));
  if (!aligned16(tmod) || !aligned16(x) || !aligned16(ws)) return H3_ERR_ALIGN;
  if (ws_bytes < h3_workspace_size(dims, B, L->S)) return H3_ERR_WORKSPACE;
  Workspace w;
  ws_parts(*dims, B, L->S, &w, ws);
  return run_block(*dims, *weights, L->view(), tmod, x, false, B, w, as_stream(stream));
}

h3_status h3_stack_forward(const h3_dims* dims, const h3_block_weights* weights, int n_blocks,
                           h3_layout_t L, const float* tmod, void* x, int B, void* ws,
                           size_t ws_bytes, h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || n_blocks < 0 || !tmod || !x || !ws || (n_blocks > 0 && !weights))
    return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  for (int i = 0; i < n_blocks; ++i) H3_TRY(check_weights(&weights[i]));
  if (!aligned16(tmod) || !aligned16(x) || !aligned16(ws)) return H3_ERR_ALIGN;
  if (ws_bytes < h3_workspace_size(dims, B, L->S)) return H3_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  Workspace w;
  ws_parts(*dims, B, L->S, &w, ws);
  // The valid rows are gathered once (in packed order, padding rows dropped:
  // they never reach a valid row's result and every block leaves them
  // unchanged) into an fp32 residual stream, which all blocks update; the
  // result is rounded to bf16 once when it is scattered back.
  const int V = L->n_valid;
  H3_CUDA(launch_permute_rows_convert(B, V, L->S, dims->hidden, L->perm, x, w.xc, true, st));
  for (int i = 0; i < n_blocks; ++i)
    H3_TRY(run_block(*dims, weights[i], L->compact_view(), tmod, w.xc, true, B, w, st));
  H3_CUDA(launch_permute_rows_convert(B, V, L->S, dims->hidden, L->perm, w.xc, x, false, st));
  return H3_OK;
}

}  // extern "C"

// ---- the denoiser around the stack ----

namespace {

h3_status check_io(const h3_dims* d, const h3_io_dims* io) {
  if (!io) return H3_ERR_ARG;
  if (!io_channels_supported(io->video_channels) || !io_channels_supported(io->audio_channels))
    return H3_ERR_SHAPE;
  if (io->text_dim <= 0 || io->text_dim % 64 != 0) return H3_ERR_SHAPE;
  if (!(io->final_norm_eps > 0.f)) return H3_ERR_ARG;
  (void)d;
  return H3_OK;
}

// Parts of h3_forward's workspace, in order: the stack's block workspace (its
// fp32 stream xc is the forward's residual stream), the refiner's fp32 text
// stream, tmod, tmod_out, and the prologue's scratch.
struct ForwardWs {
  void* block;
  float *text, *tmod, *tmod_out;
  void* prologue;
};

size_t forward_parts(const h3_dims& d, const h3_layout* L, int B, ForwardWs* w, void* base) {
  const size_t block_b = ws_parts(d, B, L->S, nullptr, nullptr);
  const size_t text_b = align256((size_t)B * L->n_text * d.hidden * 4);
  const size_t tmod_b = align256((size_t)L->n_t * 6 * d.hidden * 4);
  const size_t tout_b = align256((size_t)L->n_t * 2 * d.hidden * 4);
  const size_t pro_b = align256(timestep_workspace_bytes(d, L->n_t, true));
  if (w) {
    uint8_t* p = static_cast<uint8_t*>(base);
    w->block = p;
    w->text = reinterpret_cast<float*>(p + block_b);
    w->tmod = reinterpret_cast<float*>(p + block_b + text_b);
    w->tmod_out = reinterpret_cast<float*>(p + block_b + text_b + tmod_b);
    w->prologue = p + block_b + text_b + tmod_b + tout_b;
  }
  return block_b + text_b + tmod_b + tout_b + pro_b;
}

}  // namespace

extern "C" {

size_t h3_forward_workspace_size(const h3_dims* dims, const h3_io_dims* io, h3_layout_t L,
                                 int B) {
  if (check_dims(dims) != H3_OK || check_io(dims, io) != H3_OK || check_batch(L, B) != H3_OK)
    return 0;
  return forward_parts(*dims, L, B, nullptr, nullptr);
}

h3_status h3_forward(const h3_dims* dims, const h3_io_dims* io, const h3_io_weights* iw,
                     const h3_block_weights* refiner, int n_refiner,
                     const h3_block_weights* blocks, int n_blocks, h3_layout_t L,
                     const float* timestep, int B, const float* video, const float* audio,
                     const void* text, float* video_out, float* audio_out, float* core_residual,
                     int core_mode, void* ws, size_t ws_bytes, h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  H3_TRY(check_io(dims, io));
  if (core_mode < H3_CORE_RUN || core_mode > H3_CORE_REUSE) return H3_ERR_ARG;
  if (core_mode != H3_CORE_RUN && (!core_residual || !aligned16(core_residual)))
    return core_residual ? H3_ERR_ALIGN : H3_ERR_ARG;
  if (!L || !iw || n_refiner < 0 || n_blocks < 0 || (n_refiner > 0 && !refiner) ||
      (n_blocks > 0 && !blocks) || !ws)
    return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (L->n_t > 0 && !timestep) return H3_ERR_ARG;
  if (!iw->w_t1 || !iw->w_t2 || !iw->w_proj || !iw->w_out || !iw->out_table)
    return H3_ERR_ARG;
  if (L->n_video && (!video || !video_out || !iw->w_patch_video || !iw->w_head_video))
    return H3_ERR_ARG;
  if (L->n_audio && (!audio || !audio_out || !iw->w_patch_audio || !iw->w_head_audio))
    return H3_ERR_ARG;
  if (L->n_text && (!text || !iw->w_text)) return H3_ERR_ARG;
  for (int i = 0; i < n_refiner; ++i) H3_TRY(check_weights(&refiner[i]));
  for (int i = 0; i < n_blocks; ++i) H3_TRY(check_weights(&blocks[i]));
  const void* ptrs[] = {timestep, video, audio, text, video_out, audio_out, ws, iw->w_patch_video,
                        iw->w_patch_audio, iw->w_text, iw->w_t1, iw->w_t2, iw->w_proj,
                        iw->w_out, iw->out_table, iw->w_head_video, iw->w_head_audio};
  for (const void* p : ptrs)
    if (!aligned16(p)) return H3_ERR_ALIGN;
  if (ws_bytes < forward_parts(*dims, L, B, nullptr, nullptr)) return H3_ERR_WORKSPACE;
  if (B == 0) return H3_OK;
  cudaStream_t st = as_stream(stream);
  const h3_dims& d = *dims;
  const int H = d.hidden, V = L->n_valid;
  ForwardWs fw;
  forward_parts(d, L, B, &fw, ws);
  Workspace w, wt;
  ws_parts(d, B, L->S, &w, fw.block);
  ws_parts(d, B, L->n_text, &wt, fw.block);  // the refiner's scratch, below w.xc
  float* xc = static_cast<float*>(w.xc);
  // timestep MLP, the stack's shared AdaLN projection and norm_out's modulation
  if (L->n_t > 0)
    H3_CUDA(launch_timestep(d, L->n_t, timestep, iw->w_t1, iw->w_t2, iw->w_proj, fw.tmod,
                            fw.prologue, true, st, iw->w_out, fw.tmod_out));
  // input projections into the residual stream
  H3_CUDA(launch_patch_project(B, L->n_video, H, V, io->video_channels, video, iw->w_patch_video,
                               L->video_idx, L->c_of_row, xc, st));
  H3_CUDA(launch_patch_project(B, L->n_audio, H, V, io->audio_channels, audio, iw->w_patch_audio,
                               L->audio_idx, L->c_of_row, xc, st));
  const size_t stream_n = (size_t)B * V * H;
  if (core_mode == H3_CORE_REUSE) {
    // the stored core residual on the fresh projections (text rows carry no output)
    H3_CUDA(launch_combine(stream_n, core_residual, 1.f, xc, st));
  }
  if (core_mode != H3_CORE_REUSE && L->n_text > 0) {
    // text projection (bf16 weights, fp32 out), the refiner blocks on the text
    // rows alone, and the refiner's output norm into the residual stream
    GemmEpiArgs ea;
    ea.L.err = L->err;
    ea.out = fw.text;
    H3_CUDA(launch_gemm(EPI_F32, B * L->n_text, H, io->text_dim, text, iw->w_text, ea, st));
    for (int i = 0; i < n_refiner; ++i)
      H3_TRY(run_block(d, refiner[i], L->text_view(), fw.tmod, fw.text, true, B, wt, st));
    H3_CUDA(launch_rows_layer_norm(B, L->n_text, H, V, io->final_norm_eps, fw.text, L->text_idx,
                                   L->c_of_row, xc, st));
  }
  if (core_mode == H3_CORE_STORE && stream_n)
    H3_CUDA(cudaMemcpyAsync(core_residual, xc, stream_n * 4, cudaMemcpyDeviceToDevice, st));
  if (core_mode != H3_CORE_REUSE)
    for (int i = 0; i < n_blocks; ++i)
      H3_TRY(run_block(d, blocks[i], L->compact_view(), fw.tmod, xc, true, B, w, st));
  // the core residual: the stack's output minus its input
  if (core_mode == H3_CORE_STORE) H3_CUDA(launch_combine(stream_n, xc, -1.f, core_residual, st));
  // norm_out and the two heads, in the order of the index tensors
  H3_CUDA(launch_out_head(B, L->n_video, H, V, io->video_channels, io->final_norm_eps, xc,
                          L->video_idx, L->c_of_row, L->t_idx, iw->out_table, fw.tmod_out,
                          iw->w_head_video, video_out, st));
  H3_CUDA(launch_out_head(B, L->n_audio, H, V, io->audio_channels, io->final_norm_eps, xc,
                          L->audio_idx, L->c_of_row, L->t_idx, iw->out_table + 2 * H,
                          fw.tmod_out, iw->w_head_audio, audio_out, st));
  return H3_OK;
}

}  // extern "C"

// ---- token reduction ----

extern "C" {

h3_status h3_layout_reduce(const h3_dims* dims, h3_layout_t full, const int32_t* target,
                           h3_stream_t stream, h3_layout_t* out) {
  if (!out) return H3_ERR_ARG;
  *out = nullptr;
  H3_TRY(check_dims(dims));
  if (!full || (full->S > 0 && !target)) return H3_ERR_ARG;
  if (!aligned16(target)) return H3_ERR_ALIGN;
  if (full->red_map) return H3_ERR_ARG;  // a reduced layout is not reduced again
  cudaStream_t st = as_stream(stream);
  const int S = full->S;
  const size_t n = (size_t)(S > 0 ? S : 1);
  uint8_t* tmp = nullptr;
  // head [S] u8 | r_tags r_tidx r_src_a r_src_b r_video r_text r_audio [S] i32 | r_pos [3S] f32 | n[4]
  const size_t sz_h = align256(n), sz_i = align256(n * 4), sz_p = align256(n * 12);
  if (cudaMalloc(&tmp, sz_h + 7 * sz_i + sz_p + 256) != cudaSuccess) return H3_ERR_CUDA;
  uint8_t* head = tmp;
  int32_t* r_tags = reinterpret_cast<int32_t*>(tmp + sz_h);
  int32_t* r_tidx = reinterpret_cast<int32_t*>(tmp + sz_h + sz_i);
  int32_t* r_src_a = reinterpret_cast<int32_t*>(tmp + sz_h + 2 * sz_i);
  int32_t* r_src_b = reinterpret_cast<int32_t*>(tmp + sz_h + 3 * sz_i);
  int32_t* r_video = reinterpret_cast<int32_t*>(tmp + sz_h + 4 * sz_i);
  int32_t* r_text = reinterpret_cast<int32_t*>(tmp + sz_h + 5 * sz_i);
  int32_t* r_audio = reinterpret_cast<int32_t*>(tmp + sz_h + 6 * sz_i);
  float* r_pos = reinterpret_cast<float*>(tmp + sz_h + 7 * sz_i);
  int32_t* d_n = reinterpret_cast<int32_t*>(tmp + sz_h + 7 * sz_i + sz_p);
  h3_status rc = H3_OK;
  h3_layout_t red = nullptr;
  do {
    int hn[4] = {0, 0, 0, 0};
    if (S > 0) {
      if (launch_pair_heads(full, target, head, st) != cudaSuccess ||
          launch_reduce_build(full, head, r_tags, r_tidx, r_pos, r_src_a, r_src_b, r_video,
                              r_text, r_audio, d_n, st) != cudaSuccess ||
          cudaMemcpyAsync(hn, d_n, 16, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
          cudaStreamSynchronize(st) != cudaSuccess) {
        rc = H3_ERR_CUDA;
        break;
      }
    }
    h3_layout_desc desc{hn[0], full->n_t, hn[1], hn[3], hn[2], r_pos, r_tags, r_tidx, r_video,
                        r_audio, r_text};
    if ((rc = h3_layout_prepare(dims, &desc, stream, &red)) != H3_OK) break;
    const size_t map_b = (size_t)(red->n_valid > 0 ? red->n_valid : 1) * sizeof(int2);
    if (cudaMalloc(&red->extra, map_b) != cudaSuccess) { rc = H3_ERR_CUDA; break; }
    red->red_map = static_cast<int2*>(red->extra);
    red->red_parent_S = full->S;
    red->red_parent_V = full->n_valid;
    if (launch_reduce_map(red->S, r_tags, r_src_a, r_src_b, red->c_of_row, full->c_of_row,
                          red->red_map, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
      rc = H3_ERR_CUDA;
      break;
    }
  } while (0);
  cudaFree(tmp);
  if (rc != H3_OK) {
    h3_layout_destroy(red);
    return rc;
  }
  *out = red;
  return H3_OK;
}

size_t h3_stack_reduced_workspace_size(const h3_dims* dims, h3_layout_t full,
                                       h3_layout_t reduced, int B) {
  if (check_dims(dims) != H3_OK || check_batch(full, B) != H3_OK || !reduced) return 0;
  return ws_parts(*dims, B, full->S, nullptr, nullptr) +
         align256((size_t)B * reduced->n_valid * dims->hidden * 4);
}

h3_status h3_stack_forward_reduced(const h3_dims* dims, const h3_block_weights* weights,
                                   int n_blocks, h3_layout_t full, h3_layout_t reduced, int r0,
                                   int r1, const float* tmod, void* x, int B, void* ws,
                                   size_t ws_bytes, h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!full || !reduced || B < 0 || n_blocks < 0 || r0 < 0 || r1 < 0 || !tmod || !x || !ws ||
      (n_blocks > 0 && !weights))
    return H3_ERR_ARG;
  H3_TRY(check_batch(full, B));
  if (!reduced->red_map || reduced->red_parent_S != full->S ||
      reduced->red_parent_V != full->n_valid)
    return H3_ERR_LAYOUT;
  for (int i = 0; i < n_blocks; ++i) H3_TRY(check_weights(&weights[i]));
  if (!aligned16(tmod) || !aligned16(x) || !aligned16(ws)) return H3_ERR_ALIGN;
  if (ws_bytes < h3_stack_reduced_workspace_size(dims, full, reduced, B)) return H3_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  const h3_dims& d = *dims;
  const int V = full->n_valid, Vr = reduced->n_valid, H = d.hidden;
  Workspace w, wr;
  ws_parts(d, B, full->S, &w, ws);
  ws_parts(d, B, reduced->S, &wr, ws);  // the reduced blocks' scratch, below w.xc
  float* xc = static_cast<float*>(w.xc);
  float* xr = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                       ws_parts(d, B, full->S, nullptr, nullptr));
  const int a = r0 < n_blocks ? r0 : n_blocks;
  const int e = r1 < n_blocks ? r1 : n_blocks;
  H3_CUDA(launch_permute_rows_convert(B, V, full->S, H, full->perm, x, xc, true, st));
  for (int i = 0; i < a; ++i)
    H3_TRY(run_block(d, weights[i], full->compact_view(), tmod, xc, true, B, w, st));
  if (a < e) {
    H3_CUDA(launch_merge(B, Vr, V, H, reduced->red_map, xc, xr, st));
    for (int i = a; i < e; ++i)
      H3_TRY(run_block(d, weights[i], reduced->compact_view(), tmod, xr, true, B, wr, st));
    H3_CUDA(launch_restore(B, Vr, V, H, reduced->red_map, xr, xc, st));
  }
  for (int i = (r1 > a ? r1 : a); i < n_blocks; ++i)
    H3_TRY(run_block(d, weights[i], full->compact_view(), tmod, xc, true, B, w, st));
  H3_CUDA(launch_permute_rows_convert(B, V, full->S, H, full->perm, xc, x, false, st));
  return H3_OK;
}

}  // extern "C"

// ---- sequence-parallel block: exchanges fused into the producing kernels ----

namespace {

h3_status check_peers(const h3_dims* dims, const h3_ulysses_peers* p, int S_full) {
  if (!p) return H3_ERR_ARG;
  const int P = p->n_ranks;
  if (P < 1 || P > H3_MAX_RANKS || H3_MAX_RANKS > kMaxDst || p->rank < 0 || p->rank >= P)
    return H3_ERR_ARG;
  if (dims->heads % P != 0 || S_full % P != 0) return H3_ERR_SHAPE;
  return H3_OK;
}

}  // namespace

extern "C" {

h3_status h3_qkv_rope_to_heads(const h3_dims* dims, h3_layout_t chunk, const void* h,
                               const void* w_qkv, const void* q_norm, const void* k_norm,
                               const h3_ulysses_peers* peers, h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!chunk || !h || !w_qkv || !q_norm || !k_norm || !peers) return H3_ERR_ARG;
  H3_TRY(check_batch(chunk, 1));
  const int P = peers->n_ranks;
  if (P < 1 || P > H3_MAX_RANKS) return H3_ERR_ARG;
  const long long S_full = (long long)chunk->S * P;
  if (S_full > kMaxRows) return H3_ERR_SHAPE;
  H3_TRY(check_peers(dims, peers, (int)S_full));
  if (!aligned16(h) || !aligned16(w_qkv) || !aligned16(q_norm) || !aligned16(k_norm))
    return H3_ERR_ALIGN;
  for (int j = 0; j < P; ++j) {
    if (!peers->q[j] || !peers->k[j] || !peers->v[j]) return H3_ERR_ARG;
    if (!aligned16(peers->q[j]) || !aligned16(peers->k[j]) || !aligned16(peers->v[j]))
      return H3_ERR_ALIGN;
  }
  GemmEpiArgs e;
  e.L = chunk->view();
  e.B = 1;
  e.NH = dims->heads;
  for (int j = 0; j < P; ++j) {
    e.heads.q[j] = peers->q[j];
    e.heads.k[j] = peers->k[j];
    e.heads.v[j] = peers->v[j];
  }
  e.heads.heads_per_dst = dims->heads / P;
  e.heads.dst_rows = (int)S_full;
  e.heads.row_offset = peers->rank * chunk->S;
  e.q_norm = q_norm;
  e.k_norm = k_norm;
  e.qk_eps = dims->qk_norm_eps;
  H3_CUDA(launch_gemm(EPI_QKV, chunk->S, 3 * dims->heads * dims->head_dim, dims->hidden, h, w_qkv,
                      e, as_stream(stream)));
  return H3_OK;
}

h3_status h3_attention_to_rows(const h3_dims* dims, h3_layout_t full, const void* q,
                               const void* k, const void* v, const h3_ulysses_peers* peers,
                               h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!full || !q || !k || !v || !peers) return H3_ERR_ARG;
  H3_TRY(check_batch(full, 1));
  H3_TRY(check_peers(dims, peers, full->S));
  const int P = peers->n_ranks;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return H3_ERR_ALIGN;
  for (int j = 0; j < P; ++j) {
    if (!peers->o[j]) return H3_ERR_ARG;
    if (!aligned16(peers->o[j])) return H3_ERR_ALIGN;
  }
  const int NHl = dims->heads / P;
  RowMap m;
  for (int j = 0; j < P; ++j) m.o[j] = peers->o[j];
  m.rows_per_dst = full->S / P;
  m.row_heads = dims->heads;
  m.head_offset = peers->rank * NHl;
  if (full->S == 0) return H3_OK;
  H3_CUDA(launch_attention(full->view(), 1, NHl, q, k, v, m, as_stream(stream)));
  return H3_OK;
}

}  // extern "C"

// ---- 8-bit QKV and W1 || W3 GEMM inputs ----

extern "C" {

h3_status h3_quantize_e4m3_rows(const void* w, int rows, int K, void* codes, float* scales,
                                h3_stream_t stream) {
  if (rows < 0 || K <= 0 || (rows > 0 && (!w || !codes || !scales))) return H3_ERR_ARG;
  if (K % 16 != 0) return H3_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(codes) || !aligned16(scales)) return H3_ERR_ALIGN;
  H3_CUDA(launch_quantize_rows_e4m3(rows, K, w, codes, scales, as_stream(stream)));
  return H3_OK;
}

h3_status h3_norm_modulate_e4m3(const h3_dims* dims, h3_layout_t L, int B, int which,
                                const void* x, const float* ada_table, const float* tmod,
                                void* codes, float* scales, h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || (which != 0 && which != 1) || !x || !ada_table || !tmod || !codes ||
      !scales)
    return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (!aligned16(x) || !aligned16(ada_table) || !aligned16(tmod) || !aligned16(codes) ||
      !aligned16(scales))
    return H3_ERR_ALIGN;
  const int c0 = which == 0 ? 0 : 3;
  H3_CUDA(launch_norm_modulate_e4m3(L->view(), B, dims->hidden, c0, c0 + 1, dims->norm_eps, x,
                                    false, ada_table, tmod, codes, scales, as_stream(stream)));
  return H3_OK;
}

h3_status h3_qkv_rope_e4m3(const h3_dims* dims, h3_layout_t L, int B, const void* h_codes,
                           const float* h_scales, const void* w_codes, const float* w_scales,
                           const void* q_norm, const void* k_norm, void* q, void* k, void* v,
                           h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || !h_codes || !h_scales || !w_codes || !w_scales || !q_norm || !k_norm ||
      !q || !k || !v)
    return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (!aligned16(h_codes) || !aligned16(h_scales) || !aligned16(w_codes) ||
      !aligned16(w_scales) || !aligned16(q_norm) || !aligned16(k_norm) || !aligned16(q) ||
      !aligned16(k) || !aligned16(v))
    return H3_ERR_ALIGN;
  if (dims->hidden % 128 != 0) return H3_ERR_SHAPE;
  GemmEpiArgs e;
  e.L = L->view();
  e.B = B;
  e.NH = dims->heads;
  e.heads = plain_head_map(q, k, v, dims->heads, L->S);
  e.q_norm = q_norm;
  e.k_norm = k_norm;
  e.qk_eps = dims->qk_norm_eps;
  e.a_scale = h_scales;
  e.b_scale = w_scales;
  H3_CUDA(launch_gemm_e4m3(EPI_QKV, B * L->S, 3 * dims->heads * dims->head_dim, dims->hidden,
                           h_codes, w_codes, e, as_stream(stream)));
  return H3_OK;
}

h3_status h3_ffn_up_e4m3(const h3_dims* dims, h3_layout_t L, int B, const void* h2_codes,
                         const float* h2_scales, const void* w_codes, const float* w_scales,
                         void* g, h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || !h2_codes || !h2_scales || !w_codes || !w_scales || !g) return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (!aligned16(h2_codes) || !aligned16(h2_scales) || !aligned16(w_codes) ||
      !aligned16(w_scales) || !aligned16(g))
    return H3_ERR_ALIGN;
  if (dims->hidden % 128 != 0) return H3_ERR_SHAPE;
  GemmEpiArgs sg;
  sg.L = L->view();
  sg.out = g;
  sg.a_scale = h2_scales;
  sg.b_scale = w_scales;
  H3_CUDA(launch_gemm_e4m3(EPI_SWIGLU, B * L->S, 2 * dims->ffn, dims->hidden, h2_codes, w_codes,
                           sg, as_stream(stream)));
  return H3_OK;
}

size_t h3_workspace_size_e4m3(const h3_dims* dims, int B, int S) {
  if (check_dims(dims) != H3_OK || B < 0 || S < 0) return 0;
  const size_t rows = (size_t)B * S;
  return ws_parts(*dims, B, S, nullptr, nullptr) + align256(rows * e4m3_row_bytes(*dims)) +
         align256(rows * 4);
}

}  // extern "C"

namespace {

h3_status check_w8(const h3_dims* dims, const h3_block_weights_e4m3* w8) {
  if (!w8 || !w8->w_qkv_codes || !w8->w_qkv_scales || !w8->w13_codes || !w8->w13_scales)
    return H3_ERR_ARG;
  if ((w8->w_o_codes && !w8->w_o_scales) || (w8->w2_codes && !w8->w2_scales)) return H3_ERR_ARG;
  if (!aligned16(w8->w_qkv_codes) || !aligned16(w8->w_qkv_scales) || !aligned16(w8->w13_codes) ||
      !aligned16(w8->w13_scales) || !aligned16(w8->w_o_codes) || !aligned16(w8->w_o_scales) ||
      !aligned16(w8->w2_codes) || !aligned16(w8->w2_scales))
    return H3_ERR_ALIGN;
  if (dims->hidden % 128 != 0) return H3_ERR_SHAPE;
  if ((w8->w_o_codes || w8->w2_codes) && dims->hidden % 256 != 0) return H3_ERR_SHAPE;
  return H3_OK;
}

E4m3Operands e4m3_operands(const h3_dims& d, int B, int S, void* ws, size_t base,
                           const h3_block_weights_e4m3* w8) {
  E4m3Operands q8;
  q8.w = w8;
  q8.codes = static_cast<uint8_t*>(ws) + base;
  q8.scales = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + base +
                                       align256((size_t)B * S * e4m3_row_bytes(d)));
  return q8;
}

h3_status resid_e4m3(const h3_dims* dims, h3_layout_t L, int B, int K, int gate_chunk,
                     const void* a_codes, const float* a_scales, const void* w_codes,
                     const float* w_scales, const float* ada_table, const float* tmod, void* x,
                     h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || !a_codes || !a_scales || !w_codes || !w_scales || !ada_table || !tmod || !x)
    return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(ada_table) || !aligned16(tmod) || !aligned16(x))
    return H3_ERR_ALIGN;
  if (dims->hidden % 256 != 0 || K % 128 != 0) return H3_ERR_SHAPE;
  GemmEpiArgs r;
  r.L = L->view();
  r.B = B;
  r.x = x;
  r.table = ada_table;
  r.tmod = tmod;
  r.gate_chunk = gate_chunk;
  r.a_scale = a_scales;
  r.b_scale = w_scales;
  H3_CUDA(launch_gemm_e4m3(EPI_RESID, B * L->S, dims->hidden, K, a_codes, w_codes, r,
                           as_stream(stream)));
  return H3_OK;
}

}  // namespace

extern "C" {

h3_status h3_out_residual_e4m3(const h3_dims* dims, h3_layout_t L, int B, const void* o_codes,
                               const float* o_scales, const void* w_codes, const float* w_scales,
                               const float* ada_table, const float* tmod, void* x,
                               h3_stream_t stream) {
  if (!dims) return H3_ERR_ARG;
  return resid_e4m3(dims, L, B, dims->heads * dims->head_dim, 2, o_codes, o_scales, w_codes,
                    w_scales, ada_table, tmod, x, stream);
}

h3_status h3_ffn_down_residual_e4m3(const h3_dims* dims, h3_layout_t L, int B,
                                    const void* g_codes, const float* g_scales,
                                    const void* w_codes, const float* w_scales,
                                    const float* ada_table, const float* tmod, void* x,
                                    h3_stream_t stream) {
  if (!dims) return H3_ERR_ARG;
  return resid_e4m3(dims, L, B, dims->ffn, 5, g_codes, g_scales, w_codes, w_scales, ada_table,
                    tmod, x, stream);
}

h3_status h3_block_forward_e4m3(const h3_dims* dims, const h3_block_weights* weights,
                                const h3_block_weights_e4m3* w8, h3_layout_t L,
                                const float* tmod, void* x, int B, void* ws, size_t ws_bytes,
                                h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || !tmod || !x || !ws || !w8) return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  H3_TRY(check_weights(weights));
  H3_TRY(check_w8(dims, w8));
  if (!aligned16(tmod) || !aligned16(x) || !aligned16(ws)) return H3_ERR_ALIGN;
  if (ws_bytes < h3_workspace_size_e4m3(dims, B, L->S)) return H3_ERR_WORKSPACE;
  Workspace w;
  const size_t base = ws_parts(*dims, B, L->S, &w, ws);
  const E4m3Operands q8 = e4m3_operands(*dims, B, L->S, ws, base, w8);
  return run_block(*dims, *weights, L->view(), tmod, x, false, B, w, as_stream(stream), q8);
}

h3_status h3_stack_forward_e4m3(const h3_dims* dims, const h3_block_weights* weights,
                                const h3_block_weights_e4m3* w8, int n_blocks, h3_layout_t L,
                                const float* tmod, void* x, int B, void* ws, size_t ws_bytes,
                                h3_stream_t stream) {
  H3_TRY(check_dims(dims));
  if (!L || B < 0 || n_blocks < 0 || !tmod || !x || !ws || (n_blocks > 0 && (!weights || !w8)))
    return H3_ERR_ARG;
  H3_TRY(check_batch(L, B));
  for (int i = 0; i < n_blocks; ++i) {
    H3_TRY(check_weights(&weights[i]));
    H3_TRY(check_w8(dims, &w8[i]));
  }
  if (!aligned16(tmod) || !aligned16(x) || !aligned16(ws)) return H3_ERR_ALIGN;
  if (ws_bytes < h3_workspace_size_e4m3(dims, B, L->S)) return H3_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  Workspace w;
  const size_t base = ws_parts(*dims, B, L->S, &w, ws);
  // as h3_stack_forward: the valid rows in an fp32 residual stream
  const int V = L->n_valid;
  H3_CUDA(launch_permute_rows_convert(B, V, L->S, dims->hidden, L->perm, x, w.xc, true, st));
  for (int i = 0; i < n_blocks; ++i) {
    const E4m3Operands q8 = e4m3_operands(*dims, B, L->S, ws, base, &w8[i]);
    H3_TRY(run_block(*dims, weights[i], L->compact_view(), tmod, w.xc, true, B, w, st, q8));
  }
  H3_CUDA(launch_permute_rows_convert(B, V, L->S, dims->hidden, L->perm, w.xc, x, false, st));
  return H3_OK;
}

}  // extern "C"
