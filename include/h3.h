/*
 * h3.h — C ABI of the B200 (sm_100a) MiniMax-H3 transformer-block library.
 *
 * What the library computes is defined on the page "MiniMaxH3Transformer3DModel"
 * (diffusers v0.43.0 docs): one stack of blocks runs over a single packed 1-D
 * sequence of text, conditioning, audio and target-video rows; attention is
 * full self-attention over that sequence; the per-row modality tag selects the
 * AdaLN modulation; rows tagged -1 (padding) form their own attention document
 * under a boolean mask; the caller builds the packing and passes the layout
 * (the (t, h, w) grid, per-row tags, per-row timestep indices and the three
 * index tensors) separately from the latents (section "MiniMaxH3Transformer3DModel",
 * constructor parameters and `forward` arguments). The block structure follows
 * the same page's constructor parameters and the page "MiniMax H3 Inference
 * Engine voor Mac computers", sections "Exacte DiT fusions" (gated attention
 * residual feeding the MLP's AdaLN over a bf16 residual stream), "Checkpoint
 * layout en media pipeline" (QKV rows interleaved per head, fused
 * QK-norm + RoPE) and "Profiling en diagnostische pads" (fc1 -> SwiGLU -> fc2).
 *
 * Conventions shared by every entry point:
 *  - Ownership: the caller owns every buffer. Pointers named in structs and
 *    arguments are DEVICE pointers unless the name ends in `_host`. The library
 *    allocates device memory only in h3_layout_prepare (small per-layout tables,
 *    released by h3_layout_destroy).
 *  - Types: "bf16" buffers hold IEEE bfloat16 values (2 bytes each); "f32"
 *    buffers hold float; index buffers hold int32_t.
 *  - Matrices are row-major [out, in] (K-major for the tensor cores).
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *    default stream). Every call except h3_layout_prepare, h3_layout_error and
 *    h3_layout_export only enqueues work and returns; argument, shape and
 *    alignment errors are returned synchronously before anything is launched.
 *  - Alignment: every device pointer must be 16-byte aligned.
 *  - Shapes: head_dim == 128; hidden % 256 == 0 and <= 6144; heads even;
 *    ffn % 128 == 0; rope_freq_dim == 16; freq_dim, time_hidden and
 *    time_embed_dim % 4 == 0. S (rows) is any value in [0, 524288] (the
 *    attention kernel keeps the list of 128-row key tiles it visits in shared
 *    memory); h3_layout_prepare returns H3_ERR_SHAPE for a larger S. B (batch
 *    elements) is at most 65535 with B * S < 2^31; the batched calls return
 *    H3_ERR_SHAPE beyond.
 *  - Batch: B >= 1 elements share one layout; each element is its own attention
 *    document set (the page's "pure replication axis").
 *  - Asynchronous failures: every wait inside a kernel is bounded (about 2 s).
 *    A wait that runs out records an error in the layout's device error word;
 *    read it with h3_layout_error after the stream has been synchronised.
 */
#ifndef H3_H
#define H3_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define H3_API __attribute__((visibility("default")))
#else
#define H3_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  H3_OK = 0,
  H3_ERR_ARG = -1,       /* null pointer, negative size, unknown option */
  H3_ERR_SHAPE = -2,     /* dimensions the kernels do not support */
  H3_ERR_ALIGN = -3,     /* pointer not 16-byte aligned */
  H3_ERR_LAYOUT = -4,    /* layout tensors inconsistent (see h3_layout_prepare) */
  H3_ERR_WORKSPACE = -5, /* workspace smaller than h3_workspace_size */
  H3_ERR_CUDA = -6,      /* a CUDA runtime/driver call failed */
  H3_ERR_TIMEOUT = -7    /* a bounded in-kernel wait ran out */
} h3_status;

typedef void* h3_stream_t;

/* Block dimensions: the constructor parameters of the transformer
 * (num_attention_heads, attention_head_dim, hidden_size, ffn_dim,
 * time_embed_dim, time_embed_hidden_dim, freq_dim, rope_freq_dim, rope_theta,
 * norm_eps, qk_norm_eps). n_modalities is the number of AdaLN table rows (3:
 * video 0, text 1, audio 2). */
typedef struct {
  int hidden, heads, head_dim, ffn, time_embed_dim, time_hidden, freq_dim, rope_freq_dim,
      n_modalities;
  float rope_theta, norm_eps, qk_norm_eps;
} h3_dims;

/* The packed layout, as the `forward` arguments describe it. All DEVICE
 * pointers; read only during h3_layout_prepare (the library keeps copies).
 *   pos       [S, 3] f32  (t, h, w) rotary coordinates; fp32 so that halved
 *                         (fractional) spatial coordinates are representable
 *   tags      [S]    i32  0 video, 1 text, 2 audio, -1 padding
 *   t_idx     [S]    i32  index of the row's value in `timestep` (0 <= t_idx < n_t)
 *   video_idx [n_video], audio_idx [n_audio], text_idx [n_text]  i32:
 *             packed-row positions of the rows of each modality, in the order of
 *             that modality's latent rows. */
typedef struct {
  int S, n_t, n_video, n_audio, n_text;
  const float* pos;
  const int32_t* tags;
  const int32_t* t_idx;
  const int32_t* video_idx;
  const int32_t* audio_idx;
  const int32_t* text_idx;
} h3_layout_desc;

typedef struct h3_layout* h3_layout_t;

/* One block's parameters (DEVICE pointers, [out, in] row-major):
 *   w_qkv     [3*NH*D, H] bf16, rows interleaved per head: row n*3D + {0, D, 2D} + d
 *             holds q / k / v channel d of head n
 *   q_norm, k_norm [D] bf16  per-head RMSNorm weights (shared by all heads)
 *   w_o       [H, NH*D] bf16
 *   w13       [2F, H] bf16, W1 and W3 interleaved in 128-row blocks:
 *             rows [256j, 256j+128) = W1 rows [128j, 128j+128),
 *             rows [256j+128, 256j+256) = W3 rows [128j, 128j+128)
 *   w2        [H, F] bf16
 *   ada_table [n_modalities, 6, H] f32: per-modality AdaLN rows in the order
 *             (shift1, scale1, gate1, shift2, scale2, gate2) */
typedef struct {
  const void* w_qkv;
  const void* q_norm;
  const void* k_norm;
  const void* w_o;
  const void* w13;
  const void* w2;
  const float* ada_table;
} h3_block_weights;

/* Human-readable name of a status code (static string). */
H3_API const char* h3_status_string(h3_status status);

/* Library ABI version (increases when a signature changes). */
H3_API int h3_abi_version(void);

/* a0 — validate a packed layout and build its device tables: per-128-row tile
 * classes (all valid / all padding / mixed), the valid-key bitmask of each
 * tile, the compaction order (valid rows first, then padding rows, each in
 * packed order), the per-row source of the packing, and the per-row RoPE
 * cos/sin table (inv_freq[j] = rope_theta^(-j/rope_freq_dim)).
 * Validation (all on the GPU): tags in {-1,0,1,2}; every t_idx in [0, n_t);
 * positions finite; every index tensor in range, duplicate-free, pointing
 * only at rows of its modality and as long as the number of such rows.
 * Synchronises `stream` once. On H3_ERR_LAYOUT nothing is returned in *out.
 * The layout object owns a device error word used by the later calls. */
H3_API h3_status h3_layout_prepare(const h3_dims* dims, const h3_layout_desc* desc, h3_stream_t stream,
                            h3_layout_t* out);

/* Release a layout (synchronises the device first). NULL is ignored. */
H3_API void h3_layout_destroy(h3_layout_t layout);

/* Read and clear the layout's device error word (synchronises the device):
 * H3_OK, or H3_ERR_TIMEOUT if a bounded in-kernel wait ran out. */
H3_API h3_status h3_layout_error(h3_layout_t layout);

/* Copy the layout's tables to HOST buffers (any may be NULL):
 * perm_host [S] compaction order, tile_class_host [ceil(S/128)] (0 valid,
 * 1 padding, 2 mixed), n_valid_host [1]. Synchronous. */
H3_API h3_status h3_layout_export(h3_layout_t layout, int32_t* perm_host, uint8_t* tile_class_host,
                           int32_t* n_valid_host);

/* Bytes of device workspace h3_block_forward / h3_stack_forward need for B
 * batch elements of S rows. 0 on invalid dims. */
H3_API size_t h3_workspace_size(const h3_dims* dims, int B, int S);

/* a1 — scatter per-modality rows into the packed stream (bit-exact copies):
 * x_packed[b, video_idx[i]] = video[b, i] (same for audio and text); padding
 * rows are zero-filled. Rows are `row_elems` bf16 values wide; video [B, n_video,
 * row_elems], audio [B, n_audio, row_elems], text [B, n_text, row_elems],
 * x_packed [B, S, row_elems]. row_elems % 8 == 0. */
H3_API h3_status h3_pack_rows(h3_layout_t layout, int B, int row_elems, const void* video,
                       const void* audio, const void* text, void* x_packed, h3_stream_t stream);

/* a1 — gather packed rows back to per-modality buffers (bit-exact), in index
 * order (the page's `forward` returns velocities in the row order of
 * video_indices and audio_indices). Any output may be NULL to skip it. */
H3_API h3_status h3_unpack_rows(h3_layout_t layout, int B, int row_elems, const void* x_packed,
                         void* video, void* audio, void* text, h3_stream_t stream);

/* a2 — timestep embedding and shared AdaLN projection, fp32 throughout:
 * tmod[n, 6H] = W_proj . SiLU(W_t2 . SiLU(W_t1 . [cos(t f_i), sin(t f_i)])),
 * f_i = 10^4^(-i/(freq_dim/2)); timesteps unscaled in [0, 1] (constructor
 * parameters freq_dim, time_embed_hidden_dim, time_embed_dim).
 *   t [n_t] f32, w_t1 [time_hidden, freq_dim], w_t2 [time_embed_dim, time_hidden],
 *   w_proj [6H, time_embed_dim] (all f32), tmod [n_t, 6, H] f32.
 * ws must hold h3_timestep_workspace_size(dims, n_t) bytes (16-byte aligned).
 * From 65 timesteps on (when the widths allow) the three GEMMs run on the
 * tensor cores over three-way bf16 splits of both fp32 operands, whose copies
 * live in ws: the workspace then also holds, for the largest GEMM, n_t x 6K
 * and N x 6K bf16 values (about 1.3 GB at n_t = 8192 and the full widths).
 * The split form's GEMMs have bounded waits like every kernel here; one that
 * runs out records a timeout in a library-owned error word (one per GPU),
 * which h3_timestep_error reads. */
H3_API size_t h3_timestep_workspace_size(const h3_dims* dims, int n_t);
H3_API h3_status h3_timestep_modulation(const h3_dims* dims, int n_t, const float* t, const float* w_t1,
                                 const float* w_t2, const float* w_proj, float* tmod, void* ws,
                                 size_t ws_bytes, h3_stream_t stream);

/* Read and clear the error word of h3_timestep_modulation's split form on the
 * current device (synchronises the device): H3_OK, or H3_ERR_TIMEOUT if one of
 * its bounded in-kernel waits ran out since the last read. */
H3_API h3_status h3_timestep_error(void);

/* Same result as h3_timestep_modulation, for callers that cannot allocate device
 * memory (a serving loop whose device memory is reserved up front by its own
 * pool, or a latency-critical frame callback where allocation is forbidden).
 * The pages have no counterpart to this entry point; it exists for those
 * callers. It allocates nothing: its scratch is a fixed 4 MiB device array
 * inside the library (one per GPU that loads the library, held until exit).
 * It always uses the CUDA-core form of the GEMMs; n_t is accepted while that
 * form's scratch fits in 4 MiB (n_t <= 126 at the full constructor widths);
 * larger n_t returns H3_ERR_WORKSPACE before any work is queued. All calls on a device share the array: calls whose work
 * overlaps on the GPU race (order them on one stream or with events). Nothing in
 * the array needs to start at zero. The first call on a device looks up the
 * array's address; make it before any stream capture. The address is looked
 * up again if the device's context has been replaced since (after a
 * cudaDeviceReset). Arguments are checked like h3_timestep_modulation's: the
 * same bad input gives the same status. */
H3_API h3_status h3_timestep_modulation_noalloc(const h3_dims* dims, int n_t, const float* t,
                                                const float* w_t1, const float* w_t2,
                                                const float* w_proj, float* tmod,
                                                h3_stream_t stream);

/* ---- single steps of the block (each also runs inside h3_block_forward) ---- */

/* a3 / a7 — h = LayerNorm(x) * (1 + scale) + shift (no affine, biased
 * variance, eps = norm_eps), with shift/scale of row r = ada_table[tag(r)][c]
 * + tmod[t_idx(r)][c] for c = (shift, scale) = (0, 1) when which == 0 and
 * (3, 4) when which == 1. x, h [B, S, H] bf16; padding rows of h are zero. */
H3_API h3_status h3_norm_modulate(const h3_dims* dims, h3_layout_t layout, int B, int which,
                           const void* x, const float* ada_table, const float* tmod, void* h,
                           h3_stream_t stream);

/* a4 — qkv = h . W_qkv^T on tcgen05; per head: q, k <- RMSNorm(., q_norm/k_norm,
 * qk_norm_eps), then RoPE on channels [0, 96): pair (32a + j, 32a + j + 16),
 * a = (t, h, w), angle pos[r][a] * inv_freq[j]. q, k, v [B, NH, S, D] bf16. */
H3_API h3_status h3_qkv_rope(const h3_dims* dims, h3_layout_t layout, int B, const void* h,
                      const void* w_qkv, const void* q_norm, const void* k_norm, void* q,
                      void* k, void* v, h3_stream_t stream);

/* a5 — o = softmax(q k^T / sqrt(D)) v per head over the row's document
 * (valid rows attend valid rows). Output rows of padding queries carry no
 * result: rows of 128-row tiles that hold only padding are written as zeros;
 * padding rows inside mixed tiles hold finite values that every later step
 * ignores (they are never read back into x). q, k, v [B, NH, S, D] bf16 ->
 * o [B, S, NH*D] bf16. Only head_dim (128) and heads (any count >= 1) of dims
 * are used here, so a caller may run it on a subset of the heads. */
H3_API h3_status h3_attention(const h3_dims* dims, h3_layout_t layout, int B, const void* q,
                       const void* k, const void* v, void* o, h3_stream_t stream);

/* a6 — x += gate1 * (o . W_o^T) in place, gate1 = ada_table[tag][2] + tmod[t_idx][2];
 * padding rows of x are left untouched. o [B, S, NH*D] bf16, x [B, S, H] bf16. */
H3_API h3_status h3_out_residual(const h3_dims* dims, h3_layout_t layout, int B, const void* o,
                          const void* w_o, const float* ada_table, const float* tmod, void* x,
                          h3_stream_t stream);

/* a8 — g = SiLU(h2 . W1^T) * (h2 . W3^T) from the block-interleaved w13.
 * h2 [B, S, H] bf16 -> g [B, S, F] bf16. */
H3_API h3_status h3_ffn_up(const h3_dims* dims, h3_layout_t layout, int B, const void* h2,
                    const void* w13, void* g, h3_stream_t stream);

/* a9 — x += gate2 * (g . W2^T) in place, gate2 = ada_table[tag][5] + tmod[t_idx][5];
 * padding rows untouched. g [B, S, F] bf16, x [B, S, H] bf16. */
H3_API h3_status h3_ffn_down_residual(const h3_dims* dims, h3_layout_t layout, int B, const void* g,
                               const void* w2, const float* ada_table, const float* tmod,
                               void* x, h3_stream_t stream);

/* ---- the block and the stack ---- */

/* One block, in place on x [B, S, H] bf16: a3, a4, a5, a6, a7, a8, a9 with
 * tmod [n_t, 6, H] f32 (from h3_timestep_modulation). Padding rows of x are
 * returned bit-identical. ws: h3_workspace_size(dims, B, S) bytes. */
H3_API h3_status h3_block_forward(const h3_dims* dims, const h3_block_weights* weights,
                           h3_layout_t layout, const float* tmod, void* x, int B, void* ws,
                           size_t ws_bytes, h3_stream_t stream);

/* n_blocks blocks (weights: HOST array of n_blocks structs holding device
 * pointers) sharing one tmod, in place on x [B, S, H] bf16. Valid rows are
 * gathered once into a compact [B, V, H] f32 stream (padding rows never reach a
 * valid row's result, so the blocks then run with no mask); the residual stream
 * stays f32 across the blocks and is rounded to bf16 once when scattered back
 * at the end; padding rows of x are untouched. ws: h3_workspace_size(dims, B, S)
 * bytes. */
H3_API h3_status h3_stack_forward(const h3_dims* dims, const h3_block_weights* weights, int n_blocks,
                           h3_layout_t layout, const float* tmod, void* x, int B, void* ws,
                           size_t ws_bytes, h3_stream_t stream);

/* ---- sequence-parallel block: the head <-> sequence exchange fused into the
 * kernels that produce the exchanged tensors ---- */

/* "MiniMaxH3Transformer3DModel" page, `forward`: each batch element is one
 * attention document over one packed sequence, so one long sequence is split
 * across P ranks by rows. Every step but attention is row-local; attention is
 * independent per head. Rank r holds rows [r S/P, (r + 1) S/P) (its chunk) and,
 * for attention, heads [r NH/P, (r + 1) NH/P) of every row.
 *
 * The two exchanges are stores from the producing kernels into the receiving
 * rank's buffer: plain global stores, so a buffer may be another GPU's memory
 * mapped into this process (peer access over NVLink) or, with every rank in one
 * process, a buffer of this GPU. These calls only enqueue; the caller orders
 * them across ranks (all ranks' h3_qkv_rope_to_heads complete before any
 * rank's h3_attention_to_rows reads its q, k, v, and all ranks'
 * h3_attention_to_rows complete before any rank reads its o). */
#define H3_MAX_RANKS 8
typedef struct {
  int n_ranks; /* P, 1 .. H3_MAX_RANKS; S % P == 0 and heads % P == 0 */
  int rank;    /* this rank, 0 .. P - 1 */
  void* q[H3_MAX_RANKS]; /* rank j's q [heads / P, S, 128] bf16 (likewise k, v) */
  void* k[H3_MAX_RANKS];
  void* v[H3_MAX_RANKS];
  void* o[H3_MAX_RANKS]; /* rank j's o [S / P, heads * 128] bf16 */
} h3_ulysses_peers;

/* h3_qkv_rope (B = 1) on this rank's chunk: `chunk` is the layout of its S / P
 * rows (their positions drive RoPE), h [S/P, H]. Head n of chunk row s goes
 * to rank n / (heads / P): q[..][n % (heads / P)][rank * S / P + s][:], and
 * likewise k, v. */
H3_API h3_status h3_qkv_rope_to_heads(const h3_dims* dims, h3_layout_t chunk, const void* h,
                                      const void* w_qkv, const void* q_norm, const void* k_norm,
                                      const h3_ulysses_peers* peers, h3_stream_t stream);

/* h3_attention (B = 1) of this rank's heads / P heads over every row: `full` is
 * the layout of all S rows, q, k, v [heads / P, S, 128] this rank's buffers
 * (dims->heads is the total head count). The output of row s, local head n
 * goes to rank s / (S / P): o[..][s % (S / P)][(rank * heads / P + n) * 128 ..]. */
H3_API h3_status h3_attention_to_rows(const h3_dims* dims, h3_layout_t full, const void* q,
                                      const void* k, const void* v,
                                      const h3_ulysses_peers* peers, h3_stream_t stream);

/* ---- 8-bit (e4m3) inputs for the QKV and W1 || W3 GEMMs ---- */

/* "MiniMax H3 Inference Engine voor Mac computers", sections "Profiling en
 * diagnostische pads" and "Sampler en DiT controls": an 8-bit MLP and 8-bit QKV
 * projections with one activation scale per row. Here (reading): e4m3 codes
 * for both operands of the QKV and W1 || W3 GEMMs (tcgen05 kind::f8f6f4), one
 * scale per activation row (its largest |h| / 448, computed by the norm kernel)
 * and one per weight row; the product of the scales is applied to the fp32 dot
 * product of the codes. The O and W2 GEMMs and everything else stay as in
 * h3_block_forward. */

/* Weight rows [rows, K] bf16 -> e4m3 codes [rows, K] (one byte each) and
 * scales [rows] f32: scale = max|w| / 448 (1 for an all-zero row), code =
 * e4m3(w / scale), round to nearest even, saturating. K % 16 == 0. Enqueues. */
H3_API h3_status h3_quantize_e4m3_rows(const void* w, int rows, int K, void* codes, float* scales,
                                       h3_stream_t stream);

/* The 8-bit operands of one block (DEVICE pointers, from h3_quantize_e4m3_rows
 * applied to the block's w_qkv [3*NH*D, H] and w13 [2F, H], and optionally to
 * w_o [H, NH*D] and w2 [H, F]). With w_o_codes (w2_codes) null the output
 * projection (FFN down projection) stays bf16; with them set, its input rows
 * (o, g: bf16 as stored) are quantized per row first, one scale per row as for
 * h ("Sampler en DiT controls": an 8-bit FC2 with one activation scale per
 * row). The 8-bit O and W2 GEMMs need hidden % 256 == 0. */
typedef struct {
  const void* w_qkv_codes;
  const float* w_qkv_scales;
  const void* w13_codes;
  const float* w13_scales;
  const void* w_o_codes;   /* may be null */
  const float* w_o_scales;
  const void* w2_codes;    /* may be null */
  const float* w2_scales;
} h3_block_weights_e4m3;

/* The steps of the 8-bit block, each as in the bf16 step of the same name.
 * Activation codes are [B*S, H] bytes (row-major, one row per packed row of
 * each batch element) with scales [B*S] f32: a row's values are code * scale.
 * All pointers DEVICE, 16-byte aligned; hidden % 128 == 0 for the GEMM steps.
 *
 * h3_norm_modulate_e4m3: h3_norm_modulate followed by the per-row quantization
 * (scale = max|h| / 448 over the row's fp32 h, 1 for an all-zero row; code =
 * e4m3(h / scale), round to nearest even, saturating). Padding rows get codes 0
 * and scale 1. */
H3_API h3_status h3_norm_modulate_e4m3(const h3_dims* dims, h3_layout_t layout, int B, int which,
                                       const void* x, const float* ada_table, const float* tmod,
                                       void* codes, float* scales, h3_stream_t stream);

/* h3_qkv_rope on 8-bit operands: the fp32 dot products of h_codes [B*S, H] and
 * w_codes [3*NH*D, H] (per-row weight scales w_scales [3*NH*D]), times
 * h_scales[row] * w_scales[col], then QK-norm + RoPE as in h3_qkv_rope. */
H3_API h3_status h3_qkv_rope_e4m3(const h3_dims* dims, h3_layout_t layout, int B,
                                  const void* h_codes, const float* h_scales, const void* w_codes,
                                  const float* w_scales, const void* q_norm, const void* k_norm,
                                  void* q, void* k, void* v, h3_stream_t stream);

/* h3_ffn_up on 8-bit operands: h2_codes [B*S, H] (scales [B*S]) against the
 * W1 || W3 codes [2F, H] (scales [2F]); g as in h3_ffn_up. */
H3_API h3_status h3_ffn_up_e4m3(const h3_dims* dims, h3_layout_t layout, int B,
                                const void* h2_codes, const float* h2_scales, const void* w_codes,
                                const float* w_scales, void* g, h3_stream_t stream);

/* h3_out_residual and h3_ffn_down_residual on 8-bit operands: input codes
 * [B*S, K] with per-row scales [B*S] (K = heads*128, resp. ffn), weight codes
 * [H, K] with per-row scales [H]; the gated residual as in the bf16 steps.
 * hidden % 256 == 0. */
H3_API h3_status h3_out_residual_e4m3(const h3_dims* dims, h3_layout_t layout, int B,
                                      const void* o_codes, const float* o_scales,
                                      const void* w_codes, const float* w_scales,
                                      const float* ada_table, const float* tmod, void* x,
                                      h3_stream_t stream);
H3_API h3_status h3_ffn_down_residual_e4m3(const h3_dims* dims, h3_layout_t layout, int B,
                                           const void* g_codes, const float* g_scales,
                                           const void* w_codes, const float* w_scales,
                                           const float* ada_table, const float* tmod, void* x,
                                           h3_stream_t stream);

/* Workspace bytes of h3_block_forward_e4m3: h3_workspace_size plus the codes
 * [B*S, max(H, heads*128, ffn)] and scales [B*S] of the activation rows. */
H3_API size_t h3_workspace_size_e4m3(const h3_dims* dims, int B, int S);

/* h3_block_forward with the QKV and W1 || W3 GEMMs (and, where w8 has them, the
 * O and W2 GEMMs) on e4m3 operands; the bf16 weights they replace are not
 * read. hidden % 128 == 0 (% 256 with O or W2 in 8 bits). */
H3_API h3_status h3_block_forward_e4m3(const h3_dims* dims, const h3_block_weights* weights,
                                       const h3_block_weights_e4m3* w8, h3_layout_t layout,
                                       const float* tmod, void* x, int B, void* ws,
                                       size_t ws_bytes, h3_stream_t stream);

/* h3_stack_forward with every block on its 8-bit operands w8[i] (as
 * h3_block_forward_e4m3), over the stack's fp32 residual stream. ws:
 * h3_workspace_size_e4m3(dims, B, S) bytes. */
H3_API h3_status h3_stack_forward_e4m3(const h3_dims* dims, const h3_block_weights* weights,
                                       const h3_block_weights_e4m3* w8, int n_blocks,
                                       h3_layout_t layout, const float* tmod, void* x, int B,
                                       void* ws, size_t ws_bytes, h3_stream_t stream);

/* ---- token reduction in the middle blocks ---- */

/* Build the token-reduced layout of `full` ("MiniMax H3 Inference Engine voor
 * Mac computers", section "Token-reduction internals": adjacent horizontal
 * target-video tokens are paired in the middle blocks; text, audio and
 * reference tokens stay exact). target [S] i32 (DEVICE): nonzero marks a
 * target-video row (a row being generated; reference / conditioning frames are
 * 0). Packed rows r, r + 1 pair when both are target-video rows with the same
 * t_idx, the same t and h and w coordinates 2k and 2k + 1 (reading: the page
 * names the pairing, not its rule). The reduced sequence keeps every other row
 * in packed order; a pair becomes one row at the first row's place with the
 * mean of the two positions. Returns a layout object usable by every call that
 * takes a layout, which also records its rows' sources in `full`. Synchronises
 * `stream`; allocates small device tables, released by h3_layout_destroy. */
H3_API h3_status h3_layout_reduce(const h3_dims* dims, h3_layout_t full, const int32_t* target,
                                  h3_stream_t stream, h3_layout_t* out);

/* Workspace bytes of h3_stack_forward_reduced: h3_workspace_size of the full
 * sequence plus the reduced fp32 stream. */
H3_API size_t h3_stack_reduced_workspace_size(const h3_dims* dims, h3_layout_t full,
                                              h3_layout_t reduced, int B);

/* n_blocks blocks as h3_stack_forward, with blocks [r0, r1) run on the reduced
 * sequence: after block r0 - 1 the fp32 stream is kept as the bypass and each
 * pair's rows are merged (mean); before block r1 every full row gets its reduced
 * row's change since the merge added to the bypass (both rows of a pair the same
 * change). r0 >= r1 runs the plain stack. (The page pairs after block 3 and
 * restores before block 40, or 30 after the first ten noisy evaluations: r0 =
 * 3, r1 = 39 or 29 in 0-based block indices.) x [B, S, H] bf16 in place. */
H3_API h3_status h3_stack_forward_reduced(const h3_dims* dims, const h3_block_weights* weights,
                                          int n_blocks, h3_layout_t full, h3_layout_t reduced,
                                          int r0, int r1, const float* tmod, void* x, int B,
                                          void* ws, size_t ws_bytes, h3_stream_t stream);

/* ---- the whole transformer forward: the denoiser around the stack ---- */

/* Widths of the rows that enter and leave the transformer (constructor
 * parameters in_channels * prod(patch_size), audio_in_channels, text_dim and
 * final_norm_eps). video_channels and audio_channels are 32, 64, 96 or 128;
 * text_dim % 64 == 0. */
typedef struct {
  int video_channels, audio_channels, text_dim;
  float final_norm_eps;
} h3_io_dims;

/* Parameters outside the block stack (DEVICE pointers, [out, in] row-major):
 *   w_patch_video [H, video_channels] f32, w_patch_audio [H, audio_channels] f32:
 *             the input patch projections (float32 modules, no bias)
 *   w_text    [H, text_dim] bf16: the text projection (part of the bf16 stack)
 *   w_t1, w_t2, w_proj: the timestep MLP and the stack's shared AdaLN
 *             projection, as for h3_timestep_modulation
 *   w_out     [2H, time_embed_dim] f32: norm_out's (shift, scale) projection of
 *             SiLU(temb)
 *   out_table [2, 2, H] f32: norm_out's per-modality rows, (video, audio) x
 *             (shift, scale)
 *   w_head_video [video_channels, H] f32, w_head_audio [audio_channels, H] f32:
 *             the two output heads (float32 modules, no bias) */
typedef struct {
  const float* w_patch_video;
  const float* w_patch_audio;
  const void* w_text;
  const float* w_t1;
  const float* w_t2;
  const float* w_proj;
  const float* w_out;
  const float* out_table;
  const float* w_head_video;
  const float* w_head_audio;
} h3_io_weights;

/* Core residual reuse ("MiniMax H3 Inference Engine voor Mac computers",
 * section "Sampler en DiT controls": the previous full transformer residual is
 * held while the patch projections and the timestep-aware head are refreshed).
 * The core is the text refiner and the block stack; its residual is the stack's
 * output minus its input, core_residual [B, V, H] f32 over the V valid rows in
 * packed order. H3_CORE_RUN: a plain forward; H3_CORE_STORE: a plain forward
 * that also writes core_residual; H3_CORE_REUSE: the refiner and the stack do
 * not run, the stream is the fresh patch projections plus core_residual. */
enum { H3_CORE_RUN = 0, H3_CORE_STORE = 1, H3_CORE_REUSE = 2 };

/* Bytes of device workspace h3_forward needs for B batch elements of the
 * layout (0 on invalid arguments). */
H3_API size_t h3_forward_workspace_size(const h3_dims* dims, const h3_io_dims* io,
                                        h3_layout_t layout, int B);

/* One transformer forward ("MiniMaxH3Transformer3DModel" page, `forward`):
 * latent rows in, velocities out, each in the row order of its index tensor.
 *   video [B, n_video, video_channels] f32, audio [B, n_audio, audio_channels]
 *   f32, text [B, n_text, text_dim] bf16 (the text encoder's condition);
 *   timestep [n_t] f32 (the distinct values, unscaled in [0, 1]);
 *   video_out [B, n_video, video_channels] f32, audio_out [B, n_audio,
 *   audio_channels] f32.
 * Steps: the timestep MLP, tmod = W_proj SiLU(temb) and norm_out's modulation
 * W_out SiLU(temb) (fp32); the patch projections (fp32) written into the
 * stack's fp32 residual stream of valid rows; the text projection, then
 * n_refiner refiner blocks (the block of this library with its own weights,
 * over the text rows alone as their own sequence, modulated by the text table
 * row and the rows' timesteps) and a LayerNorm (no affine, final_norm_eps) into
 * the stream; n_blocks stack blocks (as h3_stack_forward, the stream staying
 * fp32); norm_out = LayerNorm (no affine, final_norm_eps) * (1 + scale) + shift
 * with (shift, scale) = out_table[modality] + W_out SiLU(temb) of the row's
 * timestep; the fp32 heads. Readings where the page leaves the structure open:
 * no biases; the refiner's block structure, modulation and output norm and
 * norm_out's modulation source as just described. Padding rows take no part.
 * core_residual / core_mode: see H3_CORE_RUN (core_residual may be NULL with
 * H3_CORE_RUN). ws: h3_forward_workspace_size bytes. Enqueues only; outputs
 * are written at stream completion. */
H3_API h3_status h3_forward(const h3_dims* dims, const h3_io_dims* io, const h3_io_weights* io_weights,
                            const h3_block_weights* refiner, int n_refiner,
                            const h3_block_weights* blocks, int n_blocks, h3_layout_t layout,
                            const float* timestep, int B, const float* video, const float* audio,
                            const void* text, float* video_out, float* audio_out,
                            float* core_residual, int core_mode, void* ws, size_t ws_bytes,
                            h3_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* H3_H */
