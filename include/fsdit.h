/*
 * fsdit.h -- C ABI of libfsdit.so: the few-step Flash DiT hot path on one
 * NVIDIA B200 (sm_100a).
 *
 * Sources: web write-ups of arXiv 2609.15863 ("LynnReal-Omni"):
 *   [tokendh]    tokendh.com news article, sections "一个模型如何同时干七件事：
 *                原生多模态骨干网络" (backbone, per-row tags) and "训练的核心
 *                难题：怎么让模型又快又准" (flow matching, dual clocks, Flash
 *                layer schedule, spatial token compression);
 *   [PaperDaily] longzhangge PaperDaily "LynnReal Lab视频恢复与生成：统一多模态
 *                控制，Flash降至377毫秒", section 一 (tags, control offset,
 *                separate clocks) and section 二 "Flash怎么把22帧压到377毫秒"
 *                (compression, nearest-kept update broadcast, fused ops).
 *
 * Conventions for every call
 *  - Memory: the caller owns every buffer.  Pointers marked (device) are CUDA
 *    device pointers, 16-byte aligned; (host) are host pointers.  The library
 *    allocates nothing on these paths; scratch comes from a caller-provided
 *    workspace whose size fsdit_*_workspace_size() returns.
 *  - Streams: calls enqueue kernels on `stream` and return without waiting.
 *    All argument checks run on the host before any launch; a failed check
 *    launches nothing.
 *  - Errors: every call returns an fsdit_status; fsdit_last_error() gives a
 *    thread-local message for the last failure.  Kernels never trap: a device
 *    wait that exceeds its bound sets a device error word that
 *    fsdit_device_error() reads (after synchronizing the stream).
 *  - Layout: activations are token-major, row-major [rows, hidden].  Linear
 *    weights are [out_features, in_features] row-major (K contiguous), so a
 *    projection is y = x W^T + b.  The residual stream is float32 in every
 *    configuration; `dtype` selects the type of weights, biases, norm gains,
 *    text features and GEMM operands (FSDIT_F32 or FSDIT_BF16).
 *  - Packed sequence: rows [0, n_vrows) are video latent rows (the target grid
 *    first, then clean control frames), then n_text text rows, then n_audio
 *    audio rows.  Per-row tags ([tokendh] backbone section; [PaperDaily] 一):
 *    modality (0 text, 1 video, 2 audio, 3 video control), a noise-time slot
 *    into a per-call time table, a 3D (t,h,w) RoPE position and an output
 *    mark.
 */
#ifndef FSDIT_H
#define FSDIT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FSDIT_API __attribute__((visibility("default")))
#else
#define FSDIT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fsdit_stream_t; /* == cudaStream_t */

typedef enum {
  FSDIT_OK = 0,
  FSDIT_E_NULL = -1,      /* a required pointer is NULL */
  FSDIT_E_SHAPE = -2,     /* sizes inconsistent or outside what the kernels handle */
  FSDIT_E_ALIGN = -3,     /* a pointer is not 16-byte aligned */
  FSDIT_E_DTYPE = -4,     /* unknown dtype */
  FSDIT_E_CUDA = -5,      /* a CUDA runtime/driver call failed (message says which) */
  FSDIT_E_WORKSPACE = -6, /* workspace smaller than fsdit_*_workspace_size() */
  FSDIT_E_TIMEOUT = -7    /* a kernel gave up a bounded device wait */
} fsdit_status;

typedef enum { FSDIT_F32 = 0, FSDIT_BF16 = 1 } fsdit_dtype;

enum { FSDIT_MOD_TEXT = 0, FSDIT_MOD_VIDEO = 1, FSDIT_MOD_AUDIO = 2, FSDIT_MOD_CONTROL = 3 };

/* Model dimensions.  [tokendh] backbone section: hidden 5376, 56 heads of
 * 128, FFN 14336 (the Flash model keeps 42 of the 50 layers).  The heads span
 * heads*head_dim channels (56 x 128 = 7168), which need not equal hidden: the
 * qkv projection maps hidden -> 3*heads*head_dim and the output projection
 * maps heads*head_dim -> hidden.  head_dim must be 128; rope_split gives the
 * (t,h,w) chunk widths of a head (32/48/48), each even, summing to head_dim.
 * hidden and ffn are multiples of 64, hidden <= 8192. */
typedef struct {
  int hidden, heads, head_dim, ffn;
  int rope_split[3];
  float rms_eps;    /* RMSNorm epsilon (1e-6) */
  float rope_theta; /* RoPE base (10000) */
  int dtype;        /* fsdit_dtype of weights and GEMM operands */
  int proj_fp8;     /* 1: the four block projections run on FP8 E4M3 operands
                       (dtype must be FSDIT_BF16; see "Low-bit projections"
                       below); 0: they run in `dtype` */
} fsdit_dims;

/* Weights of one pre-norm DiT block (all (device), `dtype`); A = heads*128.
 *   w_qkv [3*A, hidden]  rows: q (A), k (A), v (A); head h owns rows
 *                        [h*128, h*128+128) of each part
 *   b_qkv [3*A]
 *   w_o   [hidden, A],   b_o [hidden]
 *   w_1   [ffn, hidden],     b_1 [ffn]
 *   w_2   [hidden, ffn],     b_2 [hidden]
 *   g_attn, g_ffn [hidden]   RMSNorm gains
 * With dims.proj_fp8 = 1, w_qkv, w_o, w_1 and w_2 hold E4M3 codes (one byte
 * each, same shapes) and s_qkv [3*A], s_o [hidden], s_1 [ffn], s_2 [hidden]
 * their per-output-channel fp32 scales (fsdit_quantize_rows of the bf16
 * weights); otherwise the s_* are unused (NULL). */
typedef struct {
  const void *w_qkv, *b_qkv, *w_o, *b_o, *w_1, *b_1, *w_2, *b_2, *g_attn, *g_ffn;
  const float *s_qkv, *s_o, *s_1, *s_2;
} fsdit_block_weights;

/* Embedding, timestep-MLP and output-head weights (all (device), `dtype`).
 *   w_vin [hidden, c_video], b_vin   video/control latent -> hidden
 *   w_tin [hidden, c_text],  b_tin   text feature -> hidden
 *   w_ain [hidden, c_audio], b_ain   audio latent -> hidden
 *   mod_emb [4, hidden]              learned modality embedding
 *   w_t1 [hidden, t_freq], b_t1, w_t2 [hidden, hidden], b_t2   timestep MLP
 *   g_out [hidden]                   final RMSNorm gain
 *   w_vout [c_video, hidden], b_vout; w_aout [c_audio, hidden], b_aout */
typedef struct {
  const void *w_vin, *b_vin, *w_tin, *b_tin, *w_ain, *b_ain, *mod_emb;
  const void *w_t1, *b_t1, *w_t2, *b_t2;
  const void *g_out, *w_vout, *b_vout, *w_aout, *b_aout;
  int c_video, c_text, c_audio, t_freq;
} fsdit_io_weights;

/* Tags of a packed sequence (all arrays (device)).
 *   n_tokens = n_vrows + n_text + n_audio
 *   grid_t/h/w: the target video grid, rows [0, grid_t*grid_h*grid_w) in
 *     (t,h,w) row-major order (0,0,0 if there is none); control rows follow.
 *   keep_idx [n_keep], near_idx [grid rows]: keep-index map of that grid from
 *     fsdit_build_keep_map (NULL/0: no compression).  The host checks n_keep
 *     against the grid; the kernels check every entry as they use it (see
 *     fsdit_gather_rows and fsdit_broadcast_residual): an entry outside the
 *     grid is never followed, and a map that is not a nearest-kept map is
 *     reported, through the device error word, as FSDIT_E_SHAPE by
 *     fsdit_device_error().
 *   pos_thw [n_tokens][3] int32, modality/time_id/out_mask [n_tokens] uint8. */
typedef struct {
  int n_tokens, n_vrows, n_text, n_audio;
  int grid_t, grid_h, grid_w;
  const int32_t* pos_thw;
  const uint8_t* modality;
  const uint8_t* time_id;
  const uint8_t* out_mask;
  const int32_t* keep_idx;
  int n_keep;
  const int32_t* near_idx;
} fsdit_tokens;

/* ---------------------------------------------------------------- queries */

/* Message of this thread's last failed call (static storage of the thread,
 * overwritten by its next failure; never NULL). */
FSDIT_API const char* fsdit_last_error(void);
/* Library name, version and target architecture (static string). */
FSDIT_API const char* fsdit_version(void);

/* Synchronizes `stream` and reads the device error word, which kernels set
 * instead of trapping.  Returns FSDIT_E_TIMEOUT if a kernel gave up a bounded
 * wait since the word was last cleared, FSDIT_E_SHAPE if the embedding found
 * row tags inconsistent with the sequence's segments (modality or time slot
 * out of place) or the gather / broadcast found a keep_idx / near_idx entry
 * outside the grid or not forming a nearest-kept map, else FSDIT_OK; a
 * non-zero word is cleared and described in fsdit_last_error(). */
FSDIT_API fsdit_status fsdit_device_error(fsdit_stream_t stream);

/* Failure-path check (no fault): launches one thread that waits, through the
 * bounded mbarrier wait every tensor-core kernel of the library uses, on a
 * barrier nothing arrives at.  The wait gives up after its limit (~2 s of SM
 * clocks), sets the device error word and returns; result (device, int[2])
 * receives {wait completed (0), abort flag set (1)}.  A following
 * fsdit_device_error() returns FSDIT_E_TIMEOUT (and clears the word); the
 * context stays usable. */
FSDIT_API fsdit_status fsdit_check_bounded_wait(int* result, fsdit_stream_t stream);

/* Launch profiler (measurement aid, off by default).  Between
 * fsdit_profile_start(max_launches) and fsdit_profile_stop() every launch the
 * library enqueues is bracketed by a CUDA event pair on its own stream (events
 * are created once and reused).  stop() waits for the last event, then writes
 * one entry per kernel class with its launches, summed device time and the
 * algorithmic FLOPs and bytes of those launches (computed on the host from the
 * shapes), and returns the number of classes (negative fsdit_status on error).
 * Not thread-safe; launches beyond max_launches are not recorded. */
typedef struct {
  char name[32];
  int scopes;   /* launch scopes recorded */
  int launches; /* kernels launched inside them */
  double ms;    /* summed device time */
  double flops; /* algorithmic FLOPs */
  double bytes; /* algorithmic bytes moved */
} fsdit_prof_entry;
FSDIT_API fsdit_status fsdit_profile_start(int max_launches);
FSDIT_API int fsdit_profile_stop(fsdit_prof_entry* entries, int max_entries);

/* Number of kept tokens of a T x H x W grid: T * (H/2+1) * (W/2+1). */
FSDIT_API int fsdit_keep_count(int T, int H, int W);

/* Workspace bytes for dit_block_forward on n_tokens rows (n_keep kept grid
 * rows, 0 = no compression) and for one dit_stack_forward / dit_flow_sample
 * call. */
FSDIT_API size_t fsdit_block_workspace_size(const fsdit_dims* dims, int n_tokens, int n_keep);
FSDIT_API size_t fsdit_stack_workspace_size(const fsdit_dims* dims, const fsdit_io_weights* io,
                                  const fsdit_tokens* tok, int n_times);

/* ---------------------------------------------------------------- hot path */

/* Keep-index map of a T x H x W video grid ([tokendh] training section,
 * Flash paragraph; [PaperDaily] 二): per frame keep rows {0,2,4,..}+{H-1} and
 * columns {0,2,4,..}+{W-1}, no temporal drop.  keep_idx[c] (device, int32
 * [fsdit_keep_count]) = full-grid row id t*H*W+h*W+w of kept token c in
 * (t, kept h, kept w) order; near_idx[p] (device, int32 [T*H*W]) = compact id
 * of the kept token nearest to row p in its own frame (a dropped index lies
 * midway between two kept ones; the lower one is taken). */
FSDIT_API fsdit_status fsdit_build_keep_map(int T, int H, int W, int32_t* keep_idx, int32_t* near_idx,
                                  fsdit_stream_t stream);

/* Gather the compressed sequence: rows [0, n_keep) of x_c / pos_c are the
 * grid rows keep_idx[c] of x / pos; rows [n_keep, n_keep + n_rows - n_grid)
 * are the non-grid rows n_grid.. n_rows-1 in order (text and audio are never
 * compressed, [PaperDaily] 二).  x, x_c float32 [.., hidden] (device); pos,
 * pos_c int32 [..,3] (device, may both be NULL).  A keep_idx entry outside
 * [0, n_grid) is not followed: that row of x_c / pos_c is left unwritten and
 * the device error word is set (fsdit_device_error() returns FSDIT_E_SHAPE). */
FSDIT_API fsdit_status fsdit_gather_rows(const float* x, const int32_t* pos, float* x_c, int32_t* pos_c,
                               const int32_t* keep_idx, int n_keep, int n_grid, int n_rows,
                               int hidden, fsdit_stream_t stream);

/* Nearest-kept broadcast + residual ([PaperDaily] 二; [tokendh] training
 * section): the compressed layers' update of kept token c is
 * d_c = y_c[c] - x[keep_idx[c]]; kept grid rows take y_c, dropped grid rows p
 * take x[p] + d_{near_idx[p]} (float32 arithmetic), non-grid rows take their
 * y_c rows.  The grid is grid_t x grid_h x grid_w (rows [0, T*H*W) of x) with
 * the map of fsdit_build_keep_map (n_keep kept tokens); each kept token's
 * dropped rows lie at +1 / +W / +W+1 of it in its frame.  One launch; out may
 * equal x (every row is read and written by one block only).
 * The kernel checks the map as it uses it: every keep_idx[c] must lie in the
 * grid with near_idx[keep_idx[c]] == c, and every near_idx[p] must name a
 * kept token in p's frame at most one row above and one column left of p.
 * These conditions are exactly those under which every grid row is written
 * once.  Entries that fail are not followed (no access outside x, y_c, out or
 * the two maps; the rows they would have produced are left unwritten, which
 * for out == x means unchanged) and set the device error word, which
 * fsdit_device_error() reports as FSDIT_E_SHAPE. */
FSDIT_API fsdit_status fsdit_broadcast_residual(const float* x, const float* y_c, float* out,
                                      const int32_t* keep_idx, const int32_t* near_idx,
                                      int n_keep, int grid_t, int grid_h, int grid_w, int n_rows,
                                      int hidden, fsdit_stream_t stream);

/* RMSNorm fused into the GEMM-operand pass: xn[r] = cast(x[r] * g /
 * sqrt(mean(x[r]^2) + eps)).  x float32 [rows, hidden]; g and xn in `dtype`. */
FSDIT_API fsdit_status fsdit_rmsnorm_cast(const float* x, const void* g, void* xn, int rows, int hidden,
                                float eps, int dtype, fsdit_stream_t stream);

/* Epilogues of fsdit_linear (all add the bias first):
 *   FSDIT_EPI_BIAS       out (dtype)  = acc + b
 *   FSDIT_EPI_BIAS_F32   out (f32)    = acc + b
 *   FSDIT_EPI_QKV_ROPE   out (dtype)  = rope(acc + b) on columns < 2*heads*128
 *                        (q and k; N must be 3*heads*128), per row position
 *                        pos[row]
 *   FSDIT_EPI_GELU       out (dtype)  = gelu_tanh(acc + b)
 *   FSDIT_EPI_RESIDUAL   out (f32)    = resid + acc + b   (out may equal resid) */
enum {
  FSDIT_EPI_BIAS = 0,
  FSDIT_EPI_BIAS_F32 = 1,
  FSDIT_EPI_QKV_ROPE = 2,
  FSDIT_EPI_GELU = 3,
  FSDIT_EPI_RESIDUAL = 4
};

/* One projection out[M,N] = a[M,K] w[N,K]^T with a fused epilogue.
 * a, w, b in `dtype` (device).  bf16 runs on the tcgen05 tensor cores (TMA
 * operand staging, fp32 accumulation in tensor memory); f32 runs exact fp32
 * FMA.  K % 8 == 0; N % 32 == 0.  dims supplies head_dim / rope split / theta
 * for FSDIT_EPI_QKV_ROPE (pos int32 [M][3] (device)). */
FSDIT_API fsdit_status fsdit_linear(const fsdit_dims* dims, const void* a, const void* w, const void* b,
                          void* out, const float* resid, const int32_t* pos, int M, int N, int K,
                          int epilogue, fsdit_stream_t stream);

/* ------------------------------------------------------ low-bit projections
 * [PaperDaily] section 二, third step: suitable projections run on low-bit
 * weights and activations, with quantization fused next to the
 * normalization.  Here: FP8 E4M3 (round to nearest even, saturating at 448)
 * with one fp32 scale per row of each quantized operand -- per token for
 * activations, per output channel for weights: s = amax / 448 rounded to
 * fp32 (1 for an all-zero row), q = the E4M3 code of the exact quotient
 * value / s (ties to even; exact for s >= 2^-100).
 * A projection computes (sum_k qa qw) * sa[row] * sw[col] + b on the tcgen05
 * tensor cores (kind::f8f6f4, fp32 accumulation), then its epilogue. */

/* Per-row E4M3 quantization of a [rows, cols] matrix `a` (device; fp32 or
 * bf16 by `dtype`): q [rows, cols] E4M3 codes, s [rows] fp32 scales (device).
 * cols % 16 == 0; a, q 16-byte aligned. */
FSDIT_API fsdit_status fsdit_quantize_rows(const void* a, int dtype, int rows, int cols, uint8_t* q, float* s,
                                           fsdit_stream_t stream);

/* RMSNorm fused with the quantization of its output: y = x * rstd * g in
 * fp32 (x fp32 [rows, hidden], g bf16), then q, s as fsdit_quantize_rows. */
FSDIT_API fsdit_status fsdit_rmsnorm_quant(const float* x, const void* g, int rows, int hidden, float eps,
                                           uint8_t* q, float* s, fsdit_stream_t stream);

/* out = epilogue((qa qw^T) * sa[row] * sw[col] + b): qa [M, K], qw [N, K] E4M3
 * codes, sa [M], sw [N] fp32, b bf16; epilogues and outputs as
 * fsdit_linear with dtype bf16.  K % 16 == 0, N % 32 == 0, pointers 16-byte
 * aligned. */
FSDIT_API fsdit_status fsdit_linear_fp8(const fsdit_dims* dims, const uint8_t* qa, const float* sa, const uint8_t* qw,
                                        const float* sw, const void* b, void* out, const float* resid,
                                        const int32_t* pos, int M, int N, int K, int epilogue,
                                        fsdit_stream_t stream);

/* Tail cut of the tensor-core projections.  A projection runs as a
 * persistent grid of CTA pairs over 256 x 256 output tiles; when the tiles
 * leave the last wave mostly idle (R tiles left for P pairs, R <= P/2), the
 * *_ws calls cut each of those R tiles along K into S <= P/R units (at least
 * four 128-byte K steps each, at most 8) that run on the idle pairs.  Each
 * unit parks its fp32 partial accumulators in `scratch`; the unit that
 * completes a tile region last sums the parts in unit order (so the result
 * does not depend on which unit finishes last) and applies the epilogue.
 * scratch (device, 16-byte aligned) holds fsdit_gemm_scratch_size() bytes;
 * the call first zeroes its counters (one memset on `stream`), so calls that
 * may run at the same time (other streams) need scratch of their own; NULL
 * scratch = the plain call.  Only GEMMs of at least 32 K steps are cut, into units
 * of at least 12.  Same arguments and errors as fsdit_linear /
 * fsdit_linear_fp8, plus FSDIT_E_WORKSPACE / FSDIT_E_ALIGN for the scratch.
 * The cut shortens a GEMM run on its own (measured 16-30% on the compressed
 * Flash projections); inside a long power-capped pass the GPU's clock, not
 * its idle SMs, sets the time and the cut gains nothing, so the block,
 * stack, sampler and decoder calls run whole tiles only. */
FSDIT_API size_t fsdit_gemm_scratch_size(void);
FSDIT_API fsdit_status fsdit_linear_ws(const fsdit_dims* dims, const void* a, const void* w, const void* b,
                                       void* out, const float* resid, const int32_t* pos, int M, int N, int K,
                                       int epilogue, void* scratch, size_t scratch_bytes, fsdit_stream_t stream);
FSDIT_API fsdit_status fsdit_linear_fp8_ws(const fsdit_dims* dims, const uint8_t* qa, const float* sa,
                                           const uint8_t* qw, const float* sw, const void* b, void* out,
                                           const float* resid, const int32_t* pos, int M, int N, int K,
                                           int epilogue, void* scratch, size_t scratch_bytes,
                                           fsdit_stream_t stream);

/* Joint attention ([tokendh] backbone section: one sequence of text,
 * video and audio tokens through one denoiser): for each head,
 * softmax(q k^T / sqrt(128)) v over all n rows, no mask.  With A = heads*128:
 * qkv [n, 3*A] in `dtype` (q | k | v, RoPE already applied); out [n, A] in
 * `dtype`. */
FSDIT_API fsdit_status fsdit_attention(const fsdit_dims* dims, const void* qkv, void* out, int n,
                             fsdit_stream_t stream);

/* Attention kernel choice (bf16).  Sequences of at least `rows` rows run on
 * the CTA-pair kernel (clusters of two CTAs, 256 queries per cluster, each
 * CTA staging half of every key and value block); shorter ones on the
 * single-CTA kernel (256 queries per CTA).  Both compute the same attention;
 * the threshold is a tuning knob for the whole process (not thread-safe
 * against concurrent launches).  fsdit_attention_pair_min_rows returns the
 * current value.  Errors: FSDIT_E_SHAPE for rows < 1. */
FSDIT_API fsdit_status fsdit_set_attention_pair_min_rows(int rows);
FSDIT_API int fsdit_attention_pair_min_rows(void);

/* RMSNorm placement in stacks and the decoder (dit_stack_forward and what
 * calls it, fsdit_decoder_forward): on = 1 (the default) applies a norm that
 * follows a residual projection after the GEMM that consumes it (see
 * dit_stack_forward); on = 0 runs every norm as its own fsdit_rmsnorm_cast
 * pass.  The same RMSNorm either way, rounded in a different order.  A
 * process-wide switch (not thread-safe against concurrent launches); query
 * workspace sizes after setting it.  fsdit_norm_after_gemm returns the
 * current value.  Errors: FSDIT_E_SHAPE unless on is 0 or 1. */
FSDIT_API fsdit_status fsdit_set_norm_after_gemm(int on);
FSDIT_API int fsdit_norm_after_gemm(void);

/* One DiT block.  x_in, x_out float32 [n_tokens, hidden] (device);
 * x_out may equal x_in.  With tok->keep_idx != NULL the block is the Flash
 * compressed block in per-block form: gather the kept grid rows and all
 * non-grid rows, run the block on them, broadcast with
 * fsdit_broadcast_residual.  Positions of kept rows stay their original
 * (t,h,w). */
FSDIT_API fsdit_status dit_block_forward(const fsdit_dims* dims, const fsdit_block_weights* w,
                               const fsdit_tokens* tok, const float* x_in, float* x_out,
                               void* workspace, size_t ws_bytes, fsdit_stream_t stream);

/* One backbone evaluation: embedding (input projections + modality
 * embedding + timestep embedding of time_table[time_id[row]]), n_layers
 * blocks (layers: host array of n_layers weight structs; layer_compress: host
 * uint8 [n_layers], 1 = token-compressed; a run of compressed layers gathers
 * once and broadcasts once, which equals the per-layer form in exact
 * arithmetic), final RMSNorm and the video/audio velocity heads.  With bf16
 * dense projections and hidden % 128 == 0, a norm that follows a residual
 * projection on the same rows is applied after the GEMM that consumes it:
 * the residual epilogue writes bf16(x * g) and per-128-column sums of x^2,
 * and the consuming GEMM's epilogue forms 1/rms of each row from those sums
 * and scales its accumulators by it (the same RMSNorm in exact arithmetic; in
 * bf16 the operand is rounded before the row scale instead of after it).
 *   time_table (host) float [n_times], n_times <= 8
 *   video_lat float32 [n_vrows, c_video], audio_lat float32 [n_audio, c_audio],
 *   text_emb `dtype` [n_text, c_text]                      (device, inputs)
 *   v_video float32 [n_vrows, c_video], v_audio float32 [n_audio, c_audio]
 *                                                           (device, outputs) */
FSDIT_API fsdit_status dit_stack_forward(const fsdit_dims* dims, int n_layers,
                               const fsdit_block_weights* layers, const uint8_t* layer_compress,
                               const fsdit_io_weights* io, const fsdit_tokens* tok,
                               const float* time_table, int n_times, const float* video_lat,
                               const void* text_emb, const float* audio_lat, float* v_video,
                               float* v_audio, void* workspace, size_t ws_bytes,
                               fsdit_stream_t stream);

/* One flow-matching Euler step with a clock per modality ([tokendh]
 * training section: x_t = (1-t) x0 + t eps, the network predicts
 * v = eps - x0; [PaperDaily] 一: video and audio share the forward but keep
 * their own noise clocks): for each row r with out_mask[r] != 0,
 * x[r] += (t_next[m] - t_cur[m]) * v[r], m = row_modality[r].  x, v float32
 * [n_rows, row_width] (device); row_modality, out_mask uint8 [n_rows]
 * (device); t_cur, t_next (host) float [4] indexed by modality code. */
FSDIT_API fsdit_status flow_euler_step(float* x, const float* v, const uint8_t* row_modality,
                             const uint8_t* out_mask, int n_rows, int row_width,
                             const float* t_cur, const float* t_next, fsdit_stream_t stream);

/* The few-step sampler: n_evals evaluations of dit_stack_forward; eval e
 * uses time table {0, t_video[e], t_audio[e]} (slots 0 clean, 1 video, 2 audio)
 * and then Euler-steps the video rows from t_video[e] to t_video[e+1] and the
 * audio rows from t_audio[e] to t_audio[e+1].  Flash: 3 evaluations on
 * 0.2 -> 0.0769 -> 0.027 -> 0 (video) and 0.5 -> 0.25 -> 0.1 -> 0 (audio)
 * ([tokendh] training section).  video_lat / audio_lat (device, float32) are
 * updated in place; t_video, t_audio (host) float [n_evals + 1]. */
FSDIT_API fsdit_status dit_flow_sample(const fsdit_dims* dims, int n_layers,
                             const fsdit_block_weights* layers, const uint8_t* layer_compress,
                             const fsdit_io_weights* io, const fsdit_tokens* tok, int n_evals,
                             const float* t_video, const float* t_audio, float* video_lat,
                             const void* text_emb, float* audio_lat, void* workspace,
                             size_t ws_bytes, fsdit_stream_t stream);

/* The paper has no counterpart to this entry point; it exists for callers of
 * this library that cannot call cudaMalloc -- for example a host application
 * whose device memory is owned by its own pool allocator, or a plain C caller
 * that must not allocate after start-up -- and so cannot provide the
 * workspace dit_block_forward needs.
 *
 * Same computation and arguments as dit_block_forward, minus the workspace:
 * the scratch comes from one static device array of 32 MiB inside the
 * library (every GPU that loads libfsdit.so holds it until the process
 * exits).  The call allocates nothing: no cudaMalloc, cudaFree or allocating
 * library routine.  Returns FSDIT_E_WORKSPACE, launching nothing, when the
 * block's scratch exceeds 32 MiB.  That scratch is the workspace
 * dit_block_forward would take: fsdit_block_workspace_size(dims, n, 0) for an
 * uncompressed block of n rows, and for a compressed block the same function
 * of its compressed row count n_c = n_keep + (n_tokens - grid rows), i.e.
 * fsdit_block_workspace_size(dims, n_c, 1).  The largest blocks accepted:
 *   hidden 5376, 56 x 128 heads, FFN 14336: bf16 387 rows uncompressed,
 *     310 compressed rows; fp32 194 / 172;
 *   hidden 2048, 16 x 128 heads, FFN 8192: bf16 1,008 / 808; fp32 508 / 451;
 *   hidden 256, 2 x 128 heads, FFN 512: bf16 9,362 / 7,262; fp32 5,041 / 4,362.
 *
 * The array's device address is looked up for the current device (once per
 * device, on the first call with that device current); make that first call
 * before any stream capture.  `stream` must belong to the current device:
 * a stream of another device returns FSDIT_E_CUDA, launching nothing.  Every call shares the one array and it keeps the last call's
 * contents (nothing in it needs to start at zero: every buffer is written
 * before it is read).  Calls that overlap on the GPU -- on different streams,
 * or from different threads -- race on it; serialize them. */
FSDIT_API fsdit_status dit_block_forward_noalloc(const fsdit_dims* dims, const fsdit_block_weights* w,
                                                 const fsdit_tokens* tok, const float* x_in, float* x_out,
                                                 fsdit_stream_t stream);

/* ------------------------------------------------------------------ long video
 * Chunked generation with a bounded, multi-stride history ([tokendh] section
 * "长视频生成：怎么记住十分钟前发生的事"; [PaperDaily] section 三).  A chunk's
 * target grid is T latent frames: frame 0 is the boundary latent (the last
 * latent of the video so far; clean and never updated), frames 1..T-1 are new.
 * Its history is made of latent frames before the boundary: frame 0 of the
 * video at full resolution, the two newest at spatial stride 2 and at most
 * eight before those at stride 4 (rows and columns that are multiples of the
 * stride); frames in between are dropped.  History rows are clean video
 * conditions at their original (t, h, w) and sit after the target grid rows
 * (they are not token-compressed).  The first chunk has no boundary and no
 * history. */

#define FSDIT_HISTORY_MAX_ENTRIES 11 /* 1 full + 8 stride-4 + 2 stride-2 frames */
#define FSDIT_HISTORY_MIN_SLOTS 12   /* frame 0, the 10 newest history frames, the boundary */

/* One frame of a history plan, in time order. */
typedef struct {
  int frame;  /* index of the latent frame in the video (0 = first) */
  int stride; /* spatial stride: 1, 2 or 4 */
} fsdit_history_entry;

/* The frame store: caller-owned device memory of `capacity` latent frames,
 * each [H][W][C] fp32 (the video-latent layout of fsdit_tokens' video rows).
 * Frame 0 stays in slot 0; frame i >= 1 goes to slot 1 + (i - 1) % (capacity
 * - 1), so with capacity >= FSDIT_HISTORY_MIN_SLOTS every frame a plan names
 * is still resident.  The struct is plain data; the library keeps no state. */
typedef struct {
  float* frames;  /* device, capacity * H * W * C floats, 16-byte aligned */
  int capacity, H, W, C;
  int n_frames;   /* latent frames pushed so far */
} fsdit_history_store;

/* Bytes of a store's frame memory. */
FSDIT_API size_t fsdit_history_bytes(int capacity, int H, int W, int C);

/* Set up `s` over caller memory `frames` (no device work).  Errors:
 * FSDIT_E_NULL, FSDIT_E_SHAPE (capacity < FSDIT_HISTORY_MIN_SLOTS or a
 * non-positive size), FSDIT_E_ALIGN. */
FSDIT_API fsdit_status fsdit_history_init(fsdit_history_store* s, float* frames, int capacity, int H, int W,
                                          int C);

/* Append `n` latent frames (device, contiguous [n][H][W][C] fp32) to the
 * video: asynchronous device copies on `stream`, then s->n_frames += n. */
FSDIT_API fsdit_status fsdit_history_push(fsdit_history_store* s, const float* frames, int n,
                                          fsdit_stream_t stream);

/* Host: the history plan of a chunk whose boundary is frame `n_before` (the
 * frames 0 .. n_before-1 come before it).  Writes at most `max_entries`
 * entries to `out` and returns how many (0 .. FSDIT_HISTORY_MAX_ENTRIES), or
 * -1 when n_before < 0 or `out` is too small. */
FSDIT_API int fsdit_history_plan(int n_before, fsdit_history_entry* out, int max_entries);

/* Host: history rows of a plan for an H x W frame. */
FSDIT_API int fsdit_history_rows(const fsdit_history_entry* plan, int n_plan, int H, int W);

/* Gather the plan's rows from the store: row r of the output is one (frame,
 * h, w) of the plan, frame by frame in plan order, each frame row-major at
 * its stride.  lat [rows][ld_lat] fp32 (C values written per row; ld_lat >=
 * C) and pos [rows][3] int32 = (frame, h, w), both device.  Errors:
 * FSDIT_E_SHAPE when a planned frame is not resident (never pushed, or
 * overwritten), a stride is not 1, 2 or 4, or n_plan is out of range. */
FSDIT_API fsdit_status fsdit_history_gather(const fsdit_history_store* s, const fsdit_history_entry* plan,
                                            int n_plan, float* lat, int ld_lat, int32_t* pos,
                                            fsdit_stream_t stream);

/* Copy resident frame `frame` ([H][W][C] fp32) to device memory `dst`
 * (e.g. the boundary slot of the next chunk's latents). */
FSDIT_API fsdit_status fsdit_history_copy_frame(const fsdit_history_store* s, int frame, float* dst,
                                                fsdit_stream_t stream);

/* Host: row tags of one chunk, the layout fsdit_tokens expects: [target grid
 * T x H x W at t = base + 0 .. T-1 | n_hist history rows | n_text text |
 * n_audio audio].  Grid rows: video modality, time id 1, updated, except the
 * boundary frame 0 when has_boundary (time id 0, not updated).  History rows:
 * video modality, time id 0, not updated, pos left untouched (the gather
 * writes it).  Text rows: time id 0, pos (0,0,0).  Audio rows: time id 2,
 * updated, pos (floor(j T / n_audio) + base, 0, 0).  Host arrays of n =
 * T*H*W + n_hist + n_text + n_audio entries (pos: 3n).  Errors: FSDIT_E_NULL;
 * FSDIT_E_SHAPE for a non-positive grid size, negative counts or base, or
 * has_boundary with T < 2 (a chunk with a boundary frame has at least one new
 * frame). */
FSDIT_API fsdit_status fsdit_chunk_tags(int T, int H, int W, int base, int has_boundary, int n_hist, int n_text,
                                        int n_audio, uint8_t* modality, uint8_t* time_id, uint8_t* out_mask,
                                        int32_t* pos);

/* ------------------------------------------------------------------ decoder
 * The lightweight video decoder ([tokendh] section "解码器瓶颈：被忽视的那一半
 * 时间": 26 layers, hidden width 2048, feed-forward 4x hidden; [ananclaw
 * explainer] section 3.4: a lightweight VAE decoder), read as a transformer
 * over the latent cells of a T x H x W grid:
 *   x = z W_in^T + b_in  (one row per cell, (t, h, w) row-major; no time or
 *                         modality embedding);
 *   n_layers blocks of the backbone's form (fsdit_block_weights; RoPE at the
 *   cell's (t, h, w); full attention over the clip; never compressed);
 *   pixel head: rmsnorm(x; g_out) W_out^T + b_out, one row of
 *   c_pix * patch_t * patch_s^2 values per cell, columns ordered
 *   (channel, dt, dy, dx) with dx fastest;
 *   unpatchify (fused into the head's epilogue): column (c, dt, dy, dx) of
 *   cell (t, h, w) is pixel (patch_s*h + dy, patch_s*w + dx) of channel c in
 *   frame patch_t*t + dt - (patch_t - 1), dropped when negative (causal:
 *   latent frame 0 yields one frame), so T latent frames give
 *   fsdit_decoder_frames(T, patch_t) = 1 + patch_t*(T - 1) frames. */
typedef struct {
  const void *w_in, *b_in;   /* [hidden, c_lat], [hidden] (dims.dtype, device) */
  const void* g_out;         /* [hidden] final RMSNorm gain */
  const void *w_out, *b_out; /* [c_pix*patch_t*patch_s*patch_s, hidden], [same] */
  int c_lat;                 /* latent channels, 1..64 */
  int c_pix;                 /* pixel channels (3) */
  int patch_t;               /* frames per latent frame (4) */
  int patch_s;               /* pixels per latent cell along h and w (16); a multiple of 4 */
} fsdit_decoder_io;

/* Frames decoded from T latent frames: 1 + patch_t*(T-1) (0 when T <= 0). */
FSDIT_API int fsdit_decoder_frames(int T, int patch_t);

/* Workspace bytes of fsdit_decoder_forward on a T x H x W grid (0 on bad
 * arguments). */
FSDIT_API size_t fsdit_decoder_workspace_size(const fsdit_dims* dims, const fsdit_decoder_io* io, int T, int H,
                                              int W);

/* Pixel formats of fsdit_decoder_forward.  FSDIT_PIXELS_RGB8 is the GPU-side
 * colour conversion of [PaperDaily] section 二 (the fully accelerated
 * configuration), fused into the pixel head: each value v, read as lying in
 * [-1, 1], becomes the code round_half_even(clamp(127.5 * (v + 1), 0, 255)),
 * the product and the sum each rounded to fp32. */
enum { FSDIT_PIXELS_F32 = 0, FSDIT_PIXELS_RGB8 = 1 };

/* Decode latents (device, fp32 [T*H*W][c_lat], cells (t, h, w) row-major) into
 * pixels (device, [fsdit_decoder_frames(T, patch_t)][c_pix][H*patch_s]
 * [W*patch_s] of fp32 values or uint8 codes per pixel_format, 16-byte aligned,
 * fully written).  layers: host array of
 * n_layers block weights (device pointers; with dims.proj_fp8 the E4M3 weights
 * and scales as for the backbone).  The residual stream is fp32; the GEMMs and
 * attention run as in the backbone (bf16 on the tcgen05 tensor cores, or
 * exact fp32 with dims.dtype FSDIT_F32).  Errors: FSDIT_E_NULL,
 * FSDIT_E_SHAPE (grid empty, c_lat outside 1..64, patch sizes not positive,
 * patch_s % 4 != 0), FSDIT_E_DTYPE (unknown pixel_format), FSDIT_E_ALIGN,
 * FSDIT_E_WORKSPACE. */
FSDIT_API fsdit_status fsdit_decoder_forward(const fsdit_dims* dims, int n_layers, const fsdit_block_weights* layers,
                                             const fsdit_decoder_io* io, int T, int H, int W, const float* latents,
                                             void* pixels, int pixel_format, void* workspace, size_t ws_bytes,
                                             fsdit_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FSDIT_H */
