// C ABI of libfsdit: host-side argument checks, workspace layout and the
// launch sequence of the block, the backbone stack and the sampler.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "common.cuh"

namespace fsdit {

// ---------------------------------------------------------------- profiler
static const char* kProfNames[PC_COUNT] = {"gemm_qkv_rope", "gemm_residual", "gemm_gelu", "gemm_bias_f32",
                                           "gemm_bias",     "attention",     "rmsnorm_cast", "gather",
                                           "broadcast",     "embed",         "time_mlp",  "heads",
                                           "euler",         "keep_map",  "rope_table", "history_gather",
                                           "quantize",      "gemm_fp8_qkv_rope", "gemm_fp8_residual",
                                           "gemm_fp8_gelu", "grid_positions", "pixel_head"};
struct Prof {
  bool on = false;
  int used = 0;
  std::vector<cudaEvent_t> ev;
  std::vector<int> cls, kernels;
  std::vector<double> flops, bytes;
};
static Prof g_prof;

// Inside a stream capture the event pair must be recorded as external event
// nodes, so every replay of the graph stamps them.
static void prof_record(cudaEvent_t e, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
  else
    cudaEventRecord(e, st);
}

ProfScope::ProfScope(int c, int k, double fl, double by, cudaStream_t s) : slot(-1), st(s) {
  if (!g_prof.on || 2 * (size_t)(g_prof.used + 1) > g_prof.ev.size()) return;
  slot = g_prof.used++;
  g_prof.cls[slot] = c;
  g_prof.kernels[slot] = k;
  g_prof.flops[slot] = fl;
  g_prof.bytes[slot] = by;
  prof_record(g_prof.ev[2 * slot], st);
}
ProfScope::~ProfScope() {
  if (slot >= 0) prof_record(g_prof.ev[2 * slot + 1], st);
}
void ProfScope::add_kernels(int k) {
  if (slot >= 0) g_prof.kernels[slot] += k;
}
// The launch scope open on this thread (a projection's launcher adds the
// second kernel of a tail cut to it).
static thread_local ProfScope* t_scope = nullptr;
void prof_add_kernels(int k) {
  if (t_scope != nullptr) t_scope->add_kernels(k);
}

fsdit_status launch_keep_map(int T, int H, int W, int32_t* keep_idx, int32_t* near_idx, cudaStream_t st);
fsdit_status launch_gather(const float* x, const int32_t* pos, float* xc, int32_t* posc, const int32_t* keep_idx,
                           int n_keep, int n_grid, int n_rows, int hidden, cudaStream_t st);
fsdit_status launch_broadcast(const float* x, const float* yc, float* out, const int32_t* keep_idx,
                              const int32_t* near_idx, int n_keep, int grid_t, int grid_h, int grid_w, int n_rows,
                              int hidden, cudaStream_t st);
fsdit_status launch_rmsnorm_cast(const float* x, const void* g, void* xn, int rows, int hidden, float eps, int dtype,
                                 cudaStream_t st);
fsdit_status launch_embed(int dtype, float* x, int hidden, int row0, int rows, int kind, const float* lat, int K,
                          const void* w_in, const void* b_in, const float* text_proj, const void* mod_emb,
                          const float* temb, const uint8_t* modality, const uint8_t* time_id, int n_times, int ea,
                          int eb, cudaStream_t st);
fsdit_status launch_time_mlp(int dtype, const float* times_host, int n_times, int t_freq, const void* w1,
                             const void* b1, const void* w2, const void* b2, float* h1, float* temb, int hidden,
                             cudaStream_t st);
fsdit_status launch_rope_table(const int32_t* pos, int rows, int head_dim, int s0, int s1, float log2_theta,
                               float2* cs, cudaStream_t st);
fsdit_status launch_euler(float* x, const float* v, const uint8_t* mod, const uint8_t* mask, int n_rows, int width,
                          const float* t_cur, const float* t_next, cudaStream_t st);

// ---------------------------------------------------------------- errors
static thread_local char t_err[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof(t_err), fmt, ap);
  va_end(ap);
}

fsdit_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return FSDIT_OK;
  set_error("%s: %s", what, cudaGetErrorString(e));
  return FSDIT_E_CUDA;
}

int num_sms() {
  static PerDevice<int> sms;
  return sms.get(
      [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
          return v;
        (void)cudaGetLastError();
        return 148;
      },
      148);
}

#define FS_TRY(expr)                        \
  do {                                      \
    fsdit_status _s = (expr);               \
    if (_s != FSDIT_OK) return _s;          \
  } while (0)

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static fsdit_status need(const void* p, const char* name) {
  if (p == nullptr) {
    set_error("%s is NULL", name);
    return FSDIT_E_NULL;
  }
  if (!aligned16(p)) {
    set_error("%s is not 16-byte aligned", name);
    return FSDIT_E_ALIGN;
  }
  return FSDIT_OK;
}

static size_t dsize(int dtype) { return dtype == FSDIT_BF16 ? 2 : 4; }
// attention width: heads * head_dim (56 x 128 = 7168 next to hidden 5376)
static int attn_dim(const fsdit_dims* d) { return d->heads * d->head_dim; }

static fsdit_status check_dims(const fsdit_dims* d) {
  FS_TRY(need(d, "dims"));
  if (d->dtype != FSDIT_F32 && d->dtype != FSDIT_BF16) {
    set_error("dims.dtype %d is neither FSDIT_F32 nor FSDIT_BF16", d->dtype);
    return FSDIT_E_DTYPE;
  }
  if (d->head_dim != 128 || d->heads <= 0 || d->heads > 256 || d->hidden <= 0 || d->hidden % 64 != 0 ||
      d->hidden > 8192) {
    set_error("dims: need head_dim 128, 0 < heads <= 256, hidden %% 64 == 0, hidden <= 8192 (got %d/%d/%d)",
              d->hidden, d->heads, d->head_dim);
    return FSDIT_E_SHAPE;
  }
  if (d->ffn <= 0 || d->ffn % 64 != 0) {
    set_error("dims.ffn %d must be a positive multiple of 64", d->ffn);
    return FSDIT_E_SHAPE;
  }
  const int* s = d->rope_split;
  if (s[0] < 0 || s[1] < 0 || s[2] < 0 || (s[0] | s[1] | s[2]) & 1 || s[0] + s[1] + s[2] != d->head_dim) {
    set_error("dims.rope_split must be three even widths summing to head_dim");
    return FSDIT_E_SHAPE;
  }
  if (!(d->rms_eps >= 0.f) || !(d->rope_theta > 1.f)) {
    set_error("dims: rms_eps must be >= 0 and rope_theta > 1");
    return FSDIT_E_SHAPE;
  }
  if (d->proj_fp8 != 0 && (d->proj_fp8 != 1 || d->dtype != FSDIT_BF16)) {
    set_error("dims.proj_fp8 must be 0, or 1 with dtype FSDIT_BF16");
    return FSDIT_E_DTYPE;
  }
  return FSDIT_OK;
}

static EpiParams make_ep(const fsdit_dims* d, int epi, const void* bias, void* out, int ldo, const float* resid,
                         const int32_t* pos) {
  EpiParams e;
  e.epi = epi;
  e.bias = bias;
  e.out = out;
  e.ldo = ldo;
  e.resid = resid;
  e.ldr = ldo;
  e.pos = pos;
  e.rope_cs = nullptr;
  e.rope_cols = 2 * attn_dim(d);
  e.head_dim = d->head_dim;
  e.s0 = d->rope_split[0];
  e.s1 = d->rope_split[1];
  e.log2_theta = log2f(d->rope_theta);
  e.row_scale = nullptr;
  e.col_scale = nullptr;
  e.up_h = e.up_w = e.up_c = e.up_pt = e.up_ps = 1;
  e.up_rgb8 = 0;
  e.split_part = nullptr;
  e.split_cnt = nullptr;
  return e;
}

fsdit_status launch_linear(const fsdit_dims* d, const void* a, const void* w, const EpiParams& ep, int M, int N,
                           int K, cudaStream_t st, int prof_cls) {
  if (M <= 0) return FSDIT_OK;
  static const int cls_of[6] = {PC_GEMM_BIAS, PC_GEMM_BIAS_F32, PC_GEMM_QKV, PC_GEMM_GELU, PC_GEMM_RESID,
                                PC_PIXEL_HEAD};
  const double s = (double)dsize(d->dtype);
  const double out_b = ep.epi == EPI_UNPATCH ? (ep.up_rgb8 ? 1.0 : 4.0)
                      : (ep.epi == FSDIT_EPI_RESIDUAL || ep.epi == FSDIT_EPI_BIAS_F32) ? 4.0
                                                                                        : s;
  const double by = ((double)M * K + (double)N * K) * s + (double)M * N * out_b +
                    (ep.epi == FSDIT_EPI_RESIDUAL ? (double)M * N * 4.0 : 0.0);
  ProfScope ps(prof_cls >= 0 ? prof_cls : cls_of[ep.epi], 1, 2.0 * M * N * K, by, st);
  t_scope = &ps;
  const fsdit_status r = d->dtype == FSDIT_BF16 ? launch_linear_tc(a, w, ep, M, N, K, st)
                                                : launch_linear_simt(FSDIT_F32, a, w, ep, M, N, K, st);
  t_scope = nullptr;
  return r;
}

fsdit_status launch_linear_fp8(const fsdit_dims* d, const uint8_t* qa, const void* qw, const EpiParams& ep, int M,
                               int N, int K, cudaStream_t st) {
  if (M <= 0) return FSDIT_OK;
  const int cls = ep.epi == FSDIT_EPI_QKV_ROPE ? PC_GEMM_FP8_QKV
                  : ep.epi == FSDIT_EPI_GELU   ? PC_GEMM_FP8_GELU
                                               : PC_GEMM_FP8_RESID;
  const double out_b = (ep.epi == FSDIT_EPI_RESIDUAL || ep.epi == FSDIT_EPI_BIAS_F32) ? 4.0 : 2.0;
  const double by = (double)M * K + (double)N * K + (double)M * N * out_b +
                    (ep.epi == FSDIT_EPI_RESIDUAL ? (double)M * N * 4.0 : 0.0);
  ProfScope ps(cls, 1, 2.0 * M * N * K, by, st);
  (void)d;
  t_scope = &ps;
  const fsdit_status r = launch_linear_fp8_tc(qa, (const uint8_t*)qw, ep, M, N, K, st);
  t_scope = nullptr;
  return r;
}

fsdit_status launch_attention(const fsdit_dims* d, const void* qkv, void* out, int n, cudaStream_t st) {
  if (n <= 0) return FSDIT_OK;
  ProfScope ps(PC_ATTN, 1, 4.0 * n * (double)n * attn_dim(d), 4.0 * n * (double)attn_dim(d) * dsize(d->dtype), st);
  if (d->dtype == FSDIT_BF16)
    return n >= attention_pair_min_rows() ? launch_attention_pair(qkv, out, n, d->heads, attn_dim(d), st)
                                           : launch_attention_tc(qkv, out, n, d->heads, attn_dim(d), st);
  return launch_attention_simt(FSDIT_F32, qkv, out, n, d->heads, attn_dim(d), st);
}

// ---------------------------------------------------------------- workspace
struct Carve {
  uint8_t* base;
  size_t off;
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off += (bytes + 255) & ~(size_t)255;
    return p;
  }
};

struct BlockWs {  // every buffer null until a carve sets it
  float* xc = nullptr;       // [n_c, hidden] compressed residual (compressed mode)
  int32_t* posc = nullptr;   // [n_c, 3]
  void* xn = nullptr;        // [n, max(hidden, attn)] GEMM operand (normalized x / attention output)
  void* qkv = nullptr;       // [n, 3 attn]
  void* u = nullptr;         // [n, ffn]
  float2* rope = nullptr;    // [n, head_dim/2] (cos, sin) table of the rows' positions
  float2* rope_c = nullptr;  // stack only: table of the compressed rows
  uint8_t* q8 = nullptr;     // FP8 projections: [n, max(hidden, attn, ffn)] E4M3 operand
  float* sa = nullptr;       //                  [n] its row scales
  float* ss = nullptr;       // RMSNorm after the GEMM: [n, hidden/128] sums of squares per column group
};

// Blocks run back to back (stack, decoder) apply each RMSNorm after the GEMM
// that consumes it: the residual epilogue before the norm writes bf16(x * g)
// and per-group sums of squares, and the consuming GEMM forms 1/rms of each
// row from those sums and scales its accumulators by it.  bf16 tensor-core
// projections with hidden % 128 == 0 only.
static int g_norm_after_gemm = 1;  // fsdit_set_norm_after_gemm
static bool norm_after_gemm(const fsdit_dims* d) {
  return g_norm_after_gemm != 0 && d->dtype == FSDIT_BF16 && !d->proj_fp8 && d->hidden % 128 == 0;
}

static void carve_norm(Carve& c, const fsdit_dims* d, int n_rows, BlockWs& w) {
  if (!norm_after_gemm(d)) return;
  w.ss = (float*)c.take((size_t)n_rows * (d->hidden / 128) * 4);
}

static BlockWs carve_block(Carve& c, const fsdit_dims* d, int n_rows, int n_c, bool compressed) {
  BlockWs w;
  const int n = compressed ? n_c : n_rows;
  w.xc = compressed ? (float*)c.take((size_t)n_c * d->hidden * 4) : nullptr;
  w.posc = compressed ? (int32_t*)c.take((size_t)n_c * 3 * 4) : nullptr;
  const int wide = d->hidden > attn_dim(d) ? d->hidden : attn_dim(d);
  w.xn = c.take((size_t)n * wide * dsize(d->dtype));
  w.qkv = c.take((size_t)n * 3 * attn_dim(d) * dsize(d->dtype));
  w.u = c.take((size_t)n * d->ffn * dsize(d->dtype));
  w.rope = (float2*)c.take((size_t)n * (d->head_dim / 2) * sizeof(float2));
  w.rope_c = nullptr;
  w.q8 = nullptr;
  w.sa = nullptr;
  if (d->proj_fp8) {
    const int k8 = wide > d->ffn ? wide : d->ffn;
    w.q8 = (uint8_t*)c.take((size_t)n * k8);
    w.sa = (float*)c.take((size_t)n * 4);
  }
  return w;
}

// ---------------------------------------------------------------- block body
// x[n, hidden] (fp32, in place): x += attn(...); x += ffn(...).
static fsdit_status rope_table(const fsdit_dims* d, const int32_t* pos, int rows, float2* cs, cudaStream_t st) {
  return launch_rope_table(pos, rows, d->head_dim, d->rope_split[0], d->rope_split[1], log2f(d->rope_theta), cs, st);
}

// x_in -> x_out over n rows; `rope` is the (cos, sin) table of the rows' positions.
// E4M3 projections: each GEMM operand is quantized per row (RMSNorm fused with
// it for the QKV and FFN-up inputs; a separate pass over the bf16 attention
// and GELU outputs for the O and FFN-down inputs); the weights carry their
// per-output-channel scales; the epilogue dequantizes before the bias.
static fsdit_status block_body_fp8(const fsdit_dims* d, const fsdit_block_weights* w, float* x_in, float* x_out,
                                   const int32_t* pos, const float2* rope, int n, const BlockWs& ws,
                                   cudaStream_t st) {
  const int H = d->hidden, F = d->ffn, A = attn_dim(d);
  if (ws.q8 == nullptr || ws.sa == nullptr) {
    set_error("FP8 projections: the workspace has no quantized-operand buffers");
    return FSDIT_E_WORKSPACE;
  }
  auto scaled = [&](EpiParams e, const float* col_scale) {
    e.row_scale = ws.sa;
    e.col_scale = col_scale;
    return e;
  };
  FS_TRY(launch_rmsnorm_quant(x_in, w->g_attn, n, H, d->rms_eps, ws.q8, ws.sa, st));
  EpiParams qkv_ep = scaled(make_ep(d, FSDIT_EPI_QKV_ROPE, w->b_qkv, ws.qkv, 3 * A, nullptr, pos), w->s_qkv);
  qkv_ep.rope_cs = rope;
  FS_TRY(launch_linear_fp8(d, ws.q8, w->w_qkv, qkv_ep, n, 3 * A, H, st));
  FS_TRY(launch_attention(d, ws.qkv, ws.xn, n, st));
  FS_TRY(launch_quant_rows(ws.xn, FSDIT_BF16, n, A, ws.q8, ws.sa, st));
  FS_TRY(launch_linear_fp8(d, ws.q8, w->w_o,
                           scaled(make_ep(d, FSDIT_EPI_RESIDUAL, w->b_o, x_out, H, x_in, nullptr), w->s_o), n, H, A,
                           st));
  FS_TRY(launch_rmsnorm_quant(x_out, w->g_ffn, n, H, d->rms_eps, ws.q8, ws.sa, st));
  FS_TRY(launch_linear_fp8(d, ws.q8, w->w_1, scaled(make_ep(d, FSDIT_EPI_GELU, w->b_1, ws.u, F, nullptr, nullptr),
                                                    w->s_1),
                           n, F, H, st));
  FS_TRY(launch_quant_rows(ws.u, FSDIT_BF16, n, F, ws.q8, ws.sa, st));
  FS_TRY(launch_linear_fp8(d, ws.q8, w->w_2,
                           scaled(make_ep(d, FSDIT_EPI_RESIDUAL, w->b_2, x_out, H, x_out, nullptr), w->s_2), n, H, F,
                           st));
  return FSDIT_OK;
}

// in_ready: ws.xn already holds bf16(x_in * g_attn) and ws.ss its sums of
// squares (the previous block's FFN-down epilogue wrote them).  g_next: the
// gain of the norm that follows this block on the same rows, or null; the
// FFN-down epilogue then prepares it and *out_ready is set.
static fsdit_status block_body(const fsdit_dims* d, const fsdit_block_weights* w, float* x_in, float* x_out,
                               const int32_t* pos, const float2* rope, int n, const BlockWs& ws, cudaStream_t st,
                               bool in_ready = false, const void* g_next = nullptr, bool* out_ready = nullptr) {
  if (out_ready) *out_ready = false;
  if (d->proj_fp8) return block_body_fp8(d, w, x_in, x_out, pos, rope, n, ws, st);
  const int H = d->hidden, F = d->ffn, A = attn_dim(d);
  const bool fuse = ws.ss != nullptr;
  auto produce = [&](EpiParams e, void* xg, const void* gain) {
    e.xg = reinterpret_cast<bf16*>(xg);
    e.xg_gain = reinterpret_cast<const bf16*>(gain);
    e.ss_part = ws.ss;
    e.ss_ld = H / 128;
    return e;
  };
  auto consume = [&](EpiParams& e) {
    e.norm_ss = ws.ss;
    e.ss_ld = H / 128;
    e.norm_h = H;
    e.norm_eps = d->rms_eps;
  };
  EpiParams qkv_ep = make_ep(d, FSDIT_EPI_QKV_ROPE, w->b_qkv, ws.qkv, 3 * A, nullptr, pos);
  qkv_ep.rope_cs = rope;
  if (fuse && in_ready) {
    consume(qkv_ep);
  } else {
    FS_TRY(launch_rmsnorm_cast(x_in, w->g_attn, ws.xn, n, H, d->rms_eps, d->dtype, st));
  }
  FS_TRY(launch_linear(d, ws.xn, w->w_qkv, qkv_ep, n, 3 * A, H, st));
  FS_TRY(launch_attention(d, ws.qkv, ws.xn, n, st));
  // the FFN norm's operand goes to the qkv buffer (free after attention; the
  // O projection still reads xn)
  EpiParams o_ep = make_ep(d, FSDIT_EPI_RESIDUAL, w->b_o, x_out, H, x_in, nullptr);
  if (fuse) o_ep = produce(o_ep, ws.qkv, w->g_ffn);
  FS_TRY(launch_linear(d, ws.xn, w->w_o, o_ep, n, H, A, st));
  EpiParams up_ep = make_ep(d, FSDIT_EPI_GELU, w->b_1, ws.u, F, nullptr, nullptr);
  const void* up_a = ws.xn;
  if (fuse) {
    consume(up_ep);
    up_a = ws.qkv;
  } else {
    FS_TRY(launch_rmsnorm_cast(x_out, w->g_ffn, ws.xn, n, H, d->rms_eps, d->dtype, st));
  }
  FS_TRY(launch_linear(d, up_a, w->w_1, up_ep, n, F, H, st));
  // the next block's attention-norm operand goes to xn (FFN-down reads u)
  EpiParams down_ep = make_ep(d, FSDIT_EPI_RESIDUAL, w->b_2, x_out, H, x_out, nullptr);
  if (fuse && g_next != nullptr) down_ep = produce(down_ep, ws.xn, g_next);
  FS_TRY(launch_linear(d, ws.u, w->w_2, down_ep, n, H, F, st));
  if (out_ready) *out_ready = fuse && g_next != nullptr;
  return FSDIT_OK;
}

static fsdit_status check_block_weights(const fsdit_dims* d, const fsdit_block_weights* w) {
  FS_TRY(need(w, "weights"));
  if (d->proj_fp8) {
    FS_TRY(need(w->s_qkv, "s_qkv"));
    FS_TRY(need(w->s_o, "s_o"));
    FS_TRY(need(w->s_1, "s_1"));
    FS_TRY(need(w->s_2, "s_2"));
  }
  FS_TRY(need(w->w_qkv, "w_qkv"));
  FS_TRY(need(w->b_qkv, "b_qkv"));
  FS_TRY(need(w->w_o, "w_o"));
  FS_TRY(need(w->b_o, "b_o"));
  FS_TRY(need(w->w_1, "w_1"));
  FS_TRY(need(w->b_1, "b_1"));
  FS_TRY(need(w->w_2, "w_2"));
  FS_TRY(need(w->b_2, "b_2"));
  FS_TRY(need(w->g_attn, "g_attn"));
  FS_TRY(need(w->g_ffn, "g_ffn"));
  return FSDIT_OK;
}

static fsdit_status check_tokens(const fsdit_tokens* t, bool need_tags) {
  FS_TRY(need(t, "tokens"));
  if (t->n_tokens <= 0 || t->n_vrows < 0 || t->n_text < 0 || t->n_audio < 0 ||
      t->n_vrows + t->n_text + t->n_audio != t->n_tokens) {
    set_error("tokens: n_tokens (%d) must be n_vrows + n_text + n_audio (%d+%d+%d) and positive", t->n_tokens,
              t->n_vrows, t->n_text, t->n_audio);
    return FSDIT_E_SHAPE;
  }
  if (t->grid_t < 0 || t->grid_h < 0 || t->grid_w < 0 ||
      (long long)t->grid_t * t->grid_h * t->grid_w > (long long)t->n_vrows) {
    set_error("tokens: grid %dx%dx%d does not fit in the %d video rows", t->grid_t, t->grid_h, t->grid_w, t->n_vrows);
    return FSDIT_E_SHAPE;
  }
  FS_TRY(need(t->pos_thw, "tokens.pos_thw"));
  if (need_tags) {
    if (t->modality == nullptr || t->time_id == nullptr || t->out_mask == nullptr) {
      set_error("tokens: modality, time_id and out_mask are required");
      return FSDIT_E_NULL;
    }
  }
  if (t->keep_idx != nullptr) {
    const int n_grid = t->grid_t * t->grid_h * t->grid_w;
    if (n_grid <= 0 || t->near_idx == nullptr || t->n_keep != fsdit_keep_count(t->grid_t, t->grid_h, t->grid_w)) {
      set_error("tokens: keep map needs a non-empty grid, near_idx and n_keep == %d (got %d)",
                n_grid > 0 ? fsdit_keep_count(t->grid_t, t->grid_h, t->grid_w) : 0, t->n_keep);
      return FSDIT_E_SHAPE;
    }
    if (!aligned16(t->keep_idx) || !aligned16(t->near_idx)) {
      set_error("tokens: keep_idx / near_idx must be 16-byte aligned");
      return FSDIT_E_ALIGN;
    }
  }
  return FSDIT_OK;
}

static int n_compressed(const fsdit_tokens* t) {
  const int n_grid = t->grid_t * t->grid_h * t->grid_w;
  return t->n_keep + (t->n_tokens - n_grid);
}

}  // namespace fsdit

using namespace fsdit;

// ================================================================ C ABI

extern "C" {

const char* fsdit_last_error(void) { return t_err; }

fsdit_status fsdit_profile_start(int max_launches) {
  if (max_launches <= 0) {
    set_error("profile: max_launches must be positive");
    return FSDIT_E_SHAPE;
  }
  const size_t need_ev = 2 * (size_t)max_launches;
  while (g_prof.ev.size() < need_ev) {
    cudaEvent_t e;
    FS_TRY(cuda_check(cudaEventCreate(&e), "cudaEventCreate"));
    g_prof.ev.push_back(e);
  }
  g_prof.cls.assign(max_launches, 0);
  g_prof.kernels.assign(max_launches, 0);
  g_prof.flops.assign(max_launches, 0.0);
  g_prof.bytes.assign(max_launches, 0.0);
  g_prof.used = 0;
  g_prof.on = true;
  return FSDIT_OK;
}

int fsdit_profile_stop(fsdit_prof_entry* entries, int max_entries) {
  g_prof.on = false;
  if (g_prof.used == 0) return 0;
  if (cuda_check(cudaEventSynchronize(g_prof.ev[2 * (g_prof.used - 1) + 1]), "cudaEventSynchronize") != FSDIT_OK)
    return FSDIT_E_CUDA;
  fsdit_prof_entry acc[PC_COUNT];
  memset(acc, 0, sizeof(acc));
  for (int i = 0; i < g_prof.used; ++i) {
    float ms = 0.f;
    if (cuda_check(cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]), "cudaEventElapsedTime") !=
        FSDIT_OK)
      return FSDIT_E_CUDA;
    fsdit_prof_entry& e = acc[g_prof.cls[i]];
    e.scopes += 1;
    e.launches += g_prof.kernels[i];
    e.ms += ms;
    e.flops += g_prof.flops[i];
    e.bytes += g_prof.bytes[i];
  }
  int n = 0;
  for (int c = 0; c < PC_COUNT; ++c) {
    if (acc[c].scopes == 0) continue;
    if (entries != nullptr && n < max_entries) {
      entries[n] = acc[c];
      snprintf(entries[n].name, sizeof(entries[n].name), "%s", kProfNames[c]);
    }
    ++n;
  }
  g_prof.used = 0;
  return n;
}
const char* fsdit_version(void) { return "fsdit 0.1 sm_100a"; }

fsdit_status fsdit_device_error(fsdit_stream_t stream) {
  FS_TRY(cuda_check(cudaStreamSynchronize((cudaStream_t)stream), "cudaStreamSynchronize"));
  int v = 0;
  FS_TRY(cuda_check(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)), "read device error word"));
  if (v != 0) {
    int z = 0;
    FS_TRY(cuda_check(cudaMemcpyToSymbol(g_device_error, &z, sizeof(int)), "clear device error word"));
    set_error("device error word 0x%x (%s%s%s)", v, (v & DEVERR_TIMEOUT) ? "bounded wait timed out; " : "",
              (v & DEVERR_TAGS) ? "row tags inconsistent with segments; " : "",
              (v & DEVERR_KEEPMAP) ? "keep_idx / near_idx entry outside the grid or not a nearest-kept map; "
                                   : "");
    return (v & DEVERR_TIMEOUT) ? FSDIT_E_TIMEOUT : FSDIT_E_SHAPE;
  }
  return FSDIT_OK;
}

int fsdit_keep_count(int T, int H, int W) {
  if (T <= 0 || H <= 0 || W <= 0) return 0;
  return T * (H / 2 + 1) * (W / 2 + 1);
}

size_t fsdit_block_workspace_size(const fsdit_dims* dims, int n_tokens, int n_keep) {
  if (check_dims(dims) != FSDIT_OK || n_tokens <= 0) return 0;
  Carve c{nullptr, 0};
  // n_keep > 0 -> compressed; the compressed row count is bounded by n_tokens
  carve_block(c, dims, n_tokens, n_tokens, n_keep > 0);
  return c.off;
}

static size_t stack_carve(Carve& c, const fsdit_dims* d, const fsdit_io_weights* io, const fsdit_tokens* t,
                          int n_times, float** x, float** temb, float** h1, float** tproj, float** vv, float** va,
                          BlockWs* bw) {
  const int N = t->n_tokens;
  const bool comp = t->keep_idx != nullptr;
  *x = (float*)c.take((size_t)N * d->hidden * 4);
  *temb = (float*)c.take((size_t)n_times * d->hidden * 4);
  *h1 = (float*)c.take((size_t)n_times * d->hidden * 4);
  *tproj = (float*)c.take((size_t)(t->n_text > 0 ? t->n_text : 1) * d->hidden * 4);
  *vv = (float*)c.take((size_t)(t->n_vrows > 0 ? t->n_vrows : 1) * io->c_video * 4);
  *va = (float*)c.take((size_t)(t->n_audio > 0 ? t->n_audio : 1) * io->c_audio * 4);
  // block buffers sized for the full sequence; the compressed residual needs n_c rows
  const int n_c = comp ? n_compressed(t) : 0;
  BlockWs w;
  w.xc = comp ? (float*)c.take((size_t)n_c * d->hidden * 4) : nullptr;
  w.posc = comp ? (int32_t*)c.take((size_t)n_c * 3 * 4) : nullptr;
  const int wide = d->hidden > attn_dim(d) ? d->hidden : attn_dim(d);
  w.xn = c.take((size_t)N * wide * dsize(d->dtype));
  w.qkv = c.take((size_t)N * 3 * attn_dim(d) * dsize(d->dtype));
  w.u = c.take((size_t)N * d->ffn * dsize(d->dtype));
  w.rope = (float2*)c.take((size_t)N * (d->head_dim / 2) * sizeof(float2));
  w.rope_c = comp ? (float2*)c.take((size_t)n_c * (d->head_dim / 2) * sizeof(float2)) : nullptr;
  w.q8 = nullptr;
  w.sa = nullptr;
  if (d->proj_fp8) {
    const int k8 = wide > d->ffn ? wide : d->ffn;
    w.q8 = (uint8_t*)c.take((size_t)N * k8);
    w.sa = (float*)c.take((size_t)N * 4);
  }
  carve_norm(c, d, N, w);
  *bw = w;
  return c.off;
}

size_t fsdit_stack_workspace_size(const fsdit_dims* dims, const fsdit_io_weights* io, const fsdit_tokens* tok,
                                  int n_times) {
  if (check_dims(dims) != FSDIT_OK || io == nullptr || check_tokens(tok, false) != FSDIT_OK) return 0;
  Carve c{nullptr, 0};
  float *x, *temb, *h1, *tp, *vv, *va;
  BlockWs bw;
  return stack_carve(c, dims, io, tok, n_times > 0 ? n_times : 1, &x, &temb, &h1, &tp, &vv, &va, &bw);
}

fsdit_status fsdit_build_keep_map(int T, int H, int W, int32_t* keep_idx, int32_t* near_idx, fsdit_stream_t stream) {
  if (T <= 0 || H <= 0 || W <= 0) {
    set_error("keep map: grid %dx%dx%d must be non-empty", T, H, W);
    return FSDIT_E_SHAPE;
  }
  FS_TRY(need(keep_idx, "keep_idx"));
  FS_TRY(need(near_idx, "near_idx"));
  return launch_keep_map(T, H, W, keep_idx, near_idx, (cudaStream_t)stream);
}

fsdit_status fsdit_gather_rows(const float* x, const int32_t* pos, float* x_c, int32_t* pos_c, const int32_t* keep_idx,
                               int n_keep, int n_grid, int n_rows, int hidden, fsdit_stream_t stream) {
  FS_TRY(need(x, "x"));
  FS_TRY(need(x_c, "x_c"));
  FS_TRY(need(keep_idx, "keep_idx"));
  if ((pos == nullptr) != (pos_c == nullptr)) {
    set_error("pos and pos_c must both be given or both be NULL");
    return FSDIT_E_NULL;
  }
  if (n_keep <= 0 || n_grid < n_keep || n_rows < n_grid || hidden <= 0 || hidden % 4 != 0) {
    set_error("gather: need 0 < n_keep <= n_grid <= n_rows and hidden %% 4 == 0");
    return FSDIT_E_SHAPE;
  }
  return launch_gather(x, pos, x_c, pos_c, keep_idx, n_keep, n_grid, n_rows, hidden, (cudaStream_t)stream);
}

fsdit_status fsdit_broadcast_residual(const float* x, const float* y_c, float* out, const int32_t* keep_idx,
                                      const int32_t* near_idx, int n_keep, int grid_t, int grid_h, int grid_w,
                                      int n_rows, int hidden, fsdit_stream_t stream) {
  FS_TRY(need(x, "x"));
  FS_TRY(need(y_c, "y_c"));
  FS_TRY(need(out, "out"));
  FS_TRY(need(keep_idx, "keep_idx"));
  FS_TRY(need(near_idx, "near_idx"));
  const long long n_grid = (long long)grid_t * grid_h * grid_w;
  if (grid_t <= 0 || grid_h <= 0 || grid_w <= 0 || n_keep != fsdit_keep_count(grid_t, grid_h, grid_w) ||
      n_rows < n_grid || hidden <= 0 || hidden % 4 != 0) {
    set_error("broadcast: need a non-empty grid, n_keep == its kept count, n_rows >= grid rows, hidden %% 4 == 0");
    return FSDIT_E_SHAPE;
  }
  if (out == y_c) {
    set_error("broadcast: out must not alias y_c");
    return FSDIT_E_SHAPE;
  }
  return launch_broadcast(x, y_c, out, keep_idx, near_idx, n_keep, grid_t, grid_h, grid_w, n_rows, hidden,
                          (cudaStream_t)stream);
}

fsdit_status fsdit_rmsnorm_cast(const float* x, const void* g, void* xn, int rows, int hidden, float eps, int dtype,
                                fsdit_stream_t stream) {
  FS_TRY(need(x, "x"));
  FS_TRY(need(g, "g"));
  FS_TRY(need(xn, "xn"));
  if (dtype != FSDIT_F32 && dtype != FSDIT_BF16) {
    set_error("rmsnorm_cast: bad dtype %d", dtype);
    return FSDIT_E_DTYPE;
  }
  if (rows < 0 || hidden <= 0 || hidden % 8 != 0 || hidden > 8192) {
    set_error("rmsnorm_cast: need hidden %% 8 == 0 and hidden <= 8192");
    return FSDIT_E_SHAPE;
  }
  if (rows == 0) return FSDIT_OK;
  return launch_rmsnorm_cast(x, g, xn, rows, hidden, eps, dtype, (cudaStream_t)stream);
}

size_t fsdit_gemm_scratch_size(void) { return SPLIT_WS_BYTES + SPLIT_CNT_BYTES; }

}  // extern "C"

namespace fsdit {
// Point `ep` at caller scratch for the pair GEMM's tail cut and zero its
// counters (nothing when scratch is null).
static fsdit_status attach_scratch(EpiParams& ep, void* scratch, size_t bytes, cudaStream_t st) {
  if (scratch == nullptr) return FSDIT_OK;
  if (bytes < SPLIT_WS_BYTES + SPLIT_CNT_BYTES) {
    set_error("GEMM scratch: need %zu bytes, got %zu", SPLIT_WS_BYTES + SPLIT_CNT_BYTES, bytes);
    return FSDIT_E_WORKSPACE;
  }
  if (!aligned16(scratch)) {
    set_error("GEMM scratch must be 16-byte aligned");
    return FSDIT_E_ALIGN;
  }
  ep.split_part = (float*)scratch;
  ep.split_cnt = (int*)((uint8_t*)scratch + SPLIT_WS_BYTES);
  return cuda_check(cudaMemsetAsync(ep.split_cnt, 0, SPLIT_CNT_BYTES, st), "cudaMemsetAsync(GEMM scratch counters)");
}
}  // namespace fsdit

extern "C" {

fsdit_status fsdit_linear(const fsdit_dims* dims, const void* a, const void* w, const void* b, void* out,
                          const float* resid, const int32_t* pos, int M, int N, int K, int epilogue,
                          fsdit_stream_t stream) {
  return fsdit_linear_ws(dims, a, w, b, out, resid, pos, M, N, K, epilogue, nullptr, 0, stream);
}

fsdit_status fsdit_linear_ws(const fsdit_dims* dims, const void* a, const void* w, const void* b, void* out,
                             const float* resid, const int32_t* pos, int M, int N, int K, int epilogue,
                             void* scratch, size_t scratch_bytes, fsdit_stream_t stream) {
  FS_TRY(check_dims(dims));
  FS_TRY(need(a, "a"));
  FS_TRY(need(w, "w"));
  FS_TRY(need(b, "b"));
  FS_TRY(need(out, "out"));
  if (M < 0 || N <= 0 || K <= 0 || K % 8 != 0 || N % 32 != 0) {
    set_error("linear: need M >= 0, N %% 32 == 0, K %% 8 == 0 (got %d %d %d)", M, N, K);
    return FSDIT_E_SHAPE;
  }
  if (epilogue < FSDIT_EPI_BIAS || epilogue > FSDIT_EPI_RESIDUAL) {
    set_error("linear: unknown epilogue %d", epilogue);
    return FSDIT_E_SHAPE;
  }
  if (epilogue == FSDIT_EPI_RESIDUAL) FS_TRY(need(resid, "resid"));
  if (epilogue == FSDIT_EPI_QKV_ROPE) {
    FS_TRY(need(pos, "pos"));
    if (N != 3 * attn_dim(dims)) {
      set_error("linear: the RoPE epilogue needs N == 3*heads*head_dim");
      return FSDIT_E_SHAPE;
    }
  }
  EpiParams ep = make_ep(dims, epilogue, b, out, N, resid, pos);
  FS_TRY(attach_scratch(ep, scratch, scratch_bytes, (cudaStream_t)stream));
  return launch_linear(dims, a, w, ep, M, N, K, (cudaStream_t)stream);
}



fsdit_status fsdit_quantize_rows(const void* a, int dtype, int rows, int cols, uint8_t* q, float* s,
                                 fsdit_stream_t stream) {
  FS_TRY(need(a, "a"));
  FS_TRY(need(q, "q"));
  FS_TRY(need(s, "s"));
  if (dtype != FSDIT_F32 && dtype != FSDIT_BF16) {
    set_error("quantize_rows: bad dtype %d", dtype);
    return FSDIT_E_DTYPE;
  }
  if (rows < 0 || cols <= 0 || cols % 16 != 0) {
    set_error("quantize_rows: need rows >= 0, cols > 0, cols %% 16 == 0 (got %d %d)", rows, cols);
    return FSDIT_E_SHAPE;
  }
  if (!aligned16(a) || !aligned16(q)) {
    set_error("quantize_rows: a and q must be 16-byte aligned");
    return FSDIT_E_ALIGN;
  }
  return launch_quant_rows(a, dtype, rows, cols, q, s, (cudaStream_t)stream);
}

fsdit_status fsdit_rmsnorm_quant(const float* x, const void* g, int rows, int hidden, float eps, uint8_t* q, float* s,
                                 fsdit_stream_t stream) {
  FS_TRY(need(x, "x"));
  FS_TRY(need(g, "g"));
  FS_TRY(need(q, "q"));
  FS_TRY(need(s, "s"));
  if (rows < 0 || hidden <= 0 || hidden % 64 != 0 || hidden > 8192 || !(eps >= 0.f)) {
    set_error("rmsnorm_quant: need rows >= 0, hidden %% 64 == 0, hidden <= 8192, eps >= 0");
    return FSDIT_E_SHAPE;
  }
  if (!aligned16(x) || !aligned16(q)) {
    set_error("rmsnorm_quant: x and q must be 16-byte aligned");
    return FSDIT_E_ALIGN;
  }
  return launch_rmsnorm_quant(x, g, rows, hidden, eps, q, s, (cudaStream_t)stream);
}

fsdit_status fsdit_linear_fp8(const fsdit_dims* dims, const uint8_t* qa, const float* sa, const uint8_t* qw,
                              const float* sw, const void* b, void* out, const float* resid, const int32_t* pos, int M,
                              int N, int K, int epilogue, fsdit_stream_t stream) {
  return fsdit_linear_fp8_ws(dims, qa, sa, qw, sw, b, out, resid, pos, M, N, K, epilogue, nullptr, 0, stream);
}

fsdit_status fsdit_linear_fp8_ws(const fsdit_dims* dims, const uint8_t* qa, const float* sa, const uint8_t* qw,
                                 const float* sw, const void* b, void* out, const float* resid, const int32_t* pos,
                                 int M, int N, int K, int epilogue, void* scratch, size_t scratch_bytes,
                                 fsdit_stream_t stream) {
  FS_TRY(check_dims(dims));
  if (dims->dtype != FSDIT_BF16) {
    set_error("linear_fp8: dims.dtype must be FSDIT_BF16 (bias, outputs)");
    return FSDIT_E_DTYPE;
  }
  FS_TRY(need(qa, "qa"));
  FS_TRY(need(sa, "sa"));
  FS_TRY(need(qw, "qw"));
  FS_TRY(need(sw, "sw"));
  FS_TRY(need(b, "b"));
  FS_TRY(need(out, "out"));
  if (M < 0 || N <= 0 || K <= 0 || K % 16 != 0 || N % 32 != 0) {
    set_error("linear_fp8: need M >= 0, N %% 32 == 0, K %% 16 == 0 (got %d %d %d)", M, N, K);
    return FSDIT_E_SHAPE;
  }
  if (epilogue < FSDIT_EPI_BIAS || epilogue > FSDIT_EPI_RESIDUAL) {
    set_error("linear_fp8: unknown epilogue %d", epilogue);
    return FSDIT_E_SHAPE;
  }
  if (epilogue == FSDIT_EPI_RESIDUAL) FS_TRY(need(resid, "resid"));
  if (epilogue == FSDIT_EPI_QKV_ROPE) {
    FS_TRY(need(pos, "pos"));
    if (N != 3 * attn_dim(dims)) {
      set_error("linear_fp8: the RoPE epilogue needs N == 3*heads*head_dim");
      return FSDIT_E_SHAPE;
    }
  }
  if (!aligned16(qa) || !aligned16(qw) || !aligned16(sw) || !aligned16(b) || !aligned16(out) ||
      (resid != nullptr && !aligned16(resid))) {
    set_error("linear_fp8: qa, qw, sw, b, out and resid must be 16-byte aligned");
    return FSDIT_E_ALIGN;
  }
  EpiParams ep = make_ep(dims, epilogue, b, out, N, resid, pos);
  ep.row_scale = sa;
  ep.col_scale = sw;
  FS_TRY(attach_scratch(ep, scratch, scratch_bytes, (cudaStream_t)stream));
  return launch_linear_fp8(dims, qa, qw, ep, M, N, K, (cudaStream_t)stream);
}

fsdit_status fsdit_set_norm_after_gemm(int on) {
  if (on != 0 && on != 1) {
    set_error("set_norm_after_gemm: on must be 0 or 1, got %d", on);
    return FSDIT_E_SHAPE;
  }
  g_norm_after_gemm = on;
  return FSDIT_OK;
}

int fsdit_norm_after_gemm(void) { return g_norm_after_gemm; }

fsdit_status fsdit_attention(const fsdit_dims* dims, const void* qkv, void* out, int n, fsdit_stream_t stream) {
  FS_TRY(check_dims(dims));
  FS_TRY(need(qkv, "qkv"));
  FS_TRY(need(out, "out"));
  if (n < 0) {
    set_error("attention: n < 0");
    return FSDIT_E_SHAPE;
  }
  return launch_attention(dims, qkv, out, n, (cudaStream_t)stream);
}

fsdit_status dit_block_forward(const fsdit_dims* dims, const fsdit_block_weights* w, const fsdit_tokens* tok,
                               const float* x_in, float* x_out, void* workspace, size_t ws_bytes,
                               fsdit_stream_t stream) {
  FS_TRY(check_dims(dims));
  FS_TRY(check_block_weights(dims, w));
  FS_TRY(check_tokens(tok, false));
  FS_TRY(need(x_in, "x_in"));
  FS_TRY(need(x_out, "x_out"));
  FS_TRY(need(workspace, "workspace"));
  cudaStream_t st = (cudaStream_t)stream;
  const bool comp = tok->keep_idx != nullptr;
  const int n = tok->n_tokens;
  const int n_grid = tok->grid_t * tok->grid_h * tok->grid_w;
  const int n_c = comp ? n_compressed(tok) : n;
  Carve c{(uint8_t*)workspace, 0};
  BlockWs ws = carve_block(c, dims, n, n_c, comp);
  if (c.off > ws_bytes) {
    set_error("workspace: need %zu bytes, got %zu", c.off, ws_bytes);
    return FSDIT_E_WORKSPACE;
  }
  if (!comp) {
    FS_TRY(rope_table(dims, tok->pos_thw, n, ws.rope, st));
    return block_body(dims, w, const_cast<float*>(x_in), x_out, tok->pos_thw, ws.rope, n, ws, st);
  }
  FS_TRY(launch_gather(x_in, tok->pos_thw, ws.xc, ws.posc, tok->keep_idx, tok->n_keep, n_grid, n, dims->hidden, st));
  FS_TRY(rope_table(dims, ws.posc, n_c, ws.rope, st));
  FS_TRY(block_body(dims, w, ws.xc, ws.xc, ws.posc, ws.rope, n_c, ws, st));
  FS_TRY(launch_broadcast(x_in, ws.xc, x_out, tok->keep_idx, tok->near_idx, tok->n_keep, tok->grid_t, tok->grid_h,
                          tok->grid_w, n, dims->hidden, st));
  return FSDIT_OK;
}

static fsdit_status check_io(const fsdit_dims* d, const fsdit_io_weights* io) {
  FS_TRY(need(io, "io"));
  const void* ptrs[] = {io->w_vin, io->b_vin, io->w_tin, io->b_tin, io->w_ain, io->b_ain, io->mod_emb, io->w_t1,
                        io->b_t1,  io->w_t2,  io->b_t2,  io->g_out, io->w_vout, io->b_vout, io->w_aout, io->b_aout};
  const char* names[] = {"w_vin", "b_vin", "w_tin", "b_tin", "w_ain", "b_ain", "mod_emb", "w_t1",
                         "b_t1",  "w_t2",  "b_t2",  "g_out", "w_vout", "b_vout", "w_aout", "b_aout"};
  for (int i = 0; i < 16; ++i) FS_TRY(need(ptrs[i], names[i]));
  if (io->c_video <= 0 || io->c_video > 64 || io->c_video % 4 != 0 || io->c_audio <= 0 || io->c_audio > 64 ||
      io->c_audio % 4 != 0 || io->c_text <= 0 || io->c_text % 8 != 0 || io->t_freq <= 0 || io->t_freq % 2 != 0 ||
      io->t_freq > 1024) {
    set_error("io: need c_video, c_audio in (0, 64] and multiples of 4, c_text %% 8 == 0, even t_freq <= 1024");
    return FSDIT_E_SHAPE;
  }
  (void)d;
  return FSDIT_OK;
}

static fsdit_status stack_forward_impl(const fsdit_dims* dims, int n_layers, const fsdit_block_weights* layers,
                                       const uint8_t* layer_compress, const fsdit_io_weights* io,
                                       const fsdit_tokens* tok, const float* time_table, int n_times,
                                       const float* video_lat, const void* text_emb, const float* audio_lat,
                                       float* v_video, float* v_audio, void* workspace, size_t ws_bytes,
                                       cudaStream_t st) {
  const int H = dims->hidden;
  Carve c{(uint8_t*)workspace, 0};
  float *x, *temb, *h1, *tproj, *vv_ws, *va_ws;
  BlockWs bw;
  stack_carve(c, dims, io, tok, n_times, &x, &temb, &h1, &tproj, &vv_ws, &va_ws, &bw);
  if (c.off > ws_bytes) {
    set_error("workspace: need %zu bytes, got %zu", c.off, ws_bytes);
    return FSDIT_E_WORKSPACE;
  }
  // embedding
  FS_TRY(launch_time_mlp(dims->dtype, time_table, n_times, io->t_freq, io->w_t1, io->b_t1, io->w_t2, io->b_t2, h1,
                         temb, H, st));
  if (tok->n_text > 0) {
    EpiParams ep = make_ep(dims, FSDIT_EPI_BIAS_F32, io->b_tin, tproj, H, nullptr, nullptr);
    FS_TRY(launch_linear(dims, text_emb, io->w_tin, ep, tok->n_text, H, io->c_text, st));
  }
  FS_TRY(launch_embed(dims->dtype, x, H, 0, tok->n_vrows, 1, video_lat, io->c_video, io->w_vin, io->b_vin, nullptr,
                      io->mod_emb, temb, tok->modality, tok->time_id, n_times, FSDIT_MOD_VIDEO, FSDIT_MOD_CONTROL, st));
  FS_TRY(launch_embed(dims->dtype, x, H, tok->n_vrows, tok->n_text, 0, nullptr, 0, nullptr, nullptr, tproj,
                      io->mod_emb, temb, tok->modality, tok->time_id, n_times, FSDIT_MOD_TEXT, FSDIT_MOD_TEXT, st));
  FS_TRY(launch_embed(dims->dtype, x, H, tok->n_vrows + tok->n_text, tok->n_audio, 1, audio_lat, io->c_audio,
                      io->w_ain, io->b_ain, nullptr, io->mod_emb, temb, tok->modality, tok->time_id, n_times,
                      FSDIT_MOD_AUDIO, FSDIT_MOD_AUDIO, st));
  // layers; a run of compressed layers is one gather .. one broadcast
  const int N = tok->n_tokens;
  const int n_grid = tok->grid_t * tok->grid_h * tok->grid_w;
  const int n_c = tok->keep_idx ? n_compressed(tok) : N;
  bool have_full_rope = false, have_comp_rope = false;
  auto compressed = [&](int i) { return layer_compress[i] && tok->keep_idx != nullptr; };
  // the next layer's attention norm is prepared by this layer's FFN-down
  // epilogue when both run on the same rows
  auto next_gain = [&](int i) -> const void* {
    return i + 1 < n_layers && compressed(i + 1) == compressed(i) ? layers[i + 1].g_attn : nullptr;
  };
  bool ready = false;
  int l = 0;
  while (l < n_layers) {
    if (!compressed(l)) {
      if (!have_full_rope) {
        FS_TRY(rope_table(dims, tok->pos_thw, N, bw.rope, st));
        have_full_rope = true;
      }
      FS_TRY(block_body(dims, &layers[l], x, x, tok->pos_thw, bw.rope, N, bw, st, ready, next_gain(l), &ready));
      ++l;
      continue;
    }
    FS_TRY(launch_gather(x, tok->pos_thw, bw.xc, bw.posc, tok->keep_idx, tok->n_keep, n_grid, N, H, st));
    if (!have_comp_rope) {
      FS_TRY(rope_table(dims, bw.posc, n_c, bw.rope_c, st));
      have_comp_rope = true;
    }
    ready = false;
    while (l < n_layers && compressed(l)) {
      FS_TRY(block_body(dims, &layers[l], bw.xc, bw.xc, bw.posc, bw.rope_c, n_c, bw, st, ready, next_gain(l),
                        &ready));
      ++l;
    }
    ready = false;
    FS_TRY(launch_broadcast(x, bw.xc, x, tok->keep_idx, tok->near_idx, tok->n_keep, tok->grid_t, tok->grid_h,
                            tok->grid_w, N, H, st));
  }
  // heads: final RMSNorm into the GEMM operand buffer, then the two projections
  FS_TRY(launch_rmsnorm_cast(x, io->g_out, bw.xn, N, H, dims->rms_eps, dims->dtype, st));
  if (tok->n_vrows > 0) {
    EpiParams ep = make_ep(dims, FSDIT_EPI_BIAS_F32, io->b_vout, v_video, io->c_video, nullptr, nullptr);
    FS_TRY(launch_linear(dims, bw.xn, io->w_vout, ep, tok->n_vrows, io->c_video, H, st, PC_HEADS));
  }
  if (tok->n_audio > 0) {
    const uint8_t* xa = (const uint8_t*)bw.xn + (size_t)(tok->n_vrows + tok->n_text) * H * dsize(dims->dtype);
    EpiParams ep = make_ep(dims, FSDIT_EPI_BIAS_F32, io->b_aout, v_audio, io->c_audio, nullptr, nullptr);
    FS_TRY(launch_linear(dims, xa, io->w_aout, ep, tok->n_audio, io->c_audio, H, st, PC_HEADS));
  }
  return FSDIT_OK;
}

static fsdit_status check_stack_args(const fsdit_dims* dims, int n_layers, const fsdit_block_weights* layers,
                                     const uint8_t* layer_compress, const fsdit_io_weights* io,
                                     const fsdit_tokens* tok, int n_times, const float* video_lat,
                                     const void* text_emb, const float* audio_lat, const void* workspace) {
  FS_TRY(check_dims(dims));
  FS_TRY(check_io(dims, io));
  FS_TRY(check_tokens(tok, true));
  if (n_layers < 0 || (n_layers > 0 && (layers == nullptr || layer_compress == nullptr))) {
    set_error("stack: n_layers >= 0 and host arrays layers / layer_compress are required");
    return FSDIT_E_NULL;
  }
  for (int l = 0; l < n_layers; ++l) FS_TRY(check_block_weights(dims, &layers[l]));
  if (n_times <= 0 || n_times > 8) {
    set_error("stack: 1 <= n_times <= 8");
    return FSDIT_E_SHAPE;
  }
  if (tok->n_vrows > 0) FS_TRY(need(video_lat, "video_lat"));
  if (tok->n_text > 0) FS_TRY(need(text_emb, "text_emb"));
  if (tok->n_audio > 0) FS_TRY(need(audio_lat, "audio_lat"));
  FS_TRY(need(workspace, "workspace"));
  return FSDIT_OK;
}

fsdit_status dit_stack_forward(const fsdit_dims* dims, int n_layers, const fsdit_block_weights* layers,
                               const uint8_t* layer_compress, const fsdit_io_weights* io, const fsdit_tokens* tok,
                               const float* time_table, int n_times, const float* video_lat, const void* text_emb,
                               const float* audio_lat, float* v_video, float* v_audio, void* workspace,
                               size_t ws_bytes, fsdit_stream_t stream) {
  FS_TRY(check_stack_args(dims, n_layers, layers, layer_compress, io, tok, n_times, video_lat, text_emb, audio_lat,
                          workspace));
  if (time_table == nullptr) {
    set_error("time_table is NULL");
    return FSDIT_E_NULL;
  }
  if (tok->n_vrows > 0) FS_TRY(need(v_video, "v_video"));
  if (tok->n_audio > 0) FS_TRY(need(v_audio, "v_audio"));
  return stack_forward_impl(dims, n_layers, layers, layer_compress, io, tok, time_table, n_times, video_lat, text_emb,
                            audio_lat, v_video, v_audio, workspace, ws_bytes, (cudaStream_t)stream);
}

fsdit_status flow_euler_step(float* x, const float* v, const uint8_t* row_modality, const uint8_t* out_mask,
                             int n_rows, int row_width, const float* t_cur, const float* t_next,
                             fsdit_stream_t stream) {
  if (n_rows < 0 || row_width <= 0) {
    set_error("euler: need n_rows >= 0 and row_width > 0");
    return FSDIT_E_SHAPE;
  }
  if (n_rows == 0) return FSDIT_OK;
  FS_TRY(need(x, "x"));
  FS_TRY(need(v, "v"));
  if (row_modality == nullptr || out_mask == nullptr || t_cur == nullptr || t_next == nullptr) {
    set_error("euler: row_modality, out_mask, t_cur and t_next are required");
    return FSDIT_E_NULL;
  }
  return launch_euler(x, v, row_modality, out_mask, n_rows, row_width, t_cur, t_next, (cudaStream_t)stream);
}

fsdit_status dit_flow_sample(const fsdit_dims* dims, int n_layers, const fsdit_block_weights* layers,
                             const uint8_t* layer_compress, const fsdit_io_weights* io, const fsdit_tokens* tok,
                             int n_evals, const float* t_video, const float* t_audio, float* video_lat,
                             const void* text_emb, float* audio_lat, void* workspace, size_t ws_bytes,
                             fsdit_stream_t stream) {
  FS_TRY(check_stack_args(dims, n_layers, layers, layer_compress, io, tok, 3, video_lat, text_emb, audio_lat,
                          workspace));
  if (n_evals <= 0 || t_video == nullptr || t_audio == nullptr) {
    set_error("sample: n_evals > 0 and host clocks t_video / t_audio [n_evals+1] are required");
    return FSDIT_E_SHAPE;
  }
  cudaStream_t st = (cudaStream_t)stream;
  Carve c{(uint8_t*)workspace, 0};
  float *x, *temb, *h1, *tproj, *vv, *va;
  BlockWs bw;
  stack_carve(c, dims, io, tok, 3, &x, &temb, &h1, &tproj, &vv, &va, &bw);
  if (c.off > ws_bytes) {
    set_error("workspace: need %zu bytes, got %zu", c.off, ws_bytes);
    return FSDIT_E_WORKSPACE;
  }
  const uint8_t* vid_mod = tok->modality;
  const uint8_t* vid_mask = tok->out_mask;
  const uint8_t* aud_mod = tok->modality + tok->n_vrows + tok->n_text;
  const uint8_t* aud_mask = tok->out_mask + tok->n_vrows + tok->n_text;
  for (int e = 0; e < n_evals; ++e) {
    const float table[3] = {0.0f, t_video[e], t_audio[e]};
    FS_TRY(stack_forward_impl(dims, n_layers, layers, layer_compress, io, tok, table, 3, video_lat, text_emb,
                              audio_lat, vv, va, workspace, ws_bytes, st));
    const float tc[4] = {0.0f, t_video[e], t_audio[e], 0.0f};
    const float tn[4] = {0.0f, t_video[e + 1], t_audio[e + 1], 0.0f};
    if (tok->n_vrows > 0) FS_TRY(launch_euler(video_lat, vv, vid_mod, vid_mask, tok->n_vrows, io->c_video, tc, tn, st));
    if (tok->n_audio > 0) FS_TRY(launch_euler(audio_lat, va, aud_mod, aud_mask, tok->n_audio, io->c_audio, tc, tn, st));
  }
  return FSDIT_OK;
}

}  // extern "C"
