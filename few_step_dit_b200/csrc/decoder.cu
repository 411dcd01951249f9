// The lightweight video decoder's forward pass ([tokendh] section
// "解码器瓶颈：被忽视的那一半时间": 26 layers, hidden 2048, 4x feed-forward;
// [ananclaw explainer] section 3.4: a lightweight VAE decoder), as a
// transformer over the latent cells of a clip:
//   latent projection (embed kernel without tags) -> n_layers backbone blocks
//   at full resolution (the same block body, GEMMs and attention as the
//   denoiser) -> final RMSNorm -> pixel head on the tensor cores whose
//   epilogue writes every value straight to its frame, channel and pixel
//   (EPI_UNPATCH: no [cells, patch] intermediate and no permute pass), as
//   fp32 or, with the GPU-side colour conversion of [PaperDaily] section 二,
//   as 8-bit codes.
// Included by libfsdit.cu after api.cu, whose block helpers it reuses.

namespace fsdit {

// (t, h, w) of every cell of a T x H x W grid, row-major: the RoPE positions.
__global__ void __launch_bounds__(256) grid_pos_kernel(int T, int H, int W, int32_t* __restrict__ pos) {
  const int n = T * H * W, hw = H * W;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    pos[3 * i] = i / hw;
    pos[3 * i + 1] = (i / W) % H;
    pos[3 * i + 2] = i % W;
  }
}

static fsdit_status launch_grid_pos(int T, int H, int W, int32_t* pos, cudaStream_t st) {
  const int n = T * H * W;
  ProfScope ps(PC_GRID_POS, 1, 0.0, 12.0 * n, st);
  int blocks = (n + 255) / 256;
  if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
  grid_pos_kernel<<<blocks, 256, 0, st>>>(T, H, W, pos);
  return cuda_check(cudaGetLastError(), "grid_pos_kernel");
}

static fsdit_status check_decoder_io(const fsdit_decoder_io* io) {
  FS_TRY(need(io, "io"));
  FS_TRY(need(io->w_in, "io.w_in"));
  FS_TRY(need(io->b_in, "io.b_in"));
  FS_TRY(need(io->g_out, "io.g_out"));
  FS_TRY(need(io->w_out, "io.w_out"));
  FS_TRY(need(io->b_out, "io.b_out"));
  if (io->c_lat < 1 || io->c_lat > 64 || io->c_pix < 1 || io->c_pix > 64 || io->patch_t < 1 ||
      io->patch_t > 64 || io->patch_s < 4 || io->patch_s > 64 || io->patch_s % 4 != 0) {
    set_error("decoder io: need c_lat in 1..64, c_pix in 1..64, patch_t in 1..64, patch_s in 4..64 and %% 4 == 0 "
              "(got %d, %d, %d, %d)", io->c_lat, io->c_pix, io->patch_t, io->patch_s);
    return FSDIT_E_SHAPE;
  }
  return FSDIT_OK;
}

static fsdit_status check_decoder_grid(int T, int H, int W) {
  if (T <= 0 || H <= 0 || W <= 0 || (long long)T * H * W > (1 << 24)) {
    set_error("decoder: grid %dx%dx%d must be non-empty with at most 2^24 cells", T, H, W);
    return FSDIT_E_SHAPE;
  }
  return FSDIT_OK;
}

static int pixel_cols(const fsdit_decoder_io* io) { return io->c_pix * io->patch_t * io->patch_s * io->patch_s; }

// x [N, hidden] fp32, pos [N, 3] int32, then the block buffers of N full rows.
static size_t decoder_carve(Carve& c, const fsdit_dims* d, int N, float** x, int32_t** pos, BlockWs* ws) {
  *x = (float*)c.take((size_t)N * d->hidden * 4);
  *pos = (int32_t*)c.take((size_t)N * 3 * 4);
  *ws = carve_block(c, d, N, N, false);
  carve_norm(c, d, N, *ws);
  return c.off;
}

}  // namespace fsdit

using namespace fsdit;

extern "C" {

int fsdit_decoder_frames(int T, int patch_t) { return T > 0 && patch_t > 0 ? 1 + patch_t * (T - 1) : 0; }

size_t fsdit_decoder_workspace_size(const fsdit_dims* dims, const fsdit_decoder_io* io, int T, int H, int W) {
  if (check_dims(dims) != FSDIT_OK || check_decoder_io(io) != FSDIT_OK || check_decoder_grid(T, H, W) != FSDIT_OK)
    return 0;
  Carve c{nullptr, 0};
  float* x;
  int32_t* pos;
  BlockWs ws;
  return decoder_carve(c, dims, T * H * W, &x, &pos, &ws);
}

fsdit_status fsdit_decoder_forward(const fsdit_dims* dims, int n_layers, const fsdit_block_weights* layers,
                                   const fsdit_decoder_io* io, int T, int H, int W, const float* latents,
                                   void* pixels, int pixel_format, void* workspace, size_t ws_bytes,
                                   fsdit_stream_t stream) {
  FS_TRY(check_dims(dims));
  FS_TRY(check_decoder_io(io));
  FS_TRY(check_decoder_grid(T, H, W));
  if (n_layers < 0 || (n_layers > 0 && layers == nullptr)) {
    set_error("decoder: n_layers >= 0 and a host array of n_layers block weights are required");
    return FSDIT_E_NULL;
  }
  for (int l = 0; l < n_layers; ++l) FS_TRY(check_block_weights(dims, &layers[l]));
  if (pixel_format != FSDIT_PIXELS_F32 && pixel_format != FSDIT_PIXELS_RGB8) {
    set_error("decoder: pixel_format %d is neither FSDIT_PIXELS_F32 nor FSDIT_PIXELS_RGB8", pixel_format);
    return FSDIT_E_DTYPE;
  }
  FS_TRY(need(latents, "latents"));
  FS_TRY(need(pixels, "pixels"));
  FS_TRY(need(workspace, "workspace"));
  if (!aligned16(pixels) || !aligned16(workspace)) {
    set_error("decoder: pixels and workspace must be 16-byte aligned");
    return FSDIT_E_ALIGN;
  }
  const int N = T * H * W, Hd = dims->hidden;
  Carve c{(uint8_t*)workspace, 0};
  float* x;
  int32_t* pos;
  BlockWs ws;
  decoder_carve(c, dims, N, &x, &pos, &ws);
  if (c.off > ws_bytes) {
    set_error("workspace: need %zu bytes, got %zu", c.off, ws_bytes);
    return FSDIT_E_WORKSPACE;
  }
  cudaStream_t st = (cudaStream_t)stream;
  FS_TRY(launch_grid_pos(T, H, W, pos, st));
  FS_TRY(launch_embed(dims->dtype, x, Hd, 0, N, 1, latents, io->c_lat, io->w_in, io->b_in, nullptr, nullptr,
                      nullptr, nullptr, nullptr, 0, 0, 0, st));
  FS_TRY(rope_table(dims, pos, N, ws.rope, st));
  bool ready = false;  // each layer's FFN-down epilogue prepares the next layer's attention norm
  for (int l = 0; l < n_layers; ++l)
    FS_TRY(block_body(dims, &layers[l], x, x, pos, ws.rope, N, ws, st, ready,
                      l + 1 < n_layers ? layers[l + 1].g_attn : nullptr, &ready));
  FS_TRY(launch_rmsnorm_cast(x, io->g_out, ws.xn, N, Hd, dims->rms_eps, dims->dtype, st));
  const int n_out = pixel_cols(io);
  EpiParams ep = make_ep(dims, EPI_UNPATCH, io->b_out, pixels, n_out, nullptr, nullptr);
  ep.up_h = H;
  ep.up_w = W;
  ep.up_c = io->c_pix;
  ep.up_pt = io->patch_t;
  ep.up_ps = io->patch_s;
  ep.up_rgb8 = pixel_format == FSDIT_PIXELS_RGB8 ? 1 : 0;
  return launch_linear(dims, ws.xn, io->w_out, ep, N, n_out, Hd, st, PC_PIXEL_HEAD);
}

}  // extern "C"
