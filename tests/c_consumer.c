/*
 * A plain C99 host program that uses libfsdit.so through include/fsdit.h and
 * the CUDA runtime's C API only: no Python, no torch.  The tests compile it
 * with gcc and run it.
 *
 *   c_consumer host
 *     prints the results of the entry points that run on the host alone (no
 *     device is touched), one line per result, for the test to compare with
 *     the oracle.
 *
 *   c_consumer block DIR hidden heads ffn T H W n_text n_audio compress
 *     reads the inputs of one fp32 DiT block from DIR (raw little-endian
 *     files: the ten weight arrays of fsdit_block_weights under their field
 *     names, x.bin [n][hidden] f32, pos.bin [n][3] i32, modality.bin,
 *     time_id.bin and out_mask.bin [n] u8), builds the keep map of the T x H x W
 *     grid on device 0 when `compress` is 1, runs dit_block_forward there and
 *     writes DIR/out.bin [n][hidden] f32.
 *
 * Exit status: 0 on success; 1 on a failed library or CUDA call (the message
 * goes to stderr).
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "fsdit.h"

static int fail(const char* what, const char* msg) {
  fprintf(stderr, "c_consumer: %s: %s\n", what, msg ? msg : "");
  return 1;
}

#define CUDA_OK(call)                                                   \
  do {                                                                  \
    cudaError_t e_ = (call);                                            \
    if (e_ != cudaSuccess) return fail(#call, cudaGetErrorString(e_)); \
  } while (0)

#define FSDIT_OK_OR_FAIL(call)                                  \
  do {                                                          \
    fsdit_status s_ = (call);                                   \
    if (s_ != FSDIT_OK) return fail(#call, fsdit_last_error()); \
  } while (0)

/* ------------------------------------------------------------ host mode */

static void print_status(const char* name, fsdit_status s) {
  const char* msg = fsdit_last_error();
  printf("status %s %d %d\n", name, (int)s, msg != NULL && msg[0] != '\0');
}

static fsdit_dims full_width_dims(void) {
  fsdit_dims d;
  memset(&d, 0, sizeof d);
  d.hidden = 5376;
  d.heads = 56;
  d.head_dim = 128;
  d.ffn = 14336;
  d.rope_split[0] = 32;
  d.rope_split[1] = 48;
  d.rope_split[2] = 48;
  d.rms_eps = 1e-6f;
  d.rope_theta = 10000.0f;
  d.dtype = FSDIT_BF16;
  d.proj_fp8 = 0;
  return d;
}

static int host_mode(void) {
  static const int grids[][3] = {{6, 34, 60}, {6, 17, 30}, {12, 34, 60}, {2, 9, 10}, {1, 1, 1}, {3, 5, 7}};
  static const int frames_t[] = {1, 2, 6, 7};
  fsdit_history_entry plan[FSDIT_HISTORY_MAX_ENTRIES];
  fsdit_dims d = full_width_dims();
  size_t i;
  int nb;

  printf("version %s\n", fsdit_version());
  for (i = 0; i < sizeof grids / sizeof grids[0]; ++i)
    printf("keep %d %d %d %d\n", grids[i][0], grids[i][1], grids[i][2],
           fsdit_keep_count(grids[i][0], grids[i][1], grids[i][2]));
  for (i = 0; i < sizeof frames_t / sizeof frames_t[0]; ++i)
    printf("frames %d 4 %d\n", frames_t[i], fsdit_decoder_frames(frames_t[i], 4));
  for (nb = 0; nb < 32; ++nb) {
    int n = fsdit_history_plan(nb, plan, FSDIT_HISTORY_MAX_ENTRIES), k;
    printf("plan %d %d", nb, n);
    for (k = 0; k < n; ++k) printf(" %d %d", plan[k].frame, plan[k].stride);
    printf(" rows %d\n", n >= 0 ? fsdit_history_rows(plan, n, 34, 60) : -1);
  }
  printf("plan_small %d\n", fsdit_history_plan(30, plan, 4));
  printf("history_bytes %zu\n", fsdit_history_bytes(12, 34, 60, 24));
  printf("block_ws %zu %zu\n", fsdit_block_workspace_size(&d, 3668, 0), fsdit_block_workspace_size(&d, 12560, 3348));
  d.head_dim = 64;
  printf("block_ws_bad %zu\n", fsdit_block_workspace_size(&d, 100, 0));

  /* argument checks that fail on the host before any launch */
  print_status("keep_map_null", fsdit_build_keep_map(6, 34, 60, NULL, NULL, NULL));
  {
    fsdit_history_store s;
    memset(&s, 0, sizeof s);
    print_status("history_init_null", fsdit_history_init(&s, NULL, 12, 34, 60, 24));
    print_status("history_init_small", fsdit_history_init(&s, (float*)(size_t)0x100000, 11, 34, 60, 24));
  }
  {
    const float tc[4] = {0.f, 0.2f, 0.5f, 0.f};
    print_status("euler_null", flow_euler_step((float*)(size_t)0x100000, (const float*)(size_t)0x100000, NULL,
                                               NULL, 4, 24, tc, tc, NULL));
  }
  return 0;
}

/* ----------------------------------------------------------- block mode */

static void* read_file(const char* dir, const char* name, size_t bytes) {
  char path[4096];
  FILE* f;
  void* buf;
  snprintf(path, sizeof path, "%s/%s", dir, name);
  f = fopen(path, "rb");
  if (f == NULL) return NULL;
  buf = malloc(bytes > 0 ? bytes : 1);
  if (buf != NULL && fread(buf, 1, bytes, f) != bytes) {
    free(buf);
    buf = NULL;
  }
  fclose(f);
  return buf;
}

/* Copies DIR/name (bytes) to a new device buffer. */
static int upload(const char* dir, const char* name, size_t bytes, void** dev) {
  void* host = read_file(dir, name, bytes);
  if (host == NULL) return fail("read", name);
  if (cudaMalloc(dev, bytes) != cudaSuccess || cudaMemcpy(*dev, host, bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
    free(host);
    return fail("upload", name);
  }
  free(host);
  return 0;
}

static int block_mode(int argc, char** argv) {
  const char* dir;
  int hidden, heads, ffn, T, H, W, n_text, n_audio, compress, A, n_grid, n;
  fsdit_dims d;
  fsdit_block_weights w;
  fsdit_tokens tok;
  void *ptr[10], *x = NULL, *y = NULL, *pos = NULL, *mod = NULL, *tid = NULL, *msk = NULL, *ws = NULL;
  int32_t *keep = NULL, *near = NULL;
  size_t ws_bytes, out_bytes;
  float* out;
  FILE* f;
  char path[4096];
  int i;
  static const char* names[10] = {"w_qkv.bin", "b_qkv.bin", "w_o.bin", "b_o.bin", "w_1.bin",
                                  "b_1.bin",   "w_2.bin",   "b_2.bin", "g_attn.bin", "g_ffn.bin"};
  size_t sizes[10];

  if (argc != 12) return fail("usage", "block DIR hidden heads ffn T H W n_text n_audio compress");
  dir = argv[2];
  hidden = atoi(argv[3]);
  heads = atoi(argv[4]);
  ffn = atoi(argv[5]);
  T = atoi(argv[6]);
  H = atoi(argv[7]);
  W = atoi(argv[8]);
  n_text = atoi(argv[9]);
  n_audio = atoi(argv[10]);
  compress = atoi(argv[11]);
  A = heads * 128;
  n_grid = T * H * W;
  n = n_grid + n_text + n_audio;

  d = full_width_dims();
  d.hidden = hidden;
  d.heads = heads;
  d.ffn = ffn;
  d.dtype = FSDIT_F32;

  sizes[0] = (size_t)3 * A * hidden;
  sizes[1] = (size_t)3 * A;
  sizes[2] = (size_t)hidden * A;
  sizes[3] = (size_t)hidden;
  sizes[4] = (size_t)ffn * hidden;
  sizes[5] = (size_t)ffn;
  sizes[6] = (size_t)hidden * ffn;
  sizes[7] = (size_t)hidden;
  sizes[8] = (size_t)hidden;
  sizes[9] = (size_t)hidden;
  for (i = 0; i < 10; ++i)
    if (upload(dir, names[i], sizes[i] * sizeof(float), &ptr[i])) return 1;
  memset(&w, 0, sizeof w);
  w.w_qkv = ptr[0];
  w.b_qkv = ptr[1];
  w.w_o = ptr[2];
  w.b_o = ptr[3];
  w.w_1 = ptr[4];
  w.b_1 = ptr[5];
  w.w_2 = ptr[6];
  w.b_2 = ptr[7];
  w.g_attn = ptr[8];
  w.g_ffn = ptr[9];

  out_bytes = (size_t)n * hidden * sizeof(float);
  if (upload(dir, "x.bin", out_bytes, &x) || upload(dir, "pos.bin", (size_t)n * 3 * sizeof(int32_t), &pos) ||
      upload(dir, "modality.bin", (size_t)n, &mod) || upload(dir, "time_id.bin", (size_t)n, &tid) ||
      upload(dir, "out_mask.bin", (size_t)n, &msk))
    return 1;
  CUDA_OK(cudaMalloc(&y, out_bytes));

  memset(&tok, 0, sizeof tok);
  tok.n_tokens = n;
  tok.n_vrows = n_grid;
  tok.n_text = n_text;
  tok.n_audio = n_audio;
  tok.grid_t = T;
  tok.grid_h = H;
  tok.grid_w = W;
  tok.pos_thw = (const int32_t*)pos;
  tok.modality = (const uint8_t*)mod;
  tok.time_id = (const uint8_t*)tid;
  tok.out_mask = (const uint8_t*)msk;
  if (compress) {
    tok.n_keep = fsdit_keep_count(T, H, W);
    CUDA_OK(cudaMalloc((void**)&keep, (size_t)tok.n_keep * sizeof(int32_t)));
    CUDA_OK(cudaMalloc((void**)&near, (size_t)n_grid * sizeof(int32_t)));
    FSDIT_OK_OR_FAIL(fsdit_build_keep_map(T, H, W, keep, near, NULL));
    tok.keep_idx = keep;
    tok.near_idx = near;
  }

  ws_bytes = fsdit_block_workspace_size(&d, n, tok.n_keep);
  if (ws_bytes == 0) return fail("fsdit_block_workspace_size", fsdit_last_error());
  CUDA_OK(cudaMalloc(&ws, ws_bytes));
  FSDIT_OK_OR_FAIL(dit_block_forward(&d, &w, &tok, (const float*)x, (float*)y, ws, ws_bytes, NULL));
  CUDA_OK(cudaDeviceSynchronize());
  FSDIT_OK_OR_FAIL(fsdit_device_error(NULL));

  out = (float*)malloc(out_bytes);
  if (out == NULL) return fail("malloc", "out");
  CUDA_OK(cudaMemcpy(out, y, out_bytes, cudaMemcpyDeviceToHost));
  snprintf(path, sizeof path, "%s/out.bin", dir);
  f = fopen(path, "wb");
  if (f == NULL || fwrite(out, 1, out_bytes, f) != out_bytes) return fail("write", path);
  fclose(f);
  free(out);

  for (i = 0; i < 10; ++i) cudaFree(ptr[i]);
  cudaFree(x);
  cudaFree(y);
  cudaFree(pos);
  cudaFree(mod);
  cudaFree(tid);
  cudaFree(msk);
  cudaFree(keep);
  cudaFree(near);
  cudaFree(ws);
  printf("block ok %d rows\n", n);
  return 0;
}

int main(int argc, char** argv) {
  if (argc >= 2 && strcmp(argv[1], "host") == 0) return host_mode();
  if (argc >= 2 && strcmp(argv[1], "block") == 0) return block_mode(argc, argv);
  return fail("usage", "c_consumer host | c_consumer block DIR hidden heads ffn T H W n_text n_audio compress");
}
