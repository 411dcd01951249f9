// Long-video chunking: the bounded multi-stride history ([tokendh] section
// "长视频生成：怎么记住十分钟前发生的事"; [PaperDaily] section 三).
//
// The frame store is caller memory of `capacity` latent frames [H][W][C]
// fp32; frame 0 lives in slot 0 and frame i >= 1 in slot 1 + (i-1) % (cap-1).
// A chunk's history plan names frame 0 (full resolution), at most eight
// frames at spatial stride 4 and the two newest frames at stride 2, all
// before the chunk's boundary frame.  history_gather_kernel copies the planned
// positions into the rows that follow the chunk's target grid and writes their
// (t, h, w) RoPE coordinates next to them.  Index work only: the copy is exact.

namespace fsdit {
namespace hist {

struct GatherPlan {
  int n;                                    // entries
  int slot[FSDIT_HISTORY_MAX_ENTRIES];
  int frame[FSDIT_HISTORY_MAX_ENTRIES];
  int stride[FSDIT_HISTORY_MAX_ENTRIES];
  int cols[FSDIT_HISTORY_MAX_ENTRIES];      // positions per sampled row: ceil(W / stride)
  int row0[FSDIT_HISTORY_MAX_ENTRIES + 1];  // first output row of each entry; row0[n] = total
};

// One thread per (output row, channel); the entry of a row is found by a
// linear scan of at most 11 offsets.
__global__ void history_gather_kernel(const float* __restrict__ frames, int H, int W, int C, GatherPlan plan,
                                      float* __restrict__ lat, int ld_lat, int32_t* __restrict__ pos) {
  const long long total = (long long)plan.row0[plan.n] * C;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / C), c = (int)(i - (long long)r * C);
    int e = 0;
    while (e + 1 < plan.n && r >= plan.row0[e + 1]) ++e;
    const int local = r - plan.row0[e];
    const int s = plan.stride[e];
    const int h = (local / plan.cols[e]) * s, w = (local % plan.cols[e]) * s;
    const size_t src = (((size_t)plan.slot[e] * H + h) * W + w) * C + c;
    lat[(size_t)r * ld_lat + c] = frames[src];
    if (c == 0) {
      pos[3 * (size_t)r] = plan.frame[e];
      pos[3 * (size_t)r + 1] = h;
      pos[3 * (size_t)r + 2] = w;
    }
  }
}

inline int slot_of(const fsdit_history_store* s, int frame) {
  return frame == 0 ? 0 : 1 + (frame - 1) % (s->capacity - 1);
}

// A frame is resident while no later frame has taken its slot.
inline bool resident(const fsdit_history_store* s, int frame) {
  if (frame < 0 || frame >= s->n_frames) return false;
  return frame == 0 || frame + (s->capacity - 1) > s->n_frames - 1;
}

inline size_t frame_elems(const fsdit_history_store* s) { return (size_t)s->H * s->W * s->C; }

inline int per_axis(int n, int stride) { return (n + stride - 1) / stride; }

fsdit_status check_store(const fsdit_history_store* s) {
  if (s == nullptr || s->frames == nullptr) {
    set_error("history: store or its frame memory is NULL");
    return FSDIT_E_NULL;
  }
  if (s->capacity < FSDIT_HISTORY_MIN_SLOTS || s->H <= 0 || s->W <= 0 || s->C <= 0 || s->n_frames < 0) {
    set_error("history: bad store (capacity %d, %d x %d x %d, %d frames)", s->capacity, s->H, s->W, s->C,
              s->n_frames);
    return FSDIT_E_SHAPE;
  }
  return FSDIT_OK;
}

}  // namespace hist
}  // namespace fsdit

using namespace fsdit;

extern "C" {

FSDIT_API size_t fsdit_history_bytes(int capacity, int H, int W, int C) {
  if (capacity <= 0 || H <= 0 || W <= 0 || C <= 0) return 0;
  return (size_t)capacity * H * W * C * sizeof(float);
}

FSDIT_API fsdit_status fsdit_history_init(fsdit_history_store* s, float* frames, int capacity, int H, int W,
                                          int C) {
  if (s == nullptr || frames == nullptr) {
    set_error("history_init: NULL store or frame memory");
    return FSDIT_E_NULL;
  }
  if (((uintptr_t)frames & 15u) != 0) {
    set_error("history_init: frame memory is not 16-byte aligned");
    return FSDIT_E_ALIGN;
  }
  s->frames = frames;
  s->capacity = capacity;
  s->H = H;
  s->W = W;
  s->C = C;
  s->n_frames = 0;
  return hist::check_store(s);
}

FSDIT_API fsdit_status fsdit_history_push(fsdit_history_store* s, const float* frames, int n,
                                          fsdit_stream_t stream) {
  FS_TRY(hist::check_store(s));
  if (n < 0) {
    set_error("history_push: n < 0");
    return FSDIT_E_SHAPE;
  }
  if (n > 0 && frames == nullptr) {
    set_error("history_push: frames is NULL");
    return FSDIT_E_NULL;
  }
  const size_t fe = hist::frame_elems(s);
  for (int j = 0; j < n; ++j) {
    const int slot = hist::slot_of(s, s->n_frames + j);
    FS_TRY(cuda_check(cudaMemcpyAsync(s->frames + (size_t)slot * fe, frames + (size_t)j * fe, fe * sizeof(float),
                                      cudaMemcpyDeviceToDevice, (cudaStream_t)stream),
                      "history_push: cudaMemcpyAsync"));
  }
  s->n_frames += n;
  return FSDIT_OK;
}

FSDIT_API int fsdit_history_plan(int n_before, fsdit_history_entry* out, int max_entries) {
  if (n_before < 0 || out == nullptr) return -1;
  if (n_before == 0) return 0;
  // frame 0 at full resolution; of frames 1 .. n_before-1 the two newest at
  // stride 2 and up to eight before them at stride 4; the rest are dropped
  const int newest = n_before - 1;
  const int n_recent = newest >= 2 ? 2 : newest;  // frames 1.. available
  const int recent0 = newest - n_recent + 1;
  const int older_hi = recent0 - 1;               // newest "older" frame
  const int n_older = older_hi >= 1 ? (older_hi < 8 ? older_hi : 8) : 0;
  const int need = 1 + n_older + n_recent;
  if (need > max_entries) return -1;
  int k = 0;
  out[k++] = {0, 1};
  for (int f = older_hi - n_older + 1; f <= older_hi; ++f) out[k++] = {f, 4};
  for (int f = recent0; f <= newest; ++f) out[k++] = {f, 2};
  return k;
}

FSDIT_API int fsdit_history_rows(const fsdit_history_entry* plan, int n_plan, int H, int W) {
  if (plan == nullptr || n_plan < 0 || H <= 0 || W <= 0) return -1;
  int rows = 0;
  for (int e = 0; e < n_plan; ++e) {
    const int s = plan[e].stride;
    if (s != 1 && s != 2 && s != 4) return -1;
    rows += hist::per_axis(H, s) * hist::per_axis(W, s);
  }
  return rows;
}

FSDIT_API fsdit_status fsdit_history_gather(const fsdit_history_store* s, const fsdit_history_entry* plan,
                                            int n_plan, float* lat, int ld_lat, int32_t* pos,
                                            fsdit_stream_t stream) {
  FS_TRY(hist::check_store(s));
  if (n_plan < 0 || n_plan > FSDIT_HISTORY_MAX_ENTRIES) {
    set_error("history_gather: n_plan %d outside 0..%d", n_plan, FSDIT_HISTORY_MAX_ENTRIES);
    return FSDIT_E_SHAPE;
  }
  if (n_plan == 0) return FSDIT_OK;
  FS_TRY(need(plan, "plan"));
  FS_TRY(need(lat, "lat"));
  FS_TRY(need(pos, "pos"));
  if (ld_lat < s->C) {
    set_error("history_gather: ld_lat %d < C %d", ld_lat, s->C);
    return FSDIT_E_SHAPE;
  }
  hist::GatherPlan gp;
  gp.n = n_plan;
  gp.row0[0] = 0;
  for (int e = 0; e < n_plan; ++e) {
    const int f = plan[e].frame, st = plan[e].stride;
    if (st != 1 && st != 2 && st != 4) {
      set_error("history_gather: stride %d is not 1, 2 or 4", st);
      return FSDIT_E_SHAPE;
    }
    if (!hist::resident(s, f)) {
      set_error("history_gather: frame %d is not resident (%d frames pushed, %d slots)", f, s->n_frames,
                s->capacity);
      return FSDIT_E_SHAPE;
    }
    gp.slot[e] = hist::slot_of(s, f);
    gp.frame[e] = f;
    gp.stride[e] = st;
    gp.cols[e] = hist::per_axis(s->W, st);
    gp.row0[e + 1] = gp.row0[e] + hist::per_axis(s->H, st) * gp.cols[e];
  }
  const int rows = gp.row0[n_plan];
  ProfScope ps(PC_HISTORY, 1, 0.0, (double)rows * s->C * 8.0 + rows * 12.0, (cudaStream_t)stream);
  const long long total = (long long)rows * s->C;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > (long long)num_sms() * 8) blocks = (long long)num_sms() * 8;
  hist::history_gather_kernel<<<(int)blocks, threads, 0, (cudaStream_t)stream>>>(s->frames, s->H, s->W, s->C, gp,
                                                                                  lat, ld_lat, pos);
  return cuda_check(cudaGetLastError(), "history_gather_kernel");
}

FSDIT_API fsdit_status fsdit_history_copy_frame(const fsdit_history_store* s, int frame, float* dst,
                                                fsdit_stream_t stream) {
  FS_TRY(hist::check_store(s));
  FS_TRY(need(dst, "dst"));
  if (!hist::resident(s, frame)) {
    set_error("history_copy_frame: frame %d is not resident (%d frames pushed)", frame, s->n_frames);
    return FSDIT_E_SHAPE;
  }
  const size_t fe = hist::frame_elems(s);
  return cuda_check(cudaMemcpyAsync(dst, s->frames + (size_t)hist::slot_of(s, frame) * fe, fe * sizeof(float),
                                    cudaMemcpyDeviceToDevice, (cudaStream_t)stream),
                    "history_copy_frame: cudaMemcpyAsync");
}

FSDIT_API fsdit_status fsdit_chunk_tags(int T, int H, int W, int base, int has_boundary, int n_hist, int n_text,
                                        int n_audio, uint8_t* modality, uint8_t* time_id, uint8_t* out_mask,
                                        int32_t* pos) {
  if (modality == nullptr || time_id == nullptr || out_mask == nullptr || pos == nullptr) {
    set_error("chunk_tags: NULL output array");
    return FSDIT_E_NULL;
  }
  if (T <= 0 || H <= 0 || W <= 0 || n_hist < 0 || n_text < 0 || n_audio < 0 || base < 0 ||
      (has_boundary && T < 2)) {
    set_error("chunk_tags: bad sizes");
    return FSDIT_E_SHAPE;
  }
  const int hw = H * W, n_grid = T * hw;
  int r = 0;
  for (int t = 0; t < T; ++t)
    for (int h = 0; h < H; ++h)
      for (int w = 0; w < W; ++w, ++r) {
        const bool boundary = has_boundary && t == 0;
        modality[r] = FSDIT_MOD_VIDEO;
        time_id[r] = boundary ? 0 : 1;
        out_mask[r] = boundary ? 0 : 1;
        pos[3 * r] = base + t;
        pos[3 * r + 1] = h;
        pos[3 * r + 2] = w;
      }
  for (int i = 0; i < n_hist; ++i, ++r) {
    modality[r] = FSDIT_MOD_VIDEO;
    time_id[r] = 0;
    out_mask[r] = 0;
  }
  for (int i = 0; i < n_text; ++i, ++r) {
    modality[r] = FSDIT_MOD_TEXT;
    time_id[r] = 0;
    out_mask[r] = 0;
    pos[3 * r] = pos[3 * r + 1] = pos[3 * r + 2] = 0;
  }
  for (int j = 0; j < n_audio; ++j, ++r) {
    modality[r] = FSDIT_MOD_AUDIO;
    time_id[r] = 2;
    out_mask[r] = 1;
    pos[3 * r] = (int)(((long long)j * T) / n_audio) + base;
    pos[3 * r + 1] = pos[3 * r + 2] = 0;
  }
  (void)n_grid;
  return FSDIT_OK;
}

}  // extern "C"
