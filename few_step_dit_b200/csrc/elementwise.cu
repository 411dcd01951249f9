// HBM-bound kernels of the hot path: keep-index map, gather, nearest-kept
// broadcast + residual, RMSNorm-cast, RoPE table, embedding, timestep MLP and
// the per-modality Euler step.  Rows move with 16-byte vector accesses.
#include "common.cuh"

namespace fsdit {

// ---------------------------------------------------------------- keep map

// kept count of one axis of length n: floor(n/2) + 1
__device__ __forceinline__ int axis_kept(int n) { return n / 2 + 1; }
// nearest kept index (ties -> lower): i itself if even or last, else i-1
__device__ __forceinline__ int axis_rho(int i, int n) { return ((i & 1) == 0 || i == n - 1) ? i : i - 1; }
// compact index of a kept index i
__device__ __forceinline__ int axis_kappa(int i) { return (i + 1) >> 1; }

__global__ void keep_map_kernel(int T, int H, int W, int32_t* __restrict__ keep_idx,
                                int32_t* __restrict__ near_idx) {
  const int total = T * H * W;
  const int kh = axis_kept(H), kw = axis_kept(W);
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < total; p += gridDim.x * blockDim.x) {
    const int t = p / (H * W);
    const int h = (p / W) % H;
    const int w = p % W;
    const int rh = axis_rho(h, H), rw = axis_rho(w, W);
    const int c = t * kh * kw + axis_kappa(rh) * kw + axis_kappa(rw);
    near_idx[p] = c;
    if (rh == h && rw == w) keep_idx[c] = p;
  }
}

// ---------------------------------------------------------------- gather

// One block per output row (grid-stride over rows); float4 copies.  A keep
// index outside [0, n_grid) is not followed: the row is left as it is and the
// device error word records DEVERR_KEEPMAP.
__global__ void gather_rows_kernel(const float* __restrict__ x, const int32_t* __restrict__ pos,
                                   float* __restrict__ xc, int32_t* __restrict__ posc,
                                   const int32_t* __restrict__ keep_idx, int n_keep, int n_grid,
                                   int n_out, int hidden) {
  const int h4 = hidden >> 2;
  for (int r = blockIdx.x; r < n_out; r += gridDim.x) {
    const int src = r < n_keep ? keep_idx[r] : n_grid + (r - n_keep);
    if (r < n_keep && (src < 0 || src >= n_grid)) {
      if (threadIdx.x == 0) raise_device_error(DEVERR_KEEPMAP);
      continue;
    }
    const float4* s = reinterpret_cast<const float4*>(x + (size_t)src * hidden);
    float4* d = reinterpret_cast<float4*>(xc + (size_t)r * hidden);
    for (int i = threadIdx.x; i < h4; i += blockDim.x) d[i] = __ldg(s + i);
    if (pos != nullptr && threadIdx.x < 3) posc[(size_t)r * 3 + threadIdx.x] = pos[(size_t)src * 3 + threadIdx.x];
  }
}

// ---------------------------------------------------------------- broadcast
// Block b < n_keep owns kept token b and every grid row whose nearest kept
// token it is.  Those rows are its own row src = keep_idx[b] and, because a
// dropped index takes the kept index just below it on each axis, the rows
// among src+1, src+W, src+W+1 (same frame) whose near_idx is b.  The block
// reads y_c[b] and x[src] once: out[src] = y_c[b], out[p] = x[p] + (y_c[b] -
// x[src]) for the others.  No two blocks touch the same row, so out may equal
// x.  Blocks b >= n_keep copy the non-grid rows (text, audio, control).
//
// The maps are checked as they are used, so a map that does not come from
// fsdit_build_keep_map is never followed out of bounds and never leaves a row
// silently unwritten: a block skips its token when keep_idx[b] is outside the
// grid or near_idx[keep_idx[b]] != b (a kept row must map to itself; this
// also makes keep_idx injective), and every thread checks grid rows p in a
// grid-stride loop: near_idx[p] must name a kept token c whose row lies in
// p's frame, at most one row above and one column left of p.  Together these
// are exactly the conditions under which every grid row is written once.  A
// failed check sets DEVERR_KEEPMAP in the device error word.
__device__ __forceinline__ bool near_entry_ok(const int32_t* keep_idx, const int32_t* near_idx, int p, int n_keep,
                                              int grid_h, int grid_w, int n_grid) {
  const int c = near_idx[p];
  if (c < 0 || c >= n_keep) return false;
  const int s = keep_idx[c];
  if (s < 0 || s >= n_grid) return false;
  const int hw = grid_h * grid_w;
  if (s / hw != p / hw) return false;
  const int dh = (p % hw) / grid_w - (s % hw) / grid_w, dw = p % grid_w - s % grid_w;
  return dh >= 0 && dh <= 1 && dw >= 0 && dw <= 1;
}

__global__ void broadcast_kernel(const float* x, const float* __restrict__ yc, float* out,
                                 const int32_t* __restrict__ keep_idx, const int32_t* __restrict__ near_idx,
                                 int n_keep, int grid_h, int grid_w, int n_grid, int n_rows, int hidden) {
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < n_grid; p += gridDim.x * blockDim.x)
    if (!near_entry_ok(keep_idx, near_idx, p, n_keep, grid_h, grid_w, n_grid)) raise_device_error(DEVERR_KEEPMAP);
  const int h4 = hidden >> 2;
  const int n_blocks = n_keep + (n_rows - n_grid);
  for (int b = blockIdx.x; b < n_blocks; b += gridDim.x) {
    const float4* y = reinterpret_cast<const float4*>(yc + (size_t)b * hidden);
    if (b >= n_keep) {
      float4* o = reinterpret_cast<float4*>(out + (size_t)(n_grid + b - n_keep) * hidden);
      for (int i = threadIdx.x; i < h4; i += blockDim.x) o[i] = __ldg(y + i);
      continue;
    }
    const int src = keep_idx[b];
    if (src < 0 || src >= n_grid || near_idx[src] != b) {
      if (threadIdx.x == 0) raise_device_error(DEVERR_KEEPMAP);
      continue;
    }
    const int w = src % grid_w, h = (src / grid_w) % grid_h;
    int child[3];
    int nc = 0;
    if (w + 1 < grid_w && near_idx[src + 1] == b) child[nc++] = src + 1;
    if (h + 1 < grid_h && near_idx[src + grid_w] == b) child[nc++] = src + grid_w;
    if (w + 1 < grid_w && h + 1 < grid_h && near_idx[src + grid_w + 1] == b) child[nc++] = src + grid_w + 1;
    const float4* xk = reinterpret_cast<const float4*>(x + (size_t)src * hidden);
    float4* ok = reinterpret_cast<float4*>(out + (size_t)src * hidden);
    for (int i = threadIdx.x; i < h4; i += blockDim.x) {
      const float4 yv = __ldg(y + i), kv = xk[i];
      const float4 d = make_float4(yv.x - kv.x, yv.y - kv.y, yv.z - kv.z, yv.w - kv.w);
      for (int c = 0; c < nc; ++c) {
        const float4 a = reinterpret_cast<const float4*>(x + (size_t)child[c] * hidden)[i];
        reinterpret_cast<float4*>(out + (size_t)child[c] * hidden)[i] =
            make_float4(a.x + d.x, a.y + d.y, a.z + d.z, a.w + d.w);
      }
      ok[i] = yv;
    }
  }
}

// ---------------------------------------------------------------- RMSNorm-cast

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  const int nw = blockDim.x >> 5;
  for (int i = 0; i < nw; ++i) s += red[i];
  return s;
}

template <typename T>
__device__ __forceinline__ void store4(T* o, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store4<float>(float* o, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(o) = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void store4<bf16>(bf16* o, float a, float b, float c, float d) {
  __nv_bfloat162 h0 = __floats2bfloat162_rn(a, b), h1 = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&h0);
  u.y = *reinterpret_cast<uint32_t*>(&h1);
  *reinterpret_cast<uint2*>(o) = u;
}

template <typename T>
__device__ __forceinline__ float4 load_g4(const T* g);
template <>
__device__ __forceinline__ float4 load_g4<float>(const float* g) { return __ldg(reinterpret_cast<const float4*>(g)); }
template <>
__device__ __forceinline__ float4 load_g4<bf16>(const bf16* g) {
  uint2 u = __ldg(reinterpret_cast<const uint2*>(g));
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x), b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// One block (256 threads) per row; the row stays in registers between the
// sum-of-squares pass and the scaled store.  hidden <= 256*4*RMS_MAXV.
constexpr int RMS_MAXV = 8;
template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_cast_kernel(const float* __restrict__ x, const T* __restrict__ g,
                                                           T* __restrict__ xn, int rows, int hidden, float eps) {
  __shared__ float red[8];
  const int h4 = hidden >> 2;
  const int r = blockIdx.x;
  if (r >= rows) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)r * hidden);
  float4 v[RMS_MAXV];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < RMS_MAXV; ++k) {
    const int i = threadIdx.x + k * 256;
    if (i < h4) {
      v[k] = xr[i];
      ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
    }
  }
  const float rstd = rsqrtf(block_sum(ss, red) / (float)hidden + eps);
  T* o = xn + (size_t)r * hidden;
#pragma unroll
  for (int k = 0; k < RMS_MAXV; ++k) {
    const int i = threadIdx.x + k * 256;
    if (i < h4) {
      const float4 gg = load_g4<T>(g + 4 * i);
      store4<T>(o + 4 * i, v[k].x * rstd * gg.x, v[k].y * rstd * gg.y, v[k].z * rstd * gg.z, v[k].w * rstd * gg.w);
    }
  }
}

// ---------------------------------------------------------------- RoPE table
// cs[r][j] = (cos, sin) of the angle of pair j of a head for row r; the QKV
// epilogue reads it instead of evaluating sincos per element.  Positions are
// constant across layers and evaluations, so one table serves a whole pass.
__global__ void rope_table_kernel(const int32_t* __restrict__ pos, int rows, int head_dim, int s0, int s1,
                                  float log2_theta, float2* __restrict__ cs) {
  const int pairs = head_dim >> 1;
  const size_t total = (size_t)rows * pairs;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / pairs), j = (int)(i % pairs);
    float a = 1.0f, b = 0.0f;  // rotating (1, 0) yields (cos, sin)
    rope_pair(a, b, 2 * j, s0, s1, head_dim, pos + (size_t)r * 3, log2_theta);
    cs[i] = make_float2(a, b);
  }
}

// ---------------------------------------------------------------- embedding
// x[r] = src(r) + mod_emb[modality[r]] + temb[time_id[r]], where src(r) is the
// small-K projection lat[r'] W^T + b of a video/control or audio row, or the
// precomputed text projection row.  Without tags (modality == nullptr: the
// decoder's latent cells) x[r] = src(r).  A block owns EMB_RB rows of one segment
// and EMB_CB consecutive columns: each thread keeps its column's weight row
// in registers (each weight twice, as an f32x2 pair); the rows' latents are
// staged channel-major in shared memory, so one 16-byte read gives a channel
// of four rows and two packed FMAs advance four rows' sums (the same fma
// sequence per output as a scalar loop over k); modality and timestep
// embeddings of the block's columns are staged too; stores are coalesced.
constexpr int EMB_RB = 128, EMB_CB = 256, EMB_MAXT = 8;

typedef unsigned long long emb_f2;
__device__ __forceinline__ emb_f2 emb_pair(float a, float b) {
  emb_f2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void emb_split(emb_f2 v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ emb_f2 emb_fma2(emb_f2 a, emb_f2 b, emb_f2 c) {
  emb_f2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

template <typename TW, int KMAX>
__global__ void __launch_bounds__(256) embed_kernel(
    float* __restrict__ x, int hidden, int row0, int rows, int kind,  // kind: 0 text, 1 latent
    const float* __restrict__ lat, int K, const TW* __restrict__ w_in, const TW* __restrict__ b_in,
    const float* __restrict__ text_proj, const TW* __restrict__ mod_emb, const float* __restrict__ temb,
    const uint8_t* __restrict__ modality, const uint8_t* __restrict__ time_id, int n_times,
    int expect_a, int expect_b) {
  __shared__ __align__(16) float s_latT[KMAX][EMB_RB];  // channel-major: rows j..j+3 of channel k are one float4
  __shared__ float s_mod[4][EMB_CB];
  __shared__ float s_temb[EMB_MAXT][EMB_CB];
  __shared__ __align__(16) int s_mt[EMB_RB];  // modality | time slot << 8 of each row
  const int rb0 = blockIdx.x * EMB_RB;
  const int nr = min(EMB_RB, rows - rb0);
  const int c = blockIdx.y * EMB_CB + threadIdx.x;
  const bool col_ok = c < hidden;
  const bool tagged = modality != nullptr;
  if (tagged && threadIdx.x < EMB_RB) {
    int m = expect_a, t = 0;
    if (threadIdx.x < nr) {
      const int r = row0 + rb0 + threadIdx.x;
      m = modality[r];
      t = time_id[r];
      if ((m != expect_a && m != expect_b) || t >= n_times) {
        raise_device_error(DEVERR_TAGS);
        m = expect_a;
        t = 0;
      }
    }
    s_mt[threadIdx.x] = m | (t << 8);
  }
  if (kind == 1) {
    // the block's rows are nr * K contiguous floats, transposed into the
    // channel-major stage; channels past K and rows past nr are zero
    if (K % 4 == 0) {  // 16-byte loads (the rows start 16-byte aligned: rb0 * K * 4 = 512 * K)
      const float4* src = reinterpret_cast<const float4*>(lat + (size_t)rb0 * K);
      const int n4 = nr * K / 4;
      for (int i = threadIdx.x; i < n4; i += blockDim.x) {
        const float4 v = __ldg(src + i);
        const int e = 4 * i, rr = e / K, kk = e - rr * K;  // the 4 values share a row
        s_latT[kk][rr] = v.x;
        s_latT[kk + 1][rr] = v.y;
        s_latT[kk + 2][rr] = v.z;
        s_latT[kk + 3][rr] = v.w;
      }
      for (int i = threadIdx.x; i < EMB_RB * KMAX; i += blockDim.x) {
        const int rr = i % EMB_RB, kk = i / EMB_RB;
        if (rr >= nr || kk >= K) s_latT[kk][rr] = 0.f;
      }
    } else {
      for (int i = threadIdx.x; i < EMB_RB * KMAX; i += blockDim.x) {
        const int rr = i % EMB_RB, kk = i / EMB_RB;  // consecutive threads: consecutive rows (no bank conflict)
        s_latT[kk][rr] = (rr < nr && kk < K) ? lat[(size_t)(rb0 + rr) * K + kk] : 0.f;
      }
    }
  }
  if (tagged) {
#pragma unroll
    for (int m = 0; m < 4; ++m) s_mod[m][threadIdx.x] = col_ok ? ld_f32<TW>(mod_emb + (size_t)m * hidden + c) : 0.f;
    for (int t = 0; t < n_times; ++t) s_temb[t][threadIdx.x] = col_ok ? temb[(size_t)t * hidden + c] : 0.f;
  }
  __syncthreads();
  if (!col_ok) return;
  if (kind == 1) {
    emb_f2 wd[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      const float wv = k < K ? ld_f32<TW>(w_in + (size_t)c * K + k) : 0.f;
      wd[k] = emb_pair(wv, wv);
    }
    const float bias = ld_f32<TW>(b_in + c);
    // the added embedding of a row depends only on its (modality, time slot),
    // the same for nearly every row of a segment: keep the last pair's sum
    int last_mt = -1;
    float add = 0.f;
    float* xp = x + (size_t)(row0 + rb0) * hidden + c;
    for (int j = 0; j < nr; j += 4, xp += 4 * (size_t)hidden) {  // rows past nr are zero in s_latT, not stored
      emb_f2 a01 = emb_pair(bias, bias), a23 = emb_pair(bias, bias);
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        const float4 l4 = *reinterpret_cast<const float4*>(&s_latT[k][j]);
        a01 = emb_fma2(emb_pair(l4.x, l4.y), wd[k], a01);
        a23 = emb_fma2(emb_pair(l4.z, l4.w), wd[k], a23);
      }
      float v[4];
      emb_split(a01, v[0], v[1]);
      emb_split(a23, v[2], v[3]);
      int4 mt = make_int4(0, 0, 0, 0);
      if (tagged) mt = *reinterpret_cast<const int4*>(&s_mt[j]);
      const int mts[4] = {mt.x, mt.y, mt.z, mt.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (j + u >= nr) break;
        if (tagged && mts[u] != last_mt) {  // uniform across the block: the row's tags
          last_mt = mts[u];
          add = s_mod[last_mt & 0xFF][threadIdx.x] + s_temb[last_mt >> 8][threadIdx.x];
        }
        xp[(size_t)u * hidden] = v[u] + add;
      }
    }
  } else {
    for (int j = 0; j < nr; ++j) {
      float acc = text_proj[(size_t)(rb0 + j) * hidden + c];
      if (tagged) acc += s_mod[s_mt[j] & 0xFF][threadIdx.x] + s_temb[s_mt[j] >> 8][threadIdx.x];
      x[(size_t)(row0 + rb0 + j) * hidden + c] = acc;
    }
  }
}

// ---------------------------------------------------------------- timestep MLP
// Stage 1: h1[t, c] = silu(sum_k feat_t[k] W1[c,k] + b1[c]) with the
// sinusoidal features of 1000*t computed in shared memory.
struct Times8 { float t[8]; };
template <typename TW>
__global__ void time_mlp1_kernel(Times8 times, int n_times, int t_freq, const TW* __restrict__ w1,
                                 const TW* __restrict__ b1, float* __restrict__ h1, int hidden) {
  extern __shared__ float s_feat[];  // [n_times][t_freq]
  const int half = t_freq / 2;
  for (int i = threadIdx.x; i < n_times * half; i += blockDim.x) {
    const int t = i / half, j = i % half;
    const float freq = expf(-logf(10000.0f) * (float)j / (float)half);
    const float arg = 1000.0f * times.t[t] * freq;
    float s, c;
    sincosf(arg, &s, &c);
    s_feat[t * t_freq + j] = c;
    s_feat[t * t_freq + half + j] = s;
  }
  __syncthreads();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int c = warp; c < hidden; c += nwarps) {
    for (int t = 0; t < n_times; ++t) {
      float acc = 0.f;
      for (int k = lane; k < t_freq; k += 32) acc = fmaf(s_feat[t * t_freq + k], ld_f32<TW>(w1 + (size_t)c * t_freq + k), acc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        const float z = acc + ld_f32<TW>(b1 + c);
        h1[(size_t)t * hidden + c] = z / (1.0f + expf(-z));
      }
    }
  }
}

// Stage 2: temb[t, c] = sum_k h1[t,k] W2[c,k] + b2[c]; one warp per output
// column, 8 weights (16 bytes of bf16) per lane per step, W2 read once.
constexpr int TMLP_MAXT = 8;
template <typename TW>
__device__ __forceinline__ void load8(const TW* p, float* w);
template <>
__device__ __forceinline__ void load8<bf16>(const bf16* p, float* w) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t a[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a[i]));
    w[2 * i] = f.x;
    w[2 * i + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float* w) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}

template <typename TW>
__global__ void time_mlp2_kernel(const float* __restrict__ h1, int n_times, const TW* __restrict__ w2,
                                 const TW* __restrict__ b2, float* __restrict__ temb, int hidden) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int c = warp; c < hidden; c += nwarps) {
    float acc[TMLP_MAXT];
#pragma unroll
    for (int t = 0; t < TMLP_MAXT; ++t) acc[t] = 0.f;
    for (int k = lane * 8; k < hidden; k += 256) {
      float w[8];
      load8<TW>(w2 + (size_t)c * hidden + k, w);
#pragma unroll
      for (int t = 0; t < TMLP_MAXT; ++t) {
        if (t < n_times) {
          const float4 ha = __ldg(reinterpret_cast<const float4*>(h1 + (size_t)t * hidden + k));
          const float4 hb = __ldg(reinterpret_cast<const float4*>(h1 + (size_t)t * hidden + k) + 1);
          acc[t] += ha.x * w[0] + ha.y * w[1] + ha.z * w[2] + ha.w * w[3] + hb.x * w[4] + hb.y * w[5] + hb.z * w[6] +
                    hb.w * w[7];
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TMLP_MAXT; ++t) {
      float a = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0 && t < n_times) temb[(size_t)t * hidden + c] = a + ld_f32<TW>(b2 + c);
    }
  }
}

// ---------------------------------------------------------------- Euler
struct Clock4 { float dt[4]; };
__global__ void euler_kernel(float* __restrict__ x, const float* __restrict__ v, const uint8_t* __restrict__ mod,
                             const uint8_t* __restrict__ mask, int n_rows, int width, Clock4 clk) {
  const size_t total = (size_t)n_rows * width;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / width);
    if (mask[r]) x[i] = fmaf(clk.dt[mod[r] & 3], v[i], x[i]);
  }
}

// ================================================================ host launchers

static int grid_for_rows(int rows, int per_sm) {
  const int g = num_sms() * per_sm;
  return rows < g ? (rows > 0 ? rows : 1) : g;
}

fsdit_status launch_keep_map(int T, int H, int W, int32_t* keep_idx, int32_t* near_idx, cudaStream_t st) {
  const int total = T * H * W;
  const int blocks = (total + 255) / 256;
  ProfScope ps(PC_KEEPMAP, 1, 0.0, 4.0 * total + 4.0 * T * (H / 2 + 1) * (W / 2 + 1), st);
  keep_map_kernel<<<blocks > 0 ? blocks : 1, 256, 0, st>>>(T, H, W, keep_idx, near_idx);
  return cuda_check(cudaGetLastError(), "keep_map_kernel");
}

fsdit_status launch_gather(const float* x, const int32_t* pos, float* xc, int32_t* posc, const int32_t* keep_idx,
                           int n_keep, int n_grid, int n_rows, int hidden, cudaStream_t st) {
  const int n_out = n_keep + (n_rows - n_grid);
  ProfScope ps(PC_GATHER, 1, 0.0, 8.0 * n_out * (double)hidden + (pos ? 24.0 * n_out : 0.0), st);
  gather_rows_kernel<<<grid_for_rows(n_out, 8), 256, 0, st>>>(x, pos, xc, posc, keep_idx, n_keep, n_grid, n_out,
                                                              hidden);
  return cuda_check(cudaGetLastError(), "gather_rows_kernel");
}

fsdit_status launch_broadcast(const float* x, const float* yc, float* out, const int32_t* keep_idx,
                              const int32_t* near_idx, int n_keep, int grid_t, int grid_h, int grid_w, int n_rows,
                              int hidden, cudaStream_t st) {
  const int n_grid = grid_t * grid_h * grid_w;
  const int n_blocks = n_keep + (n_rows - n_grid);
  // unique bytes: every grid row of x read once, y_c read once, every row written once
  ProfScope ps(PC_BCAST, 1, 0.0, ((double)n_grid + n_blocks + n_rows) * hidden * 4.0, st);
  broadcast_kernel<<<grid_for_rows(n_blocks, 8), 256, 0, st>>>(x, yc, out, keep_idx, near_idx, n_keep, grid_h,
                                                               grid_w, n_grid, n_rows, hidden);
  return cuda_check(cudaGetLastError(), "broadcast_kernel");
}

fsdit_status launch_rmsnorm_cast(const float* x, const void* g, void* xn, int rows, int hidden, float eps, int dtype,
                                 cudaStream_t st) {
  if (rows <= 0) return FSDIT_OK;
  const double s = dtype == FSDIT_BF16 ? 2.0 : 4.0;
  ProfScope ps(PC_NORM, 1, 0.0, (double)rows * hidden * (4.0 + s) + hidden * s, st);
  if (dtype == FSDIT_BF16)
    rmsnorm_cast_kernel<bf16><<<rows, 256, 0, st>>>(x, (const bf16*)g, (bf16*)xn, rows, hidden, eps);
  else
    rmsnorm_cast_kernel<float><<<rows, 256, 0, st>>>(x, (const float*)g, (float*)xn, rows, hidden, eps);
  return cuda_check(cudaGetLastError(), "rmsnorm_cast_kernel");
}

template <typename TW>
static fsdit_status embed_t(float* x, int hidden, int row0, int rows, int kind, const float* lat, int K,
                            const void* w_in, const void* b_in, const float* text_proj, const void* mod_emb,
                            const float* temb, const uint8_t* modality, const uint8_t* time_id, int n_times,
                            int ea, int eb, cudaStream_t st) {
  if (rows <= 0) return FSDIT_OK;
  dim3 grid((rows + EMB_RB - 1) / EMB_RB, (hidden + EMB_CB - 1) / EMB_CB);
  ProfScope ps(PC_EMBED, 1, 2.0 * rows * (double)hidden * K,
               (double)rows * hidden * 4.0 * (kind == 0 ? 2.0 : 1.0) + (double)rows * K * 4.0 +
                   (double)hidden * K * sizeof(TW),
               st);
  if (K <= 24)
    embed_kernel<TW, 24><<<grid, EMB_CB, 0, st>>>(x, hidden, row0, rows, kind, lat, K, (const TW*)w_in,
                                                  (const TW*)b_in, text_proj, (const TW*)mod_emb, temb, modality,
                                                  time_id, n_times, ea, eb);
  else if (K <= 32)
    embed_kernel<TW, 32><<<grid, EMB_CB, 0, st>>>(x, hidden, row0, rows, kind, lat, K, (const TW*)w_in,
                                                  (const TW*)b_in, text_proj, (const TW*)mod_emb, temb, modality,
                                                  time_id, n_times, ea, eb);
  else
    embed_kernel<TW, 64><<<grid, EMB_CB, 0, st>>>(x, hidden, row0, rows, kind, lat, K, (const TW*)w_in,
                                                  (const TW*)b_in, text_proj, (const TW*)mod_emb, temb, modality,
                                                  time_id, n_times, ea, eb);
  return cuda_check(cudaGetLastError(), "embed_kernel");
}

fsdit_status launch_embed(int dtype, float* x, int hidden, int row0, int rows, int kind, const float* lat, int K,
                          const void* w_in, const void* b_in, const float* text_proj, const void* mod_emb,
                          const float* temb, const uint8_t* modality, const uint8_t* time_id, int n_times, int ea,
                          int eb, cudaStream_t st) {
  if (dtype == FSDIT_BF16)
    return embed_t<bf16>(x, hidden, row0, rows, kind, lat, K, w_in, b_in, text_proj, mod_emb, temb, modality,
                         time_id, n_times, ea, eb, st);
  return embed_t<float>(x, hidden, row0, rows, kind, lat, K, w_in, b_in, text_proj, mod_emb, temb, modality,
                        time_id, n_times, ea, eb, st);
}

fsdit_status launch_time_mlp(int dtype, const float* times_host, int n_times, int t_freq, const void* w1,
                             const void* b1, const void* w2, const void* b2, float* h1, float* temb, int hidden,
                             cudaStream_t st) {
  const size_t sm1 = (size_t)n_times * t_freq * sizeof(float);
  ProfScope ps(PC_TIMEMLP, 2, 2.0 * n_times * (double)hidden * (t_freq + hidden),
               (double)hidden * (t_freq + hidden) * (dtype == FSDIT_BF16 ? 2.0 : 4.0), st);
  Times8 times_dev;
  for (int i = 0; i < 8; ++i) times_dev.t[i] = i < n_times ? times_host[i] : 0.f;
  const int blocks1 = num_sms() * 2;
  const int blocks2 = (hidden + 7) / 8;  // one warp per output column
  if (dtype == FSDIT_BF16) {
    time_mlp1_kernel<bf16><<<blocks1, 256, sm1, st>>>(times_dev, n_times, t_freq, (const bf16*)w1, (const bf16*)b1,
                                                      h1, hidden);
    time_mlp2_kernel<bf16><<<blocks2, 256, 0, st>>>(h1, n_times, (const bf16*)w2, (const bf16*)b2, temb, hidden);
  } else {
    time_mlp1_kernel<float><<<blocks1, 256, sm1, st>>>(times_dev, n_times, t_freq, (const float*)w1,
                                                       (const float*)b1, h1, hidden);
    time_mlp2_kernel<float><<<blocks2, 256, 0, st>>>(h1, n_times, (const float*)w2, (const float*)b2, temb, hidden);
  }
  return cuda_check(cudaGetLastError(), "time_mlp kernels");
}

fsdit_status launch_rope_table(const int32_t* pos, int rows, int head_dim, int s0, int s1, float log2_theta,
                               float2* cs, cudaStream_t st) {
  if (rows <= 0) return FSDIT_OK;
  const size_t total = (size_t)rows * (head_dim / 2);
  size_t blocks = (total + 255) / 256;
  const size_t cap = (size_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  ProfScope ps(PC_ROPE, 1, 0.0, 12.0 * rows + 8.0 * total, st);
  rope_table_kernel<<<(unsigned)blocks, 256, 0, st>>>(pos, rows, head_dim, s0, s1, log2_theta, cs);
  return cuda_check(cudaGetLastError(), "rope_table_kernel");
}

fsdit_status launch_euler(float* x, const float* v, const uint8_t* mod, const uint8_t* mask, int n_rows, int width,
                          const float* t_cur, const float* t_next, cudaStream_t st) {
  Clock4 c;
  for (int i = 0; i < 4; ++i) c.dt[i] = t_next[i] - t_cur[i];
  const size_t total = (size_t)n_rows * width;
  size_t blocks = (total + 255) / 256;
  const size_t cap = (size_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks == 0) blocks = 1;
  ProfScope ps(PC_EULER, 1, 2.0 * total, 12.0 * total + 2.0 * n_rows, st);
  euler_kernel<<<(unsigned)blocks, 256, 0, st>>>(x, v, mod, mask, n_rows, width, c);
  return cuda_check(cudaGetLastError(), "euler_kernel");
}

}  // namespace fsdit
