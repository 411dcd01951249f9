// Shared device helpers of libfsdit (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/fsdit.h"

namespace fsdit {

typedef __nv_bfloat16 bf16;

// Device error word: kernels that give up a bounded wait set it; the host
// reads it through fsdit_device_error().
__device__ int g_device_error = 0;  // one translation unit (libfsdit.cu) includes every source

enum { DEVERR_TIMEOUT = 1, DEVERR_TAGS = 2, DEVERR_KEEPMAP = 4 };

__device__ __forceinline__ void raise_device_error(int code) { atomicOr(&g_device_error, code); }

// Host-side values that belong to one device's context (kernel attributes,
// occupancy, SM count) are computed once per device, on first use with that
// device current, so a process may drive several GPUs.
constexpr int MAX_DEVICES = 64;
template <typename T>
struct PerDevice {
  std::mutex mu;
  bool done[MAX_DEVICES] = {};
  T val[MAX_DEVICES] = {};
  // `init` runs with the device current; `on_error` is returned when the
  // current device cannot be read or lies beyond MAX_DEVICES.
  template <typename F>
  T get(F init, T on_error) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
      (void)cudaGetLastError();
      return on_error;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
      val[dev] = init();
      done[dev] = true;
    }
    return val[dev];
  }
};

template <typename T> __device__ __forceinline__ float ld_f32(const T* p);
template <> __device__ __forceinline__ float ld_f32<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float ld_f32<bf16>(const bf16* p) { return __bfloat162float(*p); }

template <typename T> __device__ __forceinline__ T cvt_from_f32(float v);
template <> __device__ __forceinline__ float cvt_from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 cvt_from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ float gelu_tanh(float x) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  const float k1 = 0.044715f;
  return 0.5f * x * (1.0f + tanhf(k0 * (x + k1 * x * x * x)));
}

// 3D RoPE rotation of one interleaved pair.  `d` is the even channel index of
// the pair inside its head; the head is cut into chunks of s0 (t), s1 (h) and
// the rest (w) channels; inside chunk a (width da, pair jj) the pair turns by
// pos_a * theta^(-2 jj / da).
__device__ __forceinline__ void rope_pair(float& a, float& b, int d, int s0, int s1, int head_dim,
                                          const int32_t* pos3, float log2_theta) {
  int axis, off, da;
  if (d < s0) { axis = 0; off = 0; da = s0; }
  else if (d < s0 + s1) { axis = 1; off = s0; da = s1; }
  else { axis = 2; off = s0 + s1; da = head_dim - s0 - s1; }
  const float jj = (float)((d - off) >> 1);
  const float inv_freq = exp2f(-(2.0f * jj / (float)da) * log2_theta);
  const float ang = (float)pos3[axis] * inv_freq;
  float s, c;
  sincosf(ang, &s, &c);
  const float na = a * c - b * s;
  const float nb = a * s + b * c;
  a = na;
  b = nb;
}

struct EpiParams {
  int epi;              // FSDIT_EPI_*
  const void* bias;     // [N], weight dtype
  void* out;            // [M, ldo]
  int ldo;
  const float* resid;   // [M, ldr] (FSDIT_EPI_RESIDUAL)
  int ldr;
  const int32_t* pos;   // [M][3] (FSDIT_EPI_QKV_ROPE)
  const float2* rope_cs;  // [M][head_dim/2] (cos, sin) per pair, or null: compute from pos
  int rope_cols;        // columns [0, rope_cols) are rotated
  int head_dim, s0, s1;
  float log2_theta;
  const float* row_scale;  // [M] or null: accumulators are multiplied by
  const float* col_scale;  // row_scale[row] * col_scale[col] (FP8 dequantization) before the bias
  int up_h, up_w;          // EPI_UNPATCH: the rows are the cells of a (t, h, w) grid up_h x up_w per frame,
  int up_c, up_pt, up_ps;  // each column a pixel of the cell's up_c x up_pt x up_ps x up_ps patch
  int up_rgb8;             // EPI_UNPATCH: 1 = write 8-bit codes (rgb8_code) instead of fp32 values
  float* split_part;       // pair GEMM tail cut: caller scratch for the partial accumulators
  int* split_cnt;          // (SPLIT_WS_BYTES) and its zeroed counters (SPLIT_CNT_BYTES), or null: no cut
  // RMSNorm applied after the GEMM (bf16 tensor-core kernels): a RESIDUAL
  // producer also writes the next norm's operand, xg[row * ldo + col] =
  // bf16(out * xg_gain[col]), and the sums of out^2 over each 128-column
  // group p, ss_part[row * ss_ld + p] (N % 128 == 0, whole tiles); a consumer
  // (operand bf16(x * g)) with norm_ss set scales its accumulators before the
  // bias by 1/rms(x) = rsqrt(sum of the norm_h / 128 groups of
  // norm_ss[row * ss_ld ..] in group order / norm_h + norm_eps).
  bf16* xg = nullptr;
  const bf16* xg_gain = nullptr;
  float* ss_part = nullptr;
  int ss_ld = 0;
  const float* norm_ss = nullptr;
  int norm_h = 0;
  float norm_eps = 0.0f;
};

// Scratch of the pair GEMM's tail cut: 128 units of 256 KB fp32 partials and
// 64 x 16 int counters (zero between launches; each launch leaves them zero).
constexpr size_t SPLIT_WS_BYTES = (size_t)128 << 18;
constexpr size_t SPLIT_CNT_BYTES = 64 * 16 * 4;

// Decoder pixel head (internal epilogue, not reachable through fsdit_linear):
// out (f32) = acc + b written straight into frames [F][up_c][up_h*ps][up_w*ps].
// Column (c, dt, dy, dx) of cell (t, h, w), dx fastest, is frame
// pt*t + dt - (pt - 1) (dropped when negative: latent frame 0 yields one
// frame), pixel (ps*h + dy, ps*w + dx).
constexpr int EPI_UNPATCH = 5;

// Colour conversion of a decoder value to its 8-bit code: 127.5 * (v + 1) as
// a rounded product and a rounded sum in fp32, clamped to [0, 255], rounded
// to the nearest integer (ties to even).
__device__ __forceinline__ uint32_t rgb8_code(float v) {
  const float t = fminf(fmaxf(__fadd_rn(__fmul_rn(v, 127.5f), 127.5f), 0.0f), 255.0f);
  return (uint32_t)__float2int_rn(t);
}

// Element offset of column `col` of row `row` in the frames, -1 if dropped.
__device__ __forceinline__ long long unpatch_offset(const EpiParams& p, int row, int col) {
  const int ps = p.up_ps, pt = p.up_pt;
  const int dx = col % ps, r1 = col / ps;
  const int dy = r1 % ps, r2 = r1 / ps;
  const int dt = r2 % pt, ch = r2 / pt;
  const int w = row % p.up_w, r = row / p.up_w;
  const int h = r % p.up_h, t = r / p.up_h;
  const int f = t * pt + dt - (pt - 1);
  if (f < 0) return -1;
  const long long hp = (long long)p.up_h * ps, wp = (long long)p.up_w * ps;
  return (((long long)f * p.up_c + ch) * hp + (long long)h * ps + dy) * wp + (long long)w * ps + dx;
}

// Apply the epilogue to `cnt` consecutive columns [col, col+cnt) of one row.
// v[] holds the fp32 accumulators; cnt is even and col is even.
// 1/rms of `row` from its producer's per-group sums of squares (the same
// order in every tile and kernel, so every tile of a row scales it alike).
__device__ __forceinline__ float norm_rstd(const EpiParams& p, int row) {
  const float* ss = p.norm_ss + (size_t)row * p.ss_ld;
  const int groups = p.norm_h >> 7;
  float t = 0.0f;
  int g = 0;
  for (; g + 8 <= groups; g += 8) {  // eight loads in flight, added in order
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = __ldg(ss + g + k);
#pragma unroll
    for (int k = 0; k < 8; ++k) t += a[k];
  }
  for (; g < groups; ++g) t += __ldg(ss + g);
  return rsqrtf(t / (float)p.norm_h + p.norm_eps);
}

// Returns the sum of squares of the RESIDUAL outputs when p.xg is set, else 0.
template <typename TW, int CNT>
__device__ __forceinline__ float epilogue_row(const EpiParams& p, int row, int col, float* v) {
  if (p.col_scale != nullptr) {
    const float rs = p.row_scale[row];
#pragma unroll
    for (int i = 0; i < CNT; ++i) v[i] *= rs * p.col_scale[col + i];
  }
  if (p.norm_ss != nullptr) {
    const float rs = norm_rstd(p, row);
#pragma unroll
    for (int i = 0; i < CNT; ++i) v[i] *= rs;
  }
  const TW* bias = reinterpret_cast<const TW*>(p.bias);
#pragma unroll
  for (int i = 0; i < CNT; ++i) v[i] += ld_f32<TW>(bias + col + i);
  if (p.epi == FSDIT_EPI_QKV_ROPE) {
    if (col < p.rope_cols) {
      if (p.rope_cs != nullptr) {
        // CNT consecutive columns of one head: pairs (col % head_dim)/2 ..
        const float2* cs = p.rope_cs + (size_t)row * (p.head_dim >> 1) + ((col % p.head_dim) >> 1);
#pragma unroll
        for (int i = 0; i < CNT; i += 2) {
          const float2 t = cs[i >> 1];
          const float a = v[i], b = v[i + 1];
          v[i] = a * t.x - b * t.y;
          v[i + 1] = a * t.y + b * t.x;
        }
      } else {
        const int32_t* pos3 = p.pos + (size_t)row * 3;
#pragma unroll
        for (int i = 0; i < CNT; i += 2) {
          int d = (col + i) % p.head_dim;
          rope_pair(v[i], v[i + 1], d, p.s0, p.s1, p.head_dim, pos3, p.log2_theta);
        }
      }
    }
  } else if (p.epi == FSDIT_EPI_GELU) {
#pragma unroll
    for (int i = 0; i < CNT; ++i) v[i] = gelu_tanh(v[i]);
  }
  if (p.epi == EPI_UNPATCH) {
#pragma unroll
    for (int i = 0; i < CNT; ++i) {
      const long long off = unpatch_offset(p, row, col + i);
      if (off < 0) continue;
      if (p.up_rgb8) reinterpret_cast<uint8_t*>(p.out)[off] = (uint8_t)rgb8_code(v[i]);
      else reinterpret_cast<float*>(p.out)[off] = v[i];
    }
  } else if (p.epi == FSDIT_EPI_RESIDUAL) {
    const float* r = p.resid + (size_t)row * p.ldr + col;
    float* o = reinterpret_cast<float*>(p.out) + (size_t)row * p.ldo + col;
    float ss = 0.0f;
    if constexpr (CNT % 4 == 0) {
#pragma unroll
      for (int i = 0; i < CNT; i += 4) {
        float4 rv = *reinterpret_cast<const float4*>(r + i);
        float4 ov = make_float4(rv.x + v[i], rv.y + v[i + 1], rv.z + v[i + 2], rv.w + v[i + 3]);
        *reinterpret_cast<float4*>(o + i) = ov;
        if (p.xg != nullptr) {
          const bf16* g = p.xg_gain + col + i;
          __nv_bfloat162 h0 = __floats2bfloat162_rn(ov.x * __bfloat162float(g[0]), ov.y * __bfloat162float(g[1]));
          __nv_bfloat162 h1 = __floats2bfloat162_rn(ov.z * __bfloat162float(g[2]), ov.w * __bfloat162float(g[3]));
          *reinterpret_cast<uint2*>(p.xg + (size_t)row * p.ldo + col + i) =
              make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
          ss += ov.x * ov.x + ov.y * ov.y + ov.z * ov.z + ov.w * ov.w;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < CNT; ++i) o[i] = r[i] + v[i];
    }
    return ss;
  } else if (p.epi == FSDIT_EPI_BIAS_F32) {
    float* o = reinterpret_cast<float*>(p.out) + (size_t)row * p.ldo + col;
    if constexpr (CNT % 4 == 0) {
#pragma unroll
      for (int i = 0; i < CNT; i += 4)
        *reinterpret_cast<float4*>(o + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < CNT; ++i) o[i] = v[i];
    }
  } else {
    TW* o = reinterpret_cast<TW*>(p.out) + (size_t)row * p.ldo + col;
    if constexpr (sizeof(TW) == 2 && CNT % 8 == 0) {
#pragma unroll
      for (int i = 0; i < CNT; i += 8) {
        __nv_bfloat162 h0 = __floats2bfloat162_rn(v[i], v[i + 1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(v[i + 2], v[i + 3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(v[i + 4], v[i + 5]);
        __nv_bfloat162 h3 = __floats2bfloat162_rn(v[i + 6], v[i + 7]);
        uint4 u;
        u.x = *reinterpret_cast<uint32_t*>(&h0);
        u.y = *reinterpret_cast<uint32_t*>(&h1);
        u.z = *reinterpret_cast<uint32_t*>(&h2);
        u.w = *reinterpret_cast<uint32_t*>(&h3);
        *reinterpret_cast<uint4*>(o + i) = u;
      }
    } else {
#pragma unroll
      for (int i = 0; i < CNT; ++i) o[i] = cvt_from_f32<TW>(v[i]);
    }
  }
  return 0.0f;
}

// ------------------------------------------------ tensor-core GEMM epilogue
// The bf16 tensor-core kernels hold one accumulator row per thread in chunks
// of 32 columns.  Everything a chunk needs besides its accumulators (bias, the
// RoPE (cos, sin) pairs or the fp32 residual) is loaded by epi32_prefetch
// before the accumulators are read out of TMEM, so the two latencies overlap.
struct Epi32Pre {
  uint4 bias[4];    // 32 bf16 bias values (the same for every row)
  float4 extra[8];  // QKV_ROPE: 16 (cos, sin) pairs; RESIDUAL: 32 fp32 residual values
  float4 cscale[8]; // FP8 dequantization: 32 column scales (same for every row)
  float rscale;     //                     and this row's scale
  float rrs;        // 1/rms of the row (RMSNorm after the GEMM)
};

// GELU (tanh form) with the hardware tanh approximation (relative error about
// 2^-11), used where the result is rounded to bf16 (2^-9) next.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float gelu_tanh_bf16out(float x) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  const float k1 = 0.044715f;
  return 0.5f * x * (1.0f + tanh_approx(k0 * (x + k1 * x * x * x)));
}

// Columns [col, col + 32) of `row`, all inside the output (col + 32 <= N);
// bias, out, resid and rope_cs 16-byte aligned, head_dim a power of two.
__device__ __forceinline__ void epi32_prefetch(const EpiParams& p, int row, int col, Epi32Pre& e) {
  const uint4* b = reinterpret_cast<const uint4*>(reinterpret_cast<const bf16*>(p.bias) + col);
#pragma unroll
  for (int i = 0; i < 4; ++i) e.bias[i] = __ldg(b + i);
  if (p.col_scale != nullptr) {
    const float4* cs = reinterpret_cast<const float4*>(p.col_scale + col);
#pragma unroll
    for (int i = 0; i < 8; ++i) e.cscale[i] = __ldg(cs + i);
    e.rscale = __ldg(p.row_scale + row);
  }
  if (p.norm_ss != nullptr) e.rrs = norm_rstd(p, row);
  if (p.epi == FSDIT_EPI_QKV_ROPE) {
    if (col < p.rope_cols && p.rope_cs != nullptr) {
      const float4* cs = reinterpret_cast<const float4*>(p.rope_cs + (size_t)row * (p.head_dim >> 1) +
                                                         ((col & (p.head_dim - 1)) >> 1));
#pragma unroll
      for (int i = 0; i < 8; ++i) e.extra[i] = __ldg(cs + i);
    }
  } else if (p.epi == FSDIT_EPI_RESIDUAL) {
    const float4* r = reinterpret_cast<const float4*>(p.resid + (size_t)row * p.ldr + col);
#pragma unroll
    for (int i = 0; i < 8; ++i) e.extra[i] = r[i];
  }
}

__device__ __forceinline__ void epi32_apply(const EpiParams& p, int row, int col, float* v, const Epi32Pre& e) {
  if (p.col_scale != nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[4 * i] *= e.rscale * e.cscale[i].x;
      v[4 * i + 1] *= e.rscale * e.cscale[i].y;
      v[4 * i + 2] *= e.rscale * e.cscale[i].z;
      v[4 * i + 3] *= e.rscale * e.cscale[i].w;
    }
  }
  if (p.norm_ss != nullptr) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= e.rrs;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&e.bias[i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h[j]);
      v[8 * i + 2 * j] += f.x;
      v[8 * i + 2 * j + 1] += f.y;
    }
  }
  if (p.epi == FSDIT_EPI_QKV_ROPE) {
    if (col < p.rope_cols && p.rope_cs == nullptr) {
      const int32_t* pos3 = p.pos + (size_t)row * 3;
#pragma unroll
      for (int i = 0; i < 32; i += 2)
        rope_pair(v[i], v[i + 1], (col + i) & (p.head_dim - 1), p.s0, p.s1, p.head_dim, pos3, p.log2_theta);
    } else if (col < p.rope_cols) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 t = e.extra[i];  // (cos, sin) of pairs 2i and 2i+1
        float a = v[4 * i], b = v[4 * i + 1];
        v[4 * i] = a * t.x - b * t.y;
        v[4 * i + 1] = a * t.y + b * t.x;
        a = v[4 * i + 2];
        b = v[4 * i + 3];
        v[4 * i + 2] = a * t.z - b * t.w;
        v[4 * i + 3] = a * t.w + b * t.z;
      }
    }
  } else if (p.epi == FSDIT_EPI_GELU) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = gelu_tanh_bf16out(v[i]);
  }
  if (p.epi == EPI_UNPATCH) {
    // up_ps % 4 == 0: each group of 4 columns is 4 adjacent pixels of one
    // pixel row, 16-byte aligned in fp32 frames, 4-byte aligned in 8-bit ones
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const long long off = unpatch_offset(p, row, col + 4 * i);
      if (off < 0) continue;
      if (p.up_rgb8)
        *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(p.out) + off) =
            rgb8_code(v[4 * i]) | (rgb8_code(v[4 * i + 1]) << 8) | (rgb8_code(v[4 * i + 2]) << 16) |
            (rgb8_code(v[4 * i + 3]) << 24);
      else
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + off) =
            make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  } else if (p.epi == FSDIT_EPI_RESIDUAL) {
    float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (size_t)row * p.ldo + col);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 r = e.extra[i];
      o[i] = make_float4(r.x + v[4 * i], r.y + v[4 * i + 1], r.z + v[4 * i + 2], r.w + v[4 * i + 3]);
    }
  } else if (p.epi == FSDIT_EPI_BIAS_F32) {
    float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (size_t)row * p.ldo + col);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  } else {
    uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(p.out) + (size_t)row * p.ldo + col);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * i + 2 * j], v[8 * i + 2 * j + 1]);
        u[j] = *reinterpret_cast<uint32_t*>(&h);
      }
      o[i] = make_uint4(u[0], u[1], u[2], u[3]);
    }
  }
}

// ------------------------------- coalesced epilogue of a warp's 32 x 32 block
// After tcgen05.ld lane r of a warp holds the 32 columns of row r of a 32 x 32
// accumulator block, so every lane's bias / residual / RoPE-table / output
// access hits a different row: one 16-byte piece per row and instruction.
// warp_transpose32 passes the block through 4 KB of the warp's shared memory
// (16-byte pieces, XOR-swizzled so that neither the writes nor the reads
// conflict) so that lane l then holds columns 4*(l%8) .. 4*(l%8)+3 of rows
// l/8 + 4i, i = 0..7: eight lanes share one row's 128 contiguous bytes and
// each global access of the epilogue covers four rows.  The arithmetic per
// element is that of epi32_apply, in the same order.
__device__ __forceinline__ void warp_transpose32(float4* buf, const float* v, float* w, int lane) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    buf[lane * 8 + (j ^ (lane & 7))] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = (lane >> 3) + 4 * i;
    const float4 t = buf[r * 8 + ((lane & 7) ^ (r & 7))];
    w[4 * i] = t.x;
    w[4 * i + 1] = t.y;
    w[4 * i + 2] = t.z;
    w[4 * i + 3] = t.w;
  }
  __syncwarp();  // the block is read before the buffer is written again
}

// Per-lane inputs of the transposed block (columns cl .. cl+3 of rows r0 + 4i).
struct EpiTPre {
  uint2 bias;       // the 4 bf16 bias values of the lane's columns
  float4 cscale;    // FP8 dequantization: the 4 column scales
  float rscale[8];  //                     and the row scale of each of the 8 rows
  float4 extra[8];  // QKV_ROPE: (cos, sin) of the lane's 2 pairs; RESIDUAL: 4 fp32 values; per row
  float rrs[8];     // 1/rms of each of the 8 rows
  uint2 gain;       // RESIDUAL producer: the 4 bf16 gains of the lane's columns
};

// Loads for columns [col, col + 32) (all inside the output) of the block whose
// first row is row0; rows at or past M are skipped.  Alignment as for
// epi32_prefetch.
// lane_rstd: with p.norm_ss, 1/rms of row row0 + lane (norm_rstd), computed
// once per tile by the caller.
__device__ __forceinline__ void epiT_prefetch(const EpiParams& p, int row0, int col, int M, int lane,
                                              EpiTPre& e, float lane_rstd = 0.0f) {
  const int cl = col + 4 * (lane & 7);
  const int r0 = row0 + (lane >> 3);
  e.bias = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const bf16*>(p.bias) + cl));
  if (p.col_scale != nullptr) {
    e.cscale = __ldg(reinterpret_cast<const float4*>(p.col_scale + cl));
#pragma unroll
    for (int i = 0; i < 8; ++i) e.rscale[i] = r0 + 4 * i < M ? __ldg(p.row_scale + r0 + 4 * i) : 0.0f;
  }
  if (p.norm_ss != nullptr) {  // lane k holds row row0 + k's (whole warp, converged)
#pragma unroll
    for (int i = 0; i < 8; ++i) e.rrs[i] = __shfl_sync(0xffffffffu, lane_rstd, (lane >> 3) + 4 * i);
  }
  if (p.xg != nullptr) e.gain = __ldg(reinterpret_cast<const uint2*>(p.xg_gain + cl));
  if (p.epi == FSDIT_EPI_QKV_ROPE) {
    if (col < p.rope_cols && p.rope_cs != nullptr) {
      const int pair = (cl & (p.head_dim - 1)) >> 1;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (r0 + 4 * i < M)
          e.extra[i] = __ldg(reinterpret_cast<const float4*>(p.rope_cs + (size_t)(r0 + 4 * i) * (p.head_dim >> 1) +
                                                             pair));
    }
  } else if (p.epi == FSDIT_EPI_RESIDUAL) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (r0 + 4 * i < M) e.extra[i] = *reinterpret_cast<const float4*>(p.resid + (size_t)(r0 + 4 * i) * p.ldr + cl);
  }
}

// The epilogue of the transposed block w (w[4i + j] = column cl + j of row
// r0 + 4i): dequantization or the RMSNorm row scale, bias, RoPE / GELU, then
// the residual add and the store (with the next norm's operand and the lane's
// sums of squares added to ssq[i] when p.xg is set), or the unpatchify store.
__device__ __forceinline__ void epiT_apply(const EpiParams& p, int row0, int col, int M, int lane, float* w,
                                           const EpiTPre& e, float* ssq = nullptr) {
  const int cl = col + 4 * (lane & 7);
  const int r0 = row0 + (lane >> 3);
  if (p.col_scale != nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[4 * i] *= e.rscale[i] * e.cscale.x;
      w[4 * i + 1] *= e.rscale[i] * e.cscale.y;
      w[4 * i + 2] *= e.rscale[i] * e.cscale.z;
      w[4 * i + 3] *= e.rscale[i] * e.cscale.w;
    }
  }
  if (p.norm_ss != nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[4 * i] *= e.rrs[i];
      w[4 * i + 1] *= e.rrs[i];
      w[4 * i + 2] *= e.rrs[i];
      w[4 * i + 3] *= e.rrs[i];
    }
  }
  {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&e.bias);
    const float2 b01 = __bfloat1622float2(h[0]), b23 = __bfloat1622float2(h[1]);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[4 * i] += b01.x;
      w[4 * i + 1] += b01.y;
      w[4 * i + 2] += b23.x;
      w[4 * i + 3] += b23.y;
    }
  }
  if (p.epi == FSDIT_EPI_QKV_ROPE) {
    if (col < p.rope_cols && p.rope_cs == nullptr) {
      // angles from the positions (rope_pair's arithmetic): the lane's two
      // pairs keep their axis and frequency across its eight rows
      int axis[2];
      float inv_freq[2];
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int d = (cl + 2 * m) & (p.head_dim - 1);
        int off, da;
        if (d < p.s0) { axis[m] = 0; off = 0; da = p.s0; }
        else if (d < p.s0 + p.s1) { axis[m] = 1; off = p.s0; da = p.s1; }
        else { axis[m] = 2; off = p.s0 + p.s1; da = p.head_dim - p.s0 - p.s1; }
        const float jj = (float)((d - off) >> 1);
        inv_freq[m] = exp2f(-(2.0f * jj / (float)da) * p.log2_theta);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (r0 + 4 * i >= M) continue;
        const int32_t* pos3 = p.pos + (size_t)(r0 + 4 * i) * 3;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const float ang = (float)__ldg(pos3 + axis[m]) * inv_freq[m];
          float sn, cs;
          sincosf(ang, &sn, &cs);
          const float a = w[4 * i + 2 * m], b = w[4 * i + 2 * m + 1];
          w[4 * i + 2 * m] = a * cs - b * sn;
          w[4 * i + 2 * m + 1] = a * sn + b * cs;
        }
      }
    } else if (col < p.rope_cols) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 t = e.extra[i];  // (cos, sin) of the lane's two pairs
        float a = w[4 * i], b = w[4 * i + 1];
        w[4 * i] = a * t.x - b * t.y;
        w[4 * i + 1] = a * t.y + b * t.x;
        a = w[4 * i + 2];
        b = w[4 * i + 3];
        w[4 * i + 2] = a * t.z - b * t.w;
        w[4 * i + 3] = a * t.w + b * t.z;
      }
    }
  } else if (p.epi == FSDIT_EPI_GELU) {
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i] = gelu_tanh_bf16out(w[i]);
  }
  if (p.epi == EPI_UNPATCH) {
    // unpatch_offset's mapping with its divisions done once: the lane's
    // columns fix (channel, dt, dy, dx) and its rows are the cells r0 + 4i,
    // stepped four cells at a time through (t, h, w)
    const int ps = p.up_ps, pt = p.up_pt;
    const int dx = cl % ps, c1 = cl / ps;
    const int dy = c1 % ps, c2 = c1 / ps;
    const int dt = c2 % pt, ch = c2 / pt;
    int cw = r0 % p.up_w, ct = r0 / p.up_w;
    int chh = ct % p.up_h;
    ct /= p.up_h;
    const long long hp = (long long)p.up_h * ps, wp = (long long)p.up_w * ps;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int f = ct * pt + dt - (pt - 1);
      if (r0 + 4 * i < M && f >= 0) {  // up_ps % 4 == 0: 4 adjacent pixels of one pixel row
        const float* x = w + 4 * i;
        const long long off =
            (((long long)f * p.up_c + ch) * hp + (long long)chh * ps + dy) * wp + (long long)cw * ps + dx;
        if (p.up_rgb8)
          *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(p.out) + off) =
              rgb8_code(x[0]) | (rgb8_code(x[1]) << 8) | (rgb8_code(x[2]) << 16) | (rgb8_code(x[3]) << 24);
        else
          *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + off) = make_float4(x[0], x[1], x[2], x[3]);
      }
      cw += 4;
      while (cw >= p.up_w) {  // at most 4 / up_w + 1 steps
        cw -= p.up_w;
        if (++chh == p.up_h) {
          chh = 0;
          ++ct;
        }
      }
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = r0 + 4 * i;
    if (row >= M) continue;
    const float* x = w + 4 * i;
    if (p.epi == FSDIT_EPI_RESIDUAL) {
      const float4 r = e.extra[i];
      const float4 o = make_float4(r.x + x[0], r.y + x[1], r.z + x[2], r.w + x[3]);
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (size_t)row * p.ldo + cl) = o;
      if (p.xg != nullptr) {
        const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&e.gain.x));
        const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&e.gain.y));
        __nv_bfloat162 h0 = __floats2bfloat162_rn(o.x * g01.x, o.y * g01.y);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(o.z * g23.x, o.w * g23.y);
        *reinterpret_cast<uint2*>(p.xg + (size_t)row * p.ldo + cl) =
            make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
        ssq[i] += o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
      }
    } else if (p.epi == FSDIT_EPI_BIAS_F32) {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (size_t)row * p.ldo + cl) =
          make_float4(x[0], x[1], x[2], x[3]);
    } else {
      __nv_bfloat162 h0 = __floats2bfloat162_rn(x[0], x[1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(x[2], x[3]);
      *reinterpret_cast<uint2*>(reinterpret_cast<bf16*>(p.out) + (size_t)row * p.ldo + cl) =
          make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
    }
  }
}

}  // namespace fsdit

// Host-side internal API shared by the .cu files.
namespace fsdit {
// Launch profiler: while fsdit_profile_start() is active, every launch scope
// records a CUDA event pair on its stream plus the algorithmic FLOPs / bytes
// of the work it launches (host arithmetic; nothing is read back until stop).
enum ProfClass {
  PC_GEMM_QKV, PC_GEMM_RESID, PC_GEMM_GELU, PC_GEMM_BIAS_F32, PC_GEMM_BIAS, PC_ATTN, PC_NORM,
  PC_GATHER, PC_BCAST, PC_EMBED, PC_TIMEMLP, PC_HEADS, PC_EULER, PC_KEEPMAP, PC_ROPE, PC_HISTORY, PC_QUANT,
  PC_GEMM_FP8_QKV, PC_GEMM_FP8_RESID, PC_GEMM_FP8_GELU, PC_GRID_POS, PC_PIXEL_HEAD, PC_COUNT
};
struct ProfScope {
  ProfScope(int cls, int kernels, double flops, double bytes, cudaStream_t st);
  ~ProfScope();
  void add_kernels(int k);
  int slot;
  cudaStream_t st;
};
// Count k more kernels in the projection launch scope open on this thread.
void prof_add_kernels(int k);

int num_sms();
void set_error(const char* fmt, ...);
fsdit_status cuda_check(cudaError_t e, const char* what);

fsdit_status launch_linear(const fsdit_dims* d, const void* a, const void* w, const EpiParams& ep,
                           int M, int N, int K, cudaStream_t st, int prof_cls = -1);
fsdit_status launch_linear_simt(int dtype, const void* a, const void* w, const EpiParams& ep,
                                int M, int N, int K, cudaStream_t st);
fsdit_status launch_linear_tc(const void* a, const void* w, const EpiParams& ep, int M, int N,
                              int K, cudaStream_t st);
fsdit_status launch_attention(const fsdit_dims* d, const void* qkv, void* out, int n,
                              cudaStream_t st);
fsdit_status launch_linear_fp8(const fsdit_dims* d, const uint8_t* qa, const void* qw, const EpiParams& ep, int M,
                               int N, int K, cudaStream_t st);
fsdit_status launch_linear_fp8_tc(const uint8_t* qa, const uint8_t* qw, const EpiParams& ep, int M, int N, int K,
                                  cudaStream_t st);
fsdit_status launch_quant_rows(const void* a, int dtype, int rows, int cols, uint8_t* q, float* s, cudaStream_t st);
fsdit_status launch_rmsnorm_quant(const float* x, const void* g, int rows, int hidden, float eps, uint8_t* q,
                                  float* s, cudaStream_t st);
fsdit_status launch_attention_simt(int dtype, const void* qkv, void* out, int n, int heads,
                                   int hidden, cudaStream_t st);
fsdit_status launch_attention_tc(const void* qkv, void* out, int n, int heads, int attn,
                                 cudaStream_t st);
// CTA-pair attention for long sequences (attn_pair.cu) and the row count from
// which launch_attention uses it.
fsdit_status launch_attention_pair(const void* qkv, void* out, int n, int heads, int attn, cudaStream_t st);
int attention_pair_min_rows();
}  // namespace fsdit
