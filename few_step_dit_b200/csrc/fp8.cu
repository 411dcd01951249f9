// FP8 (E4M3) quantization for the low-bit block projections ([PaperDaily]
// section 二, third step: low-bit weights and activations, quantization fused
// next to the normalization).
//
// One fp32 scale per row: s = amax / 448 (fp32 division; 1 for an all-zero
// row) and codes E4M3(v / s), the exact quotient rounded to nearest with
// ties to even, saturating at 448.  The quotient is not formed: each value
// is multiplied by r = fp32(1 / s), and the product t, within about one fp32
// ulp of the quotient, only picks the E4M3 interval; the side of that
// interval's midpoint m on which the exact quotient lies is then read off
// the sign of v - m * s, which one fused multiply-add gives exactly.
// Activations are quantized per token, weights per output channel (rows of
// [N, K]).

#include <type_traits>

namespace fsdit {
namespace q8 {

constexpr float E4M3_MAX = 448.0f;

// Two E4M3 codes, `lo` in the low byte.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  float m = 0.f;
  const int nw = blockDim.x >> 5;
  for (int i = 0; i < nw; ++i) m = fmaxf(m, red[i]);
  return m;
}

__device__ __forceinline__ float row_scale(float amax) { return amax > 0.f ? __fdiv_rn(amax, E4M3_MAX) : 1.0f; }

// 8 consecutive values as fp32.
template <typename T> __device__ __forceinline__ void load8(const T* p, float* v);
template <> __device__ __forceinline__ void load8<float>(const float* p, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <> __device__ __forceinline__ void load8<bf16>(const bf16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// The fp32 value whose round-to-nearest-even E4M3 conversion is the code of
// v / s (s > 0, rs = fp32(1 / s)).  t = |v| rs lies within about one fp32
// ulp of |v| / s, so the two can fall on different sides only of the
// midpoint m of the E4M3 interval holding t.  The interval is read from t's
// bits: above 2^-6 it keeps t's sign, exponent and top three mantissa bits
// (m sets the fourth and clears the rest); below 2^-6 E4M3 steps by 2^-9,
// the step of the binade [2^-6, 2^-5), so t is shifted up by 2^-6 and m back
// down (both exact).  fma(-m, s, |v|) is |v| - m s rounded once, so its sign
// is that of |v| / s - m (exact for s >= 2^-100: the difference is then a
// multiple of 2^-149).  The result is m itself for an exact tie (the
// conversion then picks the even code) or the fp32 neighbour of m on the
// quotient's side, with v's sign.
__device__ __forceinline__ float quotient_arg(float v, float s, float rs) {
  const float av = fabsf(v);
  const float t = __fmul_rn(av, rs);
  const bool low = t < 0.015625f;
  const float tb = low ? __fadd_rn(t, 0.015625f) : t;
  float m = __uint_as_float((__float_as_uint(tb) & 0xFFF00000u) | 0x00080000u);
  if (low) m = __fsub_rn(m, 0.015625f);
  const float r = __fmaf_rn(-m, s, av);
  const uint32_t mb = __float_as_uint(m);
  const float a = r > 0.f ? __uint_as_float(mb + 1u) : (r < 0.f ? __uint_as_float(mb - 1u) : m);
  return copysignf(a, v);
}

// Whether the product t = |v| rs (t >= 0) can round to another code than
// the exact quotient: t lies within 2 ulps of |v| / s, so only a t within 2
// ulps of an E4M3 midpoint can -- above 2^-6 the midpoints are the values
// whose low 20 bits are 0x80000 -- or a t below 2^-6, where the step is
// fixed (checked on the slow path, rare for scaled rows).
__device__ __forceinline__ bool near_midpoint(float t) {
  return t < 0.015625f || (__float_as_uint(t) & 0xFFFFFu) - 0x7FFFEu <= 4u;
}

// 8 codes of v[0..7] / s as one 8-byte word (rs: fp32(1 / s)).  With
// SCREEN the product decides every code far from a midpoint and only the few
// others take quotient_arg: the choice for fp32 rows, where about 1e-4 of the
// values need it.  bf16 rows hold ratios v / amax of two 8-bit significands,
// which put about 1% of the quotients within an ulp of a midpoint, so nearly
// every warp would take the second path; they run quotient_arg throughout.
template <bool SCREEN>
__device__ __forceinline__ uint2 codes8(const float* v, float s, float rs) {
  float a[8];
  if (!SCREEN) {
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = quotient_arg(v[i], s, rs);
    uint2 out;
    out.x = (uint32_t)e4m3x2(a[0], a[1]) | ((uint32_t)e4m3x2(a[2], a[3]) << 16);
    out.y = (uint32_t)e4m3x2(a[4], a[5]) | ((uint32_t)e4m3x2(a[6], a[7]) << 16);
    return out;
  }
  bool slow = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float t = __fmul_rn(fabsf(v[i]), rs);
    slow |= near_midpoint(t);
    a[i] = copysignf(t, v[i]);
  }
  if (slow) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (near_midpoint(fabsf(a[i]))) a[i] = quotient_arg(v[i], s, rs);
  }
  uint2 out;
  out.x = (uint32_t)e4m3x2(a[0], a[1]) | ((uint32_t)e4m3x2(a[2], a[3]) << 16);
  out.y = (uint32_t)e4m3x2(a[4], a[5]) | ((uint32_t)e4m3x2(a[6], a[7]) << 16);
  return out;
}

// 4 codes of v / s as one 32-bit word, the same way.
__device__ __forceinline__ uint32_t codes4(float4 v, float s, float rs) {
  const float in[4] = {v.x, v.y, v.z, v.w};
  float a[4];
  bool slow = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float t = __fmul_rn(fabsf(in[i]), rs);
    slow |= near_midpoint(t);
    a[i] = copysignf(t, in[i]);
  }
  if (slow) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (near_midpoint(fabsf(a[i]))) a[i] = quotient_arg(in[i], s, rs);
  }
  return (uint32_t)e4m3x2(a[0], a[1]) | ((uint32_t)e4m3x2(a[2], a[3]) << 16);
}

// 8 raw input values of a row kept in registers between the amax pass and
// the codes: packed for bf16 (16 bytes), as fp32 otherwise.
template <typename T> struct Raw8;
template <> struct Raw8<bf16> {
  uint4 u;
  __device__ __forceinline__ void load(const bf16* p) { u = *reinterpret_cast<const uint4*>(p); }
  __device__ __forceinline__ void get(float* v) const { load8<bf16>(reinterpret_cast<const bf16*>(&u), v); }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = *reinterpret_cast<const float4*>(p);
    b = *reinterpret_cast<const float4*>(p + 4);
  }
  __device__ __forceinline__ void get(float* v) const {
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};

// One 256-thread block per row (cols % 8 == 0, cols <= 256 * 8 * CH): the
// row is read once into registers, reduced to its amax, then turned into
// codes.
template <typename T, int CH>
__global__ void __launch_bounds__(256) quant_rows_kernel(const T* __restrict__ a, int cols, uint8_t* __restrict__ q,
                                                         float* __restrict__ s) {
  __shared__ float red[8];
  const int r = blockIdx.x;
  const T* ar = a + (size_t)r * cols;
  Raw8<T> raw[CH];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int c = (threadIdx.x + k * 256) * 8;
    if (c < cols) {
      raw[k].load(ar + c);
      float v[8];
      raw[k].get(v);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
  }
  const float sc = row_scale(block_max(amax, red));
  if (threadIdx.x == 0) s[r] = sc;
  const float rs = __frcp_rn(sc);
  uint8_t* qr = q + (size_t)r * cols;
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int c = (threadIdx.x + k * 256) * 8;
    if (c < cols) {
      float v[8];
      raw[k].get(v);
      *reinterpret_cast<uint2*>(qr + c) = codes8<!std::is_same<T, bf16>::value>(v, sc, rs);
    }
  }
}

// Rows longer than 256 * 8 * 8 values: two passes over the row.
template <typename T>
__global__ void __launch_bounds__(256) quant_rows_long_kernel(const T* __restrict__ a, int cols,
                                                              uint8_t* __restrict__ q, float* __restrict__ s) {
  __shared__ float red[8];
  const int r = blockIdx.x;
  const T* ar = a + (size_t)r * cols;
  float amax = 0.f;
  for (int c = threadIdx.x * 8; c < cols; c += 256 * 8) {
    float v[8];
    load8<T>(ar + c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
  const float sc = row_scale(block_max(amax, red));
  if (threadIdx.x == 0) s[r] = sc;
  const float rs = __frcp_rn(sc);
  uint8_t* qr = q + (size_t)r * cols;
  for (int c = threadIdx.x * 8; c < cols; c += 256 * 8) {
    float v[8];
    load8<T>(ar + c, v);
    *reinterpret_cast<uint2*>(qr + c) = codes8<!std::is_same<T, bf16>::value>(v, sc, rs);
  }
}

// RMSNorm of an fp32 row (gain bf16) fused with the quantization of its
// output: y = x * rstd * g in fp32, kept in registers for the amax pass and
// the codes (hidden <= 256 * 4 * RMS_MAXV, hidden % 4 == 0).
__global__ void __launch_bounds__(256) rmsnorm_quant_kernel(const float* __restrict__ x, const bf16* __restrict__ g,
                                                            int hidden, float eps, uint8_t* __restrict__ q,
                                                            float* __restrict__ s) {
  __shared__ float red[8];
  __shared__ float red2[8];
  const int h4 = hidden >> 2;
  const int r = blockIdx.x;
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
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < RMS_MAXV; ++k) {
    const int i = threadIdx.x + k * 256;
    if (i < h4) {
      const float4 gg = load_g4<bf16>(g + 4 * i);
      v[k] = make_float4(v[k].x * rstd * gg.x, v[k].y * rstd * gg.y, v[k].z * rstd * gg.z, v[k].w * rstd * gg.w);
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[k].x), fabsf(v[k].y)), fmaxf(fabsf(v[k].z), fabsf(v[k].w))));
    }
  }
  const float sc = row_scale(block_max(amax, red2));
  if (threadIdx.x == 0) s[r] = sc;
  const float rs = __frcp_rn(sc);
  uint32_t* qr = reinterpret_cast<uint32_t*>(q + (size_t)r * hidden);
#pragma unroll
  for (int k = 0; k < RMS_MAXV; ++k) {
    const int i = threadIdx.x + k * 256;
    if (i < h4)
      qr[i] = codes4(v[k], sc, rs);
  }
}

}  // namespace q8

fsdit_status launch_quant_rows(const void* a, int dtype, int rows, int cols, uint8_t* q, float* s, cudaStream_t st) {
  if (rows <= 0) return FSDIT_OK;
  ProfScope ps(PC_QUANT, 1, 0.0, (double)rows * cols * (dtype == FSDIT_BF16 ? 2.0 : 4.0) + (double)rows * (cols + 4),
               st);
  // register-resident rows of up to 2048 * CH values, CH a power of two
  const int ch = (cols + 2047) / 2048;
  auto go = [&](auto tag) {
    using T = decltype(tag);
    const T* p = (const T*)a;
    if (ch <= 1) q8::quant_rows_kernel<T, 1><<<rows, 256, 0, st>>>(p, cols, q, s);
    else if (ch <= 2) q8::quant_rows_kernel<T, 2><<<rows, 256, 0, st>>>(p, cols, q, s);
    else if (ch <= 4) q8::quant_rows_kernel<T, 4><<<rows, 256, 0, st>>>(p, cols, q, s);
    else if (ch <= 8) q8::quant_rows_kernel<T, 8><<<rows, 256, 0, st>>>(p, cols, q, s);
    else q8::quant_rows_long_kernel<T><<<rows, 256, 0, st>>>(p, cols, q, s);
  };
  if (dtype == FSDIT_BF16) go(bf16());
  else go(float());
  return cuda_check(cudaGetLastError(), "quant_rows_kernel");
}

fsdit_status launch_rmsnorm_quant(const float* x, const void* g, int rows, int hidden, float eps, uint8_t* q, float* s,
                                  cudaStream_t st) {
  if (rows <= 0) return FSDIT_OK;
  ProfScope ps(PC_NORM, 1, 0.0, (double)rows * (hidden * 5.0 + 4.0), st);
  q8::rmsnorm_quant_kernel<<<rows, 256, 0, st>>>(x, (const bf16*)g, hidden, eps, q, s);
  return cuda_check(cudaGetLastError(), "rmsnorm_quant_kernel");
}

}  // namespace fsdit
