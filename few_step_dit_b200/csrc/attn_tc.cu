// Joint attention on the sm_100a tensor cores (bf16 operands, fp32 softmax).
//
// One CTA per (256 queries, head) = two 128-row query tiles A and B sharing
// every K/V tile; 320 threads:
//   warp 0  lane 0: TMA producer.  Q_A, Q_B, K and V tiles are 128 x 128
//           boxes cut straight out of the packed qkv buffer [n, 3A] (two
//           64-column boxes each, 128-byte swizzle); K and V each go through
//           a 2-stage ring.
//   warp 1  allocates all 512 TMEM columns; lane 0 issues tcgen05.mma:
//             S_t   = Q_t K_j^T          (TMEM cols 128t .. 128t+127, fp32)
//             O_t  += P_t V_j            (TMEM cols 256+128t .., fp32)
//           where P_t is read from TMEM (it overwrites the first 64 columns of
//           S_t as packed bf16) and V is an MN-major shared-memory operand.
//           Order per key tile j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1); the
//           tensor pipe runs them in issue order, so the commit that
//           publishes S_t(j+1) also covers PV_t(j) and frees P_t(j).
//   warps 2-5 / 6-9: softmax of tile A / tile B, one thread per query row
//           (TMEM lane).  Each thread reads its S row, keeps its running max
//           m and sum l in the log2 domain, writes P = exp2(s*scale - m)
//           back into TMEM as bf16, and rescales its O row only when its max
//           grew by more than 8 (P < 2^8, exact in fp32 accumulation).  While
//           one group exponentiates, the tensor core works on the other
//           tile.  At the end O / l is stored as bf16.
// Keys past n are masked (TMA zero-fills rows past n).
#include "tc_ptx.cuh"

namespace fsdit {
namespace attn {

constexpr int BQ = 128, BKV = 128, D = 128;
constexpr int TILE_BYTES = 128 * 128 * 2;  // 32 KB: two 64-column swizzled boxes
constexpr int HALF_BYTES = TILE_BYTES / 2;
constexpr int THREADS = 320;
constexpr int OFF_Q = 0;                   // Q_A, Q_B
constexpr int OFF_K = 2 * TILE_BYTES;      // K stage s at OFF_K + s * TILE_BYTES
constexpr int OFF_V = 4 * TILE_BYTES;      // V stage s at OFF_V + s * TILE_BYTES
constexpr int OFF_BAR = 6 * TILE_BYTES;
enum { B_QFULL = 0, B_KFULL = 1, B_VFULL = 3, B_KEMPTY = 5, B_VEMPTY = 7, B_SFULL = 9, B_PFULL = 11,
       B_ODONE = 13, B_DRAIN = 15, NUM_BARS = 16 };
constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_S = ptx::idesc_bf16(BQ, BKV, 0);
constexpr uint32_t IDESC_PV = ptx::idesc_bf16(BQ, D, 1);
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Max of 128 values as eight independent chains of three-input max (depth 8
// plus a 3-level combine) instead of one 127-long dependent chain.
__device__ __forceinline__ float row_max128(const float* s) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float a = max3(s[k], s[k + 8], s[k + 16]);
#pragma unroll
    for (int i = 3; i < 15; i += 2) a = max3(a, s[k + 8 * i], s[k + 8 * (i + 1)]);
    mx[k] = fmaxf(a, s[k + 8 * 15]);
  }
  return max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// ---- packed fp32 pairs (f32x2 FMA-pipe instructions of sm_100) ----
typedef unsigned long long f2_t;
__device__ __forceinline__ f2_t f2(float a, float b) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_split(f2_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ f2_t f2_fma(f2_t a, f2_t b, f2_t c) {
  f2_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ f2_t f2_add(f2_t a, f2_t b) {
  f2_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// O (+)= P V with P [128 x 16k] in TMEM (A operand) and V in shared memory.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct Args {
  int n, heads, attn;  // attn = heads * 128
  bf16* out;           // [n, attn]
  float scale_log2;    // log2(e) / sqrt(128)
};

__global__ void __launch_bounds__(THREADS, 1)
    tc_attention_kernel(const __grid_constant__ CUtensorMap tm, const Args args) {
  using namespace ptx;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bar0 = base + OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + OFF_BAR + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int q0 = blockIdx.x * 2 * BQ;
  const int n = args.n;
  const int nkv = (n + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
      mbar_init(bar(B_SFULL + s), 1);   // per query tile
      mbar_init(bar(B_PFULL + s), 4);   // per query tile: one arrive per softmax warp
      mbar_init(bar(B_ODONE + s), 1);   // per query tile
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tm);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int cq = head * D, ck = args.attn + head * D, cv = 2 * args.attn + head * D;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int last_bar = -1;
      uint32_t last_ph = 0;
      mbar_expect_tx(bar(B_QFULL), 2 * TILE_BYTES);
      for (int t = 0; t < 2; ++t) {
        tma_load_2d(base + OFF_Q + t * TILE_BYTES, &tm, cq, q0 + t * BQ, bar(B_QFULL));
        tma_load_2d(base + OFF_Q + t * TILE_BYTES + HALF_BYTES, &tm, cq + 64, q0 + t * BQ, bar(B_QFULL));
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        const uint32_t sk = base + OFF_K + st * TILE_BYTES, sv = base + OFF_V + st * TILE_BYTES;
        if (!mbar_wait(bar(B_KEMPTY + st), ph ^ 1u, abort_flag)) { ok = false; break; }
        mbar_expect_tx(bar(B_KFULL + st), TILE_BYTES);
        tma_load_2d(sk, &tm, ck, j * BKV, bar(B_KFULL + st));
        tma_load_2d(sk + HALF_BYTES, &tm, ck + 64, j * BKV, bar(B_KFULL + st));
        if (!mbar_wait(bar(B_VEMPTY + st), ph ^ 1u, abort_flag)) { ok = false; break; }
        mbar_expect_tx(bar(B_VFULL + st), TILE_BYTES);
        tma_load_2d(sv, &tm, cv, j * BKV, bar(B_VFULL + st));
        tma_load_2d(sv + HALF_BYTES, &tm, cv + 64, j * BKV, bar(B_VFULL + st));
        last_bar = B_VFULL + st;
        last_ph = ph;
      }
      if (!ok && last_bar >= 0) mbar_wait(bar(last_bar), last_ph, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(bar(B_QFULL), 0, abort_flag);
      // S_t(j) = Q_t K_j^T into TMEM columns 128t
      auto issue_s = [&](int t, int j) {
        const uint32_t sk = base + OFF_K + (j & 1) * TILE_BYTES;
        const uint32_t sq = base + OFF_Q + t * TILE_BYTES;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (uint32_t)((k >> 2) * HALF_BYTES + (k & 3) * 32);
          mma_bf16_ss(tmem + (uint32_t)(t * BKV), sw128_desc(sq + off, 16, 1024), sw128_desc(sk + off, 16, 1024),
                      IDESC_S, k > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_SFULL + t));
      };
      // O_t += P_t(j) V_j, P_t in TMEM columns 128t .. 128t+63 (packed bf16)
      auto issue_pv = [&](int t, int j) {
        const uint32_t sv = base + OFF_V + (j & 1) * TILE_BYTES;
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          mma_bf16_ts(tmem + 256u + (uint32_t)(t * D), tmem + (uint32_t)(t * BKV + k * 8),
                      sw128_desc(sv + (uint32_t)(k * 2048), HALF_BYTES, 1024), IDESC_PV, (j > 0 || k > 0) ? 1u : 0u);
      };
      if (ok) ok = mbar_wait(bar(B_KFULL), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        tc_commit(bar(B_KEMPTY));
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        const bool more = j + 1 < nkv;
        if (!mbar_wait(bar(B_VFULL + st), ph, abort_flag)) { ok = false; break; }
        if (more && !mbar_wait(bar(B_KFULL + (st ^ 1)), (uint32_t)((j + 1) >> 1) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        for (int t = 0; t < 2; ++t) {
          if (!mbar_wait(bar(B_PFULL + t), (uint32_t)j & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_pv(t, j);
          if (more) issue_s(t, j + 1);
          else tc_commit(bar(B_ODONE + t));
        }
        if (!ok) break;
        tc_commit(bar(B_VEMPTY + st));
        if (more) tc_commit(bar(B_KEMPTY + (st ^ 1)));
      }
      // every MMA this thread issued has completed once B_DRAIN flips
      tc_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, nullptr);
    }
  } else {
    // softmax warpgroups: tile t, thread <-> query row r of the tile (TMEM lane r)
    const int t = (warp - 2) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const uint32_t s_col = (uint32_t)(t * BKV);
    const uint32_t o_col = 256u + (uint32_t)(t * D);
    const float sl2 = args.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait(bar(B_SFULL + t), (uint32_t)j & 1u, abort_flag) ? 1 : 0;
      w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
      if (!w_ok) { ok = false; break; }
      tc_fence_after();
      float s[BKV];
      tmem_ld128(tmem + lane_addr + s_col, s);
      const int valid = n - j * BKV;  // keys past n are masked
      if (valid < BKV) {
#pragma unroll
        for (int c = 0; c < BKV; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      const float m_cand = row_max128(s) * sl2;
      const bool grow = m_cand > m + RESCALE_THRESHOLD;
      const float m_new = grow ? m_cand : m;
      const float corr = grow ? ex2(m - m_new) : 1.0f;
      // O_t is stable here: PV_t(j-1) completed before S_t(j) did
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          const uint32_t ta = tmem + lane_addr + o_col + (uint32_t)(c * 32);
          tmem_ld32(ta, o);
          uint32_t u[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(o[i] * corr);
          tmem_st32(ta, u);
        }
      }
      const f2_t scale2 = f2(sl2, sl2), negm2 = f2(-m_new, -m_new);
      f2_t acc[4] = {0ull, 0ull, 0ull, 0ull};  // four independent partial row sums (pairs)
      uint32_t pk[BKV / 2];
#pragma unroll
      for (int c = 0; c < BKV; c += 2) {
        float x0, x1;
        f2_split(f2_fma(f2(s[c], s[c + 1]), scale2, negm2), x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        acc[(c >> 1) & 3] = f2_add(acc[(c >> 1) & 3], f2(p0, p1));
        pk[c >> 1] = pack_bf16(p0, p1);
      }
      tmem_st64(tmem + lane_addr + s_col, pk);
      float a0, a1;
      f2_split(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
      const float sum = a0 + a1;
      l = l * corr + sum;
      m = m_new;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PFULL + t));
    }
    if (ok && nkv > 0) {
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait(bar(B_ODONE + t), 0, abort_flag) ? 1 : 0;
      w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
      if (w_ok) {
        tc_fence_after();
        const int row = q0 + t * BQ + r;
        const float inv = 1.0f / l;
        bf16* orow = args.out + (size_t)row * args.attn + head * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tmem + lane_addr + o_col + (uint32_t)(c * 32), o);
          if (row < n) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 v = make_uint4(pack_bf16(o[i] * inv, o[i + 1] * inv), pack_bf16(o[i + 2] * inv, o[i + 3] * inv),
                                   pack_bf16(o[i + 4] * inv, o[i + 5] * inv), pack_bf16(o[i + 6] * inv, o[i + 7] * inv));
              *reinterpret_cast<uint4*>(orow + c * 32 + i) = v;
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace attn


fsdit_status launch_attention_tc(const void* qkv, void* out, int n, int heads, int attn_w, cudaStream_t st) {
  using namespace attn;
  static PerDevice<cudaError_t> attr;
  const cudaError_t attr_err = attr.get(
      [] { return cudaFuncSetAttribute(tc_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES); },
      cudaErrorInvalidDevice);
  if (attr_err != cudaSuccess) return cuda_check(attr_err, "cudaFuncSetAttribute(tc_attention_kernel)");
  CUtensorMap tm;
  fsdit_status s = make_tmap_bf16(&tm, qkv, (uint64_t)n, (uint64_t)3 * attn_w, (uint64_t)3 * attn_w, BQ, 64);
  if (s != FSDIT_OK) return s;
  Args a;
  a.n = n;
  a.heads = heads;
  a.attn = attn_w;
  a.out = reinterpret_cast<bf16*>(out);
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  dim3 grid((n + 2 * BQ - 1) / (2 * BQ), heads);
  tc_attention_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tm, a);
  return cuda_check(cudaGetLastError(), "tc_attention_kernel");
}

}  // namespace fsdit
